// Peer buffers of a real Nd-rank job (include/zero_peer.h): CUDA IPC
// descriptors that let rank r's step load the other ranks' gradients and store
// into their fp16 parameter buffers ([P1] "The part that sounds too good:
// communication": the reduce-scatter and all-gather of stages 1 and 2).
//
// Host code only. The allocation holding a buffer is found with the driver's
// address-range query, reached through the runtime's entry-point lookup so
// that the library needs no link-time dependency on the driver library.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <unistd.h>

#include <array>
#include <chrono>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <random>
#include <utility>

#include "zero_peer.h"

#define ZERO_API extern "C" __attribute__((visibility("default")))

static_assert(sizeof(cudaIpcMemHandle_t) == 64, "IPC handle size");
static_assert(sizeof(zero_peer_desc) == 104, "descriptor layout");

namespace {

std::mutex g_mu;
int g_last_cuda = 0;

struct Mapping {
    void* base;
    int refs;
};
// (importing device, IPC handle bytes) -> mapping of that allocation
using Key = std::pair<int, std::array<unsigned char, 64>>;
std::map<Key, Mapping> g_maps;

uint64_t random_word()
{
    uint64_t r = 0;
    try {
        std::random_device rd;
        r = (uint64_t(rd()) << 32) ^ uint64_t(rd());
    } catch (...) {
        r = uint64_t(std::chrono::steady_clock::now().time_since_epoch().count());
    }
    return r;
}

// A token of the calling process: random per load of the library, mixed with
// the pid so that a forked child does not pass for its parent.
uint64_t process_token()
{
    static const uint64_t r = random_word();
    uint64_t t = r ^ (uint64_t(getpid()) * 0x9E3779B97F4A7C15ull);
    return t ? t : 1;
}

int fail_cuda(cudaError_t e)
{
    std::lock_guard<std::mutex> g(g_mu);
    g_last_cuda = int(e);
    (void)cudaGetLastError();  // leave no error behind for the caller's next check
    return ZERO_ERR_CUDA;
}

int fail_driver(int code)
{
    std::lock_guard<std::mutex> g(g_mu);
    g_last_cuda = code;
    return ZERO_ERR_CUDA;
}

PFN_cuMemGetAddressRange_v3020 address_range()
{
    static const PFN_cuMemGetAddressRange_v3020 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            p = nullptr;
        }
        return reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(p);
    }();
    return fn;
}

bool desc_ok(const zero_peer_desc* d)
{
    return d && d->magic == ZERO_PEER_MAGIC && d->bytes > 0 && d->offset + d->bytes > d->offset &&
           (d->address & 15) == 0 && (d->offset & 15) == 0;
}

Key key_of(int device, const zero_peer_desc* d)
{
    Key k;
    k.first = device;
    std::memcpy(k.second.data(), d->ipc, 64);
    return k;
}

}  // namespace

ZERO_API int zero_peer_export(const void* dev_ptr, size_t bytes, zero_peer_desc* out)
{
    if (!dev_ptr || !out || bytes == 0 || bytes > (size_t(1) << 62)) return ZERO_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(dev_ptr) & 15) return ZERO_ERR_ALIGN;
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, dev_ptr);
    if (e != cudaSuccess) return fail_cuda(e);
    if (attr.type != cudaMemoryTypeDevice) return ZERO_ERR_ARG;
    PFN_cuMemGetAddressRange_v3020 range = address_range();
    if (!range) return fail_cuda(cudaErrorNotSupported);
    CUdeviceptr base = 0;
    size_t size = 0;
    const CUdeviceptr p = CUdeviceptr(reinterpret_cast<uintptr_t>(dev_ptr));
    const CUresult r = range(&base, &size, p);
    if (r != CUDA_SUCCESS) return fail_driver(int(r));
    const uint64_t off = uint64_t(p - base);
    if (p < base || off + bytes > size) return ZERO_ERR_ARG;
    cudaIpcMemHandle_t h;
    e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
    if (e != cudaSuccess) return fail_cuda(e);
    zero_peer_desc d;
    std::memset(&d, 0, sizeof d);
    d.magic = ZERO_PEER_MAGIC;
    d.device = attr.device;
    d.process = process_token();
    d.offset = off;
    d.bytes = uint64_t(bytes);
    d.address = uint64_t(reinterpret_cast<uintptr_t>(dev_ptr));
    std::memcpy(d.ipc, &h, 64);
    *out = d;
    return ZERO_OK;
}

ZERO_API int zero_peer_open(const zero_peer_desc* desc, void** dev_ptr)
{
    if (!desc_ok(desc) || !dev_ptr) return ZERO_ERR_ARG;
    if (desc->process == process_token()) {  // this process's own buffer
        *dev_ptr = reinterpret_cast<void*>(uintptr_t(desc->address));
        return ZERO_OK;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda(e);
    std::unique_lock<std::mutex> g(g_mu);
    const Key k = key_of(dev, desc);
    auto it = g_maps.find(k);
    void* base = nullptr;
    if (it != g_maps.end()) {
        it->second.refs += 1;
        base = it->second.base;
    } else {
        cudaIpcMemHandle_t h;
        std::memcpy(&h, desc->ipc, 64);
        e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
        if (e != cudaSuccess) {
            g.unlock();
            return fail_cuda(e);
        }
        g_maps.emplace(k, Mapping{base, 1});
    }
    *dev_ptr = static_cast<char*>(base) + desc->offset;
    return ZERO_OK;
}

ZERO_API int zero_peer_close(const zero_peer_desc* desc, void* dev_ptr)
{
    if (!desc_ok(desc) || !dev_ptr) return ZERO_ERR_ARG;
    if (desc->process == process_token())
        return dev_ptr == reinterpret_cast<void*>(uintptr_t(desc->address)) ? ZERO_OK : ZERO_ERR_ARG;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda(e);
    std::unique_lock<std::mutex> g(g_mu);
    auto it = g_maps.find(key_of(dev, desc));
    if (it == g_maps.end() || static_cast<char*>(it->second.base) + desc->offset != dev_ptr) return ZERO_ERR_ARG;
    if (--it->second.refs > 0) return ZERO_OK;
    void* base = it->second.base;
    g_maps.erase(it);
    g.unlock();
    e = cudaIpcCloseMemHandle(base);
    return e == cudaSuccess ? ZERO_OK : fail_cuda(e);
}

ZERO_API int zero_peer_open_count(void)
{
    std::lock_guard<std::mutex> g(g_mu);
    return int(g_maps.size());
}

ZERO_API int zero_peer_last_cuda_error(void)
{
    std::lock_guard<std::mutex> g(g_mu);
    return g_last_cuda;
}

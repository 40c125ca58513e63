// The offloaded step (include/zero_offload.h): fp32 master/m/v in host memory,
// Adam on the host cores, the cross-rank gradient sum and the fp16 write-back
// on the GPU, chunks pipelined over PCIe.
//
// Per step:
//   s_red : overflow check over every gradient element (read-only pass), then
//           per chunk the unscaled reduced gradient into a device slot
//   s_d2h : slot -> page-locked host slot
//   host  : Adam on the chunk (thread pool), fp16 of the new master into a
//           page-locked host slot
//   s_h2d : host fp16 slot -> device fp16 slot
//   s_bc  : device fp16 slot -> the Nd replicas (stage 1/2) or the shards
// Slots are reused every ZERO_OFFLOAD_SLOTS chunks; events order each reuse
// after the last reader of the slot. The device passes are HBM-light next to
// the PCIe transfers and the host update, so their kernels are plain
// grid-stride loops.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <condition_variable>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#if defined(__x86_64__)
#include <xmmintrin.h>
#endif

#include "zero.h"
#include "zero_device.cuh"
#include "zero_host_adam.h"
#include "zero_internal.h"
#include "zero_layout.h"
#include "zero_nvtx.h"
#include "zero_offload.h"

#define ZERO_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int S = ZERO_OFFLOAD_SLOTS;
constexpr int64_t kAlignB = 256;
constexpr int kBlock = 256;

int64_t up(int64_t x) { return (x + kAlignB - 1) / kAlignB * kAlignB; }

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A piece of a run inside one chunk: local indices [local_begin, local_begin
// + len) of the chunk map to gradient index grad_begin + (j - local_begin) and
// output index out_begin + (j - local_begin).
struct OffRun {
    long long grad_begin;
    long long local_begin;
    long long out_begin;
    long long len;
    int decay;
    int pad;
};

// ---------------- device ----------------

__device__ __forceinline__ int find_off(const OffRun* runs, int n, long long j)
{
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (runs[mid].local_begin <= j)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

template <class T>
__device__ __forceinline__ void load_table(T* const* src, int n, T** dst)
{
    for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src[i];
    __syncthreads();
}

// Overflow check of the whole step: every gradient element is summed over the
// ranks in order, unscaled and tested. Nothing is written but the flag.
__global__ void __launch_bounds__(kBlock) off_check_kernel(const uint16_t* const* grads, int nd, long long n,
                                                           float inv, unsigned* flag)
{
    extern __shared__ const uint16_t* s_g[];
    load_table(grads, nd, s_g);
    bool bad = false;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nq = n / 4;  // quads: 8-byte loads (the buffers are 16-byte aligned)
    for (long long q = tid; q < nq; q += stride) {
        float s[4], x[4];
        zk::unpack(__ldcs(reinterpret_cast<const uint2*>(s_g[0]) + q), s);
        for (int r = 1; r < nd; ++r) {
            zk::unpack(__ldcs(reinterpret_cast<const uint2*>(s_g[r]) + q), x);
#pragma unroll
            for (int i = 0; i < 4; ++i) s[i] = __fadd_rn(s[i], x[i]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) bad |= zk::nonfinite(__fmul_rn(s[i], inv));
    }
    for (long long i = nq * 4 + tid; i < n; i += stride) {
        float s = zk::h2f(s_g[0][i]);
        for (int r = 1; r < nd; ++r) s = __fadd_rn(s, zk::h2f(s_g[r][i]));
        bad |= zk::nonfinite(__fmul_rn(s, inv));
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(flag, 1u);
}

// The unscaled reduced gradient of one chunk, in the chunk's local order.
__global__ void __launch_bounds__(kBlock) off_reduce_kernel(const OffRun* runs, int n_runs, long long len,
                                                            const uint16_t* const* grads, int nd, float inv,
                                                            float* red)
{
    extern __shared__ const uint16_t* s_g[];
    load_table(grads, nd, s_g);
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long j = (long long)blockIdx.x * blockDim.x + threadIdx.x; j < len; j += stride) {
        const OffRun& r = runs[find_off(runs, n_runs, j)];
        const long long gi = r.grad_begin + (j - r.local_begin);
        float s = zk::h2f(__ldcs(s_g[0] + gi));
        for (int k = 1; k < nd; ++k) s = __fadd_rn(s, zk::h2f(__ldcs(s_g[k] + gi)));
        __stcs(red + j, __fmul_rn(s, inv));
    }
}

// One chunk of fp16 parameters to every output.
__global__ void __launch_bounds__(kBlock) off_bcast_kernel(const OffRun* runs, int n_runs, long long len,
                                                           const uint16_t* src, uint16_t* const* outs, int n_out)
{
    extern __shared__ uint16_t* s_o[];
    load_table(outs, n_out, s_o);
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long j = (long long)blockIdx.x * blockDim.x + threadIdx.x; j < len; j += stride) {
        const OffRun& r = runs[find_off(runs, n_runs, j)];
        const long long oi = r.out_begin + (j - r.local_begin);
        const uint16_t h = __ldcs(src + j);
        for (int k = 0; k < n_out; ++k) __stcs(s_o[k] + oi, h);
    }
}

// ---------------- host: sizes ----------------

struct OffLayout {
    int64_t E = 0, C = 0, n_chunks = 0;
    // device
    int64_t d_flag = 0, d_grad_tab = 0, d_out_tab = 0, d_runs = 0, d_gather = 0, d_red[S] = {}, d_p16[S] = {},
            d_total = 0;
    // host staging
    int64_t h_flag = 0, h_grad_tab = 0, h_out_tab = 0, h_red[S] = {}, h_p16[S] = {}, h_total = 0;
    // chunk tables
    std::vector<OffRun> runs;          // all chunks' pieces, chunk after chunk
    std::vector<int64_t> chunk_run0;   // n_chunks + 1
};

int off_layout(const zl::Layout& L, int64_t chunk_elems, OffLayout* O)
{
    if (L.bf16) return ZERO_ERR_ARG;  // the offloaded step keeps an fp32 master
    if (L.stage == 3 && L.view >= 0) return ZERO_ERR_ARG;  // no offloaded stage-3 rank of a real job
    O->E = L.state_elems;
    if (chunk_elems == 0) {
        // at most ZERO_OFFLOAD_DEFAULT_CHUNK, and at least 8 chunks for
        // states above 8 Mi elements so the pipeline overlaps
        chunk_elems = std::min<int64_t>(ZERO_OFFLOAD_DEFAULT_CHUNK,
                                        std::max<int64_t>(1 << 20, (O->E / 8 + 255) / 256 * 256));
    } else if (chunk_elems < 256 || chunk_elems > (int64_t(1) << 30) || chunk_elems % 256 != 0) {
        return ZERO_ERR_ARG;
    }
    O->C = std::min<int64_t>(chunk_elems, std::max<int64_t>(256, (O->E + 255) / 256 * 256));
    O->n_chunks = (O->E + O->C - 1) / O->C;
    // the run table must tile the state index space in order
    int64_t expect = 0;
    for (const zk::SegDesc& d : L.step_segs) {
        if (d.state_begin != expect) return ZERO_ERR_INTERNAL;
        expect += d.len;
    }
    if (expect != O->E) return ZERO_ERR_INTERNAL;
    O->chunk_run0.assign(1, 0);
    size_t r = 0;
    for (int64_t k = 0; k < O->n_chunks; ++k) {
        const int64_t c0 = k * O->C, c1 = std::min(O->E, c0 + O->C);
        while (r < L.step_segs.size() && L.step_segs[r].state_begin + L.step_segs[r].len <= c0) ++r;
        for (size_t i = r; i < L.step_segs.size() && L.step_segs[i].state_begin < c1; ++i) {
            const zk::SegDesc& d = L.step_segs[i];
            const int64_t lo = std::max<int64_t>(d.state_begin, c0);
            const int64_t hi = std::min<int64_t>(d.state_begin + d.len, c1);
            if (hi <= lo) continue;
            OffRun o{};
            o.grad_begin = d.grad_begin + (lo - d.state_begin);
            o.local_begin = lo - c0;
            o.out_begin = d.out_begin + (lo - d.state_begin);
            o.len = hi - lo;
            o.decay = d.decay;
            O->runs.push_back(o);
        }
        O->chunk_run0.push_back((int64_t)O->runs.size());
    }
    int64_t off = 0;
    O->d_flag = off;
    off += kAlignB;
    O->d_grad_tab = off;
    off += up((int64_t)L.nd * 8);
    O->d_out_tab = off;
    off += up((int64_t)std::max(L.n_out, 1) * 8);
    O->d_runs = off;
    off += up((int64_t)std::max<size_t>(O->runs.size(), 1) * sizeof(OffRun));
    O->d_gather = off;  // stage 3: the layer-gather run table (shard index -> unit index)
    off += up((int64_t)L.gather_segs.size() * sizeof(zk::SegDesc));
    for (int s = 0; s < S; ++s) {
        O->d_red[s] = off;
        off += up(4 * O->C);
    }
    for (int s = 0; s < S; ++s) {
        O->d_p16[s] = off;
        off += up(2 * O->C);
    }
    O->d_total = off;
    off = 0;
    O->h_flag = off;
    off += kAlignB;
    O->h_grad_tab = off;
    off += up((int64_t)L.nd * 8);
    O->h_out_tab = off;
    off += up((int64_t)std::max(L.n_out, 1) * 8);
    for (int s = 0; s < S; ++s) {
        O->h_red[s] = off;
        off += up(4 * O->C);
    }
    for (int s = 0; s < S; ++s) {
        O->h_p16[s] = off;
        off += up(2 * O->C);
    }
    O->h_total = off;
    return ZERO_OK;
}

void fill_off_ledger(const zl::Layout& L, const OffLayout& O, zero_offload_ledger* out)
{
    std::memset(out, 0, sizeof(*out));
    out->state_elems = O.E;
    out->host_state_bytes = 12 * O.E;
    out->host_staging_bytes = O.h_total;
    out->device_bytes = O.d_total;
    out->chunk_elems = O.C;
    out->n_chunks = O.n_chunks;
    out->d2h_bytes_per_step = 4 * O.E;
    out->h2d_bytes_per_step = 2 * O.E;
    int64_t max_part = 0, max_shard = 0;
    for (int r = 0; r < L.nd; ++r) {
        int64_t b, e;
        zl::split(L.psi, L.nd, r, &b, &e);
        max_part = std::max(max_part, e - b);
        int64_t s = 0;
        for (int64_t n : L.numel) {
            int64_t cb, ce;
            zl::split(n, L.nd, r, &cb, &ce);
            s += ce - cb;
        }
        max_shard = std::max(max_shard, s);
    }
    out->device_state_bytes = L.stage == 1 ? 4 * L.psi : L.stage == 2 ? 2 * L.psi + 2 * max_part : 4 * max_shard;
    out->n_out = L.n_out;
}

// ---------------- host: thread pool of the update ----------------

#if defined(__x86_64__)
// The update assumes the default binary32 environment: round to nearest, no
// flush-to-zero, no denormals-are-zero.
struct DefaultFpEnv {
    unsigned saved;
    DefaultFpEnv() : saved(_mm_getcsr()) { _mm_setcsr(0x1f80u); }
    ~DefaultFpEnv() { _mm_setcsr(saved); }
};
#else
struct DefaultFpEnv {};
#endif

class Pool {
public:
    explicit Pool(int n) : n_(n)
    {
        for (int i = 1; i < n; ++i) th_.emplace_back([this, i] { work(i); });
    }
    ~Pool()
    {
        {
            std::lock_guard<std::mutex> g(mu_);
            stop_ = true;
        }
        cv_.notify_all();
        for (auto& t : th_) t.join();
    }
    int size() const { return n_; }
    // Run f(i) for i = 0 .. n-1, i = 0 on the calling thread; returns when all are done.
    void run(const std::function<void(int)>& f)
    {
        {
            std::lock_guard<std::mutex> g(mu_);
            job_ = &f;
            left_ = n_ - 1;
            ++gen_;
        }
        cv_.notify_all();
        {
            DefaultFpEnv env;
            f(0);
        }
        std::unique_lock<std::mutex> lk(mu_);
        done_.wait(lk, [this] { return left_ == 0; });
        job_ = nullptr;
    }

private:
    void work(int i)
    {
        DefaultFpEnv env;
        uint64_t seen = 0;
        for (;;) {
            const std::function<void(int)>* f;
            {
                std::unique_lock<std::mutex> lk(mu_);
                cv_.wait(lk, [&] { return stop_ || gen_ != seen; });
                if (stop_) return;
                seen = gen_;
                f = job_;
            }
            (*f)(i);
            {
                std::lock_guard<std::mutex> g(mu_);
                if (--left_ == 0) done_.notify_one();
            }
        }
    }
    int n_;
    std::vector<std::thread> th_;
    std::mutex mu_;
    std::condition_variable cv_, done_;
    const std::function<void(int)>* job_ = nullptr;
    int left_ = 0;
    uint64_t gen_ = 0;
    bool stop_ = false;
};

using AdamFn = void (*)(const float*, float*, float*, float*, uint16_t*, int64_t, const ZhCoef*, float);
using CastFn = void (*)(const float*, uint16_t*, int64_t);

bool cpu_has_avx2()
{
#if defined(__x86_64__)
    __builtin_cpu_init();
    return __builtin_cpu_supports("avx2") && __builtin_cpu_supports("f16c");
#else
    return false;
#endif
}

void bias_corr(float b1, float b2, int64_t t, float* bc1, float* bc2)
{
    double p1 = 1.0, p2 = 1.0;
    for (int64_t k = 0; k < t; ++k) {
        p1 = p1 * (double)b1;
        p2 = p2 * (double)b2;
    }
    *bc1 = (float)(1.0 - p1);
    *bc2 = (float)(1.0 - p2);
}

ZhCoef make_coef(const zero_hyper* hp, int64_t t)
{
    ZhCoef c;
    c.lr = hp->lr;
    c.b1 = hp->beta1;
    c.b2 = hp->beta2;
    c.omb1 = 1.0f - hp->beta1;
    c.omb2 = 1.0f - hp->beta2;
    c.eps = hp->eps;
    bias_corr(hp->beta1, hp->beta2, t, &c.bc1, &c.bc2);
    return c;
}

}  // namespace

struct zero_offload_handle {
    zl::Layout L;
    OffLayout O;
    char* dws = nullptr;
    char* hst = nullptr;  // page-locked staging
    float* w = nullptr;
    float* m = nullptr;
    float* v = nullptr;
    Pool* pool = nullptr;
    AdamFn adam = nullptr;
    CastFn cast = nullptr;
    cudaStream_t s_red = nullptr, s_d2h = nullptr, s_h2d = nullptr, s_bc = nullptr;
    cudaEvent_t ev_start = nullptr, ev_end = nullptr, ev_flag = nullptr;
    cudaEvent_t ev_red[S] = {}, ev_d2h[S] = {}, ev_h2d[S] = {}, ev_bc[S] = {};
    int sms = 0;
    int64_t t = 0;
    bool broken = false;
    int last_cuda = 0;

    float* d_red(int s) const { return reinterpret_cast<float*>(dws + O.d_red[s]); }
    uint16_t* d_p16(int s) const { return reinterpret_cast<uint16_t*>(dws + O.d_p16[s]); }
    float* h_red(int s) const { return reinterpret_cast<float*>(hst + O.h_red[s]); }
    uint16_t* h_p16(int s) const { return reinterpret_cast<uint16_t*>(hst + O.h_p16[s]); }
    const OffRun* d_runs() const { return reinterpret_cast<const OffRun*>(dws + O.d_runs); }
    const zk::SegDesc* d_gather() const { return reinterpret_cast<const zk::SegDesc*>(dws + O.d_gather); }
    uint16_t* shards = nullptr;  // stage 3: the fp16 shard buffer (param_bufs[0])
    int occ_gather = 0;
    const uint16_t* const* d_grad_tab() const { return reinterpret_cast<const uint16_t* const*>(dws + O.d_grad_tab); }
    uint16_t* const* d_out_tab() const { return reinterpret_cast<uint16_t* const*>(dws + O.d_out_tab); }
    unsigned* d_flag() const { return reinterpret_cast<unsigned*>(dws + O.d_flag); }
    int64_t chunk_begin(int64_t k) const { return k * O.C; }
    int64_t chunk_len(int64_t k) const { return std::min(O.E, (k + 1) * O.C) - k * O.C; }
    int grid(int64_t n) const
    {
        const int64_t want = (n + kBlock - 1) / kBlock;
        return (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8));
    }
};

namespace {

void release(zero_offload_handle* h)
{
    if (!h) return;
    cudaStream_t ss[4] = {h->s_red, h->s_d2h, h->s_h2d, h->s_bc};
    for (cudaStream_t s : ss)
        if (s) cudaStreamSynchronize(s);
    cudaEvent_t one[3] = {h->ev_start, h->ev_end, h->ev_flag};
    for (cudaEvent_t e : one)
        if (e) cudaEventDestroy(e);
    for (int s = 0; s < S; ++s) {
        cudaEvent_t es[4] = {h->ev_red[s], h->ev_d2h[s], h->ev_h2d[s], h->ev_bc[s]};
        for (cudaEvent_t e : es)
            if (e) cudaEventDestroy(e);
    }
    for (cudaStream_t s : ss)
        if (s) cudaStreamDestroy(s);
    delete h->pool;
    delete h;
}

int fail(zero_offload_handle* h, cudaError_t e)
{
    h->last_cuda = (int)e;
    h->broken = true;
    return ZERO_ERR_CUDA;
}

// Split the chunk's pieces over the pool: thread i takes local indices
// [lo_i, hi_i) (multiples of 64 elements) and calls f(piece, from, to) for
// each overlap with a piece, from/to local to the chunk.
template <class F>
void for_chunk(zero_offload_handle* h, int64_t k, F f)
{
    const OffRun* runs = h->O.runs.data() + h->O.chunk_run0[k];
    const int n_runs = (int)(h->O.chunk_run0[k + 1] - h->O.chunk_run0[k]);
    const int64_t len = h->chunk_len(k);
    const int n = h->pool->size();
    const std::function<void(int)> job = [&](int i) {
        const int64_t per = ((len + n - 1) / n + 63) / 64 * 64;
        const int64_t lo = std::min(len, (int64_t)i * per), hi = std::min(len, lo + per);
        for (int r = 0; r < n_runs && lo < hi; ++r) {
            const int64_t a = std::max<int64_t>(lo, runs[r].local_begin);
            const int64_t b = std::min<int64_t>(hi, runs[r].local_begin + runs[r].len);
            if (b > a) f(runs[r], a, b);
        }
    };
    h->pool->run(job);
}

// Enqueue the fp16 upload of chunk k from host slot s and its broadcast.
cudaError_t upload_chunk(zero_offload_handle* h, int64_t k, int s)
{
    const int64_t len = h->chunk_len(k);
    cudaError_t e = cudaStreamWaitEvent(h->s_h2d, h->ev_bc[s], 0);  // device slot free
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(h->d_p16(s), h->h_p16(s), 2 * len, cudaMemcpyHostToDevice, h->s_h2d);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_h2d[s], h->s_h2d);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->s_bc, h->ev_h2d[s], 0);
    if (e == cudaSuccess) {
        const int n_runs = (int)(h->O.chunk_run0[k + 1] - h->O.chunk_run0[k]);
        off_bcast_kernel<<<h->grid(len), kBlock, h->L.n_out * sizeof(void*), h->s_bc>>>(
            h->d_runs() + h->O.chunk_run0[k], n_runs, len, h->d_p16(s), h->d_out_tab(), h->L.n_out);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_bc[s], h->s_bc);
    return e;
}

// Enqueue the reduce of chunk k into device slot s and its download.
cudaError_t download_chunk(zero_offload_handle* h, int64_t k, int s, float inv)
{
    const int64_t len = h->chunk_len(k);
    const int n_runs = (int)(h->O.chunk_run0[k + 1] - h->O.chunk_run0[k]);
    off_reduce_kernel<<<h->grid(len), kBlock, h->L.nd * sizeof(void*), h->s_red>>>(
        h->d_runs() + h->O.chunk_run0[k], n_runs, len, h->d_grad_tab(), h->L.nd, inv, h->d_red(s));
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_red[s], h->s_red);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->s_d2h, h->ev_red[s], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(h->h_red(s), h->d_red(s), 4 * len, cudaMemcpyDeviceToHost, h->s_d2h);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_d2h[s], h->s_d2h);
    return e;
}

// Write the host state chunk by chunk with fill(piece, chunk begin, from, to)
// on the pool, upload the fp16 of each chunk's master and broadcast it; the
// caller's stream waits for the last broadcast, and so does the host.
template <class F>
cudaError_t fill_state(zero_offload_handle* h, cudaStream_t cs, F fill)
{
    cudaError_t e = cudaEventRecord(h->ev_start, cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->s_bc, h->ev_start, 0);
    for (int64_t k = 0; k < h->O.n_chunks && e == cudaSuccess; ++k) {
        const int s = (int)(k % S);
        e = cudaEventSynchronize(h->ev_h2d[s]);  // host slot s free
        if (e != cudaSuccess) break;
        const int64_t c0 = h->chunk_begin(k);
        uint16_t* p16 = h->h_p16(s);
        for_chunk(h, k, [&](const OffRun& r, int64_t a, int64_t b) {
            fill(r, c0, a, b);
            h->cast(h->w + c0 + a, p16 + a, b - a);
        });
        e = upload_chunk(h, k, s);
    }
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_end, h->s_bc);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, h->ev_end, 0);
    if (e == cudaSuccess) e = cudaEventSynchronize(h->ev_end);
    return e;
}

}  // namespace

ZERO_API int zero_offload_bytes(const zero_config* cfg, int64_t chunk_elems, zero_offload_ledger* out)
{
    if (!out) return ZERO_ERR_ARG;
    zl::Layout L;
    int rc = zl::build_layout(cfg, &L);
    if (rc != ZERO_OK) return rc;
    OffLayout O;
    rc = off_layout(L, chunk_elems, &O);
    if (rc != ZERO_OK) return rc;
    fill_off_ledger(L, O, out);
    return ZERO_OK;
}

ZERO_API int zero_offload_init(const zero_config* cfg, int64_t chunk_elems, void* device_ws, size_t device_bytes,
                               void* host_staging, size_t staging_bytes, float* host_state,
                               const float* master_init, uint16_t* const* param_bufs, int n_threads, void* stream,
                               zero_offload_handle** out)
{
    if (!out) return ZERO_ERR_ARG;
    *out = nullptr;
    zero_offload_handle* h = new (std::nothrow) zero_offload_handle();
    if (!h) return ZERO_ERR_INTERNAL;
    int rc = zl::build_layout(cfg, &h->L);
    if (rc == ZERO_OK) rc = off_layout(h->L, chunk_elems, &h->O);
    const zl::Layout& L = h->L;
    const OffLayout& O = h->O;
    if (rc == ZERO_OK) {
        if (!device_ws || !host_staging || !host_state || !param_bufs || (!master_init && O.E > 0) ||
            n_threads < 1 || n_threads > 256)
            rc = ZERO_ERR_ARG;
        else if (!al16(device_ws) || !al16(host_staging))
            rc = ZERO_ERR_ALIGN;
        else if ((int64_t)device_bytes < O.d_total || (int64_t)staging_bytes < O.h_total)
            rc = ZERO_ERR_WORKSPACE;
    }
    for (int k = 0; rc == ZERO_OK && k < L.n_out; ++k) {
        if (!param_bufs[k]) rc = ZERO_ERR_ARG;
        else if (!al16(param_bufs[k])) rc = ZERO_ERR_ALIGN;
    }
    if (rc == ZERO_OK) {
        cudaPointerAttributes at{};
        if (cudaPointerGetAttributes(&at, host_staging) != cudaSuccess || at.type != cudaMemoryTypeHost) {
            cudaGetLastError();
            rc = ZERO_ERR_ARG;  // staging must be page-locked for asynchronous copies
        }
    }
    if (rc != ZERO_OK) {
        delete h;
        return rc;
    }
    h->dws = static_cast<char*>(device_ws);
    h->hst = static_cast<char*>(host_staging);
    h->w = host_state;
    h->m = host_state + O.E;
    h->v = host_state + 2 * O.E;
    const bool avx2 = cpu_has_avx2();
    h->adam = avx2 ? zh_adam_avx2 : zh_adam_base;
    h->cast = avx2 ? zh_cast_avx2 : zh_cast_base;
    h->pool = new (std::nothrow) Pool(n_threads);
    if (!h->pool) {
        delete h;
        return ZERO_ERR_INTERNAL;
    }

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, dev);
    cudaStream_t* ss[4] = {&h->s_red, &h->s_d2h, &h->s_h2d, &h->s_bc};
    for (cudaStream_t* s : ss)
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
    cudaEvent_t* one[3] = {&h->ev_start, &h->ev_end, &h->ev_flag};
    for (cudaEvent_t* ev : one)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    for (int s = 0; s < S && e == cudaSuccess; ++s) {
        cudaEvent_t* es[4] = {&h->ev_red[s], &h->ev_d2h[s], &h->ev_h2d[s], &h->ev_bc[s]};
        for (cudaEvent_t* ev : es)
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
        rc = fail(h, e);
        release(h);
        return rc;
    }

    // tables: output pointers through the page-locked staging, runs directly
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    std::memcpy(h->hst + O.h_out_tab, param_bufs, (size_t)L.n_out * sizeof(uint16_t*));
    e = cudaEventRecord(h->ev_start, cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->s_bc, h->ev_start, 0);
    if (e == cudaSuccess) e = cudaMemsetAsync(h->dws + O.d_flag, 0, kAlignB, h->s_bc);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(h->dws + O.d_out_tab, h->hst + O.h_out_tab, (size_t)L.n_out * sizeof(uint16_t*),
                            cudaMemcpyHostToDevice, h->s_bc);
    if (e == cudaSuccess && !O.runs.empty())
        e = cudaMemcpyAsync(h->dws + O.d_runs, O.runs.data(), O.runs.size() * sizeof(OffRun), cudaMemcpyHostToDevice,
                            h->s_bc);
    if (e == cudaSuccess && !L.gather_segs.empty())
        e = cudaMemcpyAsync(h->dws + O.d_gather, L.gather_segs.data(), L.gather_segs.size() * sizeof(zk::SegDesc),
                            cudaMemcpyHostToDevice, h->s_bc);
    if (e == cudaSuccess && L.stage == 3) {
        h->shards = param_bufs[0];
        e = zk::occupancy(zk::K_GATHER, 0, &h->occ_gather);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(h->s_bc);

    // host state in state order (each thread first-touches the pages it will
    // update), fp16 parameters uploaded chunk by chunk
    if (e == cudaSuccess)
        e = fill_state(h, cs, [&](const OffRun& r, int64_t c0, int64_t a, int64_t b) {
            std::memcpy(h->w + c0 + a, master_init + r.grad_begin + (a - r.local_begin), (size_t)(b - a) * 4);
            std::memset(h->m + c0 + a, 0, (size_t)(b - a) * 4);
            std::memset(h->v + c0 + a, 0, (size_t)(b - a) * 4);
        });
    if (e != cudaSuccess) {
        rc = fail(h, e);
        release(h);
        return rc;
    }
    *out = h;
    return ZERO_OK;
}

ZERO_API int zero_offload_step(zero_offload_handle* h, const uint16_t* const* grads, float loss_scale,
                               const zero_hyper* hp, void* stream)
{
    const zk::NvtxRange nvtx_range("zero_offload_step");
    if (!h || !grads || !hp) return ZERO_ERR_ARG;
    if (h->broken) return ZERO_ERR_CUDA;
    if (!(loss_scale > 0.0f) || !std::isfinite(loss_scale)) return ZERO_ERR_ARG;
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->beta1) || !std::isfinite(hp->beta2) ||
        !std::isfinite(hp->eps) || !std::isfinite(hp->weight_decay))
        return ZERO_ERR_ARG;
    const zl::Layout& L = h->L;
    const OffLayout& O = h->O;
    for (int k = 0; k < L.nd; ++k) {
        if (!grads[k]) return ZERO_ERR_ARG;
        if (!al16(grads[k])) return ZERO_ERR_ALIGN;
    }
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const float inv = (float)(1.0 / (double)loss_scale);

    // ---- overflow check: the whole step's flag before any state changes ----
    std::memcpy(h->hst + O.h_grad_tab, grads, (size_t)L.nd * sizeof(uint16_t*));
    unsigned* h_flag = reinterpret_cast<unsigned*>(h->hst + O.h_flag);
    cudaError_t e = cudaEventRecord(h->ev_start, cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->s_red, h->ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->s_bc, h->ev_start, 0);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(h->dws + O.d_grad_tab, h->hst + O.h_grad_tab, (size_t)L.nd * sizeof(uint16_t*),
                            cudaMemcpyHostToDevice, h->s_red);
    if (e == cudaSuccess) e = cudaMemsetAsync(h->d_flag(), 0, 4, h->s_red);
    if (e == cudaSuccess && L.grad_len > 0) {
        off_check_kernel<<<h->grid((L.grad_len + 3) / 4), kBlock, L.nd * sizeof(void*), h->s_red>>>(
            h->d_grad_tab(), L.nd, L.grad_len, inv, h->d_flag());
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(h_flag, h->d_flag(), 4, cudaMemcpyDeviceToHost, h->s_red);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_flag, h->s_red);
    // start the first downloads while the flag travels: they only read
    for (int64_t k = 0; k < std::min<int64_t>(S, O.n_chunks) && e == cudaSuccess; ++k)
        e = download_chunk(h, k, (int)k, inv);
    if (e == cudaSuccess) e = cudaEventSynchronize(h->ev_flag);
    if (e != cudaSuccess) return fail(h, e);
    if (*h_flag != 0) {
        // skipped: nothing changes; drain the speculative downloads
        if (O.n_chunks > 0) e = cudaStreamSynchronize(h->s_d2h);
        if (e != cudaSuccess) return fail(h, e);
        return ZERO_SKIPPED;
    }

    // ---- the update, chunk by chunk ----
    const int64_t t_new = h->t + 1;
    const ZhCoef c = make_coef(hp, t_new);
    const float wd = hp->weight_decay;
    for (int64_t k = 0; k < O.n_chunks; ++k) {
        const int s = (int)(k % S);
        e = cudaEventSynchronize(h->ev_d2h[s]);           // reduced gradient of chunk k on the host
        if (e == cudaSuccess) e = cudaEventSynchronize(h->ev_h2d[s]);  // host fp16 slot free
        if (e != cudaSuccess) return fail(h, e);
        const zk::NvtxRange chunk_range("offload host update chunk");
        const int64_t c0 = h->chunk_begin(k);
        const float* g = h->h_red(s);
        uint16_t* p16 = h->h_p16(s);
        for_chunk(h, k, [&](const OffRun& r, int64_t a, int64_t b) {
            h->adam(g + a, h->w + c0 + a, h->m + c0 + a, h->v + c0 + a, p16 + a, b - a, &c, r.decay ? wd : 0.0f);
        });
        e = upload_chunk(h, k, s);
        if (e == cudaSuccess && k + S < O.n_chunks) e = download_chunk(h, k + S, s, inv);
        if (e != cudaSuccess) return fail(h, e);
    }
    h->t = t_new;
    e = cudaEventRecord(h->ev_end, h->s_bc);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, h->ev_end, 0);
    if (e != cudaSuccess) return fail(h, e);
    return ZERO_OK;
}

ZERO_API int zero_offload_gather_layer(zero_offload_handle* h, int32_t unit, uint16_t* out, void* stream)
{
    const zk::NvtxRange nvtx_range("zero_offload_gather_layer");
    if (!h) return ZERO_ERR_ARG;
    const zl::Layout& L = h->L;
    if (L.stage != 3) return ZERO_ERR_STAGE;
    if (unit < 0 || unit >= L.n_units || !out) return ZERO_ERR_ARG;
    if (!al16(out)) return ZERO_ERR_ALIGN;
    const zl::Unit& U = L.units[unit];
    if (U.n_chunks == 0) return ZERO_OK;
    zk::GatherArgs g{};
    g.segs = h->d_gather() + U.seg0;
    g.n_segs = (int)U.n_segs;
    g.n_chunks = U.n_chunks;
    g.src = h->shards;
    g.dst = out;
    g.err = h->d_flag() + 1;
    g.src_len = L.state_elems;
    g.dst_len = U.numel;
    const int64_t want = (U.n_chunks + zk::kThreads / 32 - 1) / (zk::kThreads / 32);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)h->sms * std::max(1, h->occ_gather)));
    const cudaError_t e = zk::launch_gather(g, grid, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        h->last_cuda = (int)e;
        return ZERO_ERR_CUDA;
    }
    return ZERO_OK;
}

ZERO_API int zero_offload_set_state(zero_offload_handle* h, const float* master, const float* m, const float* v,
                                    int64_t t, void* stream)
{
    if (!h || h->broken || t < 0) return ZERO_ERR_ARG;
    if (h->O.E > 0 && (!master || !m || !v)) return ZERO_ERR_ARG;
    const cudaError_t e =
        fill_state(h, static_cast<cudaStream_t>(stream), [&](const OffRun&, int64_t c0, int64_t a, int64_t b) {
            const size_t bytes = (size_t)(b - a) * 4;
            if (h->w + c0 + a != master + c0 + a) std::memcpy(h->w + c0 + a, master + c0 + a, bytes);
            if (h->m + c0 + a != m + c0 + a) std::memcpy(h->m + c0 + a, m + c0 + a, bytes);
            if (h->v + c0 + a != v + c0 + a) std::memcpy(h->v + c0 + a, v + c0 + a, bytes);
        });
    if (e != cudaSuccess) return fail(h, e);
    h->t = t;
    return ZERO_OK;
}

ZERO_API int zero_offload_state(zero_offload_handle* h, const float** master, const float** m, const float** v,
                                int64_t* t)
{
    if (!h) return ZERO_ERR_ARG;
    if (master) *master = h->w;
    if (m) *m = h->m;
    if (v) *v = h->v;
    if (t) *t = h->t;
    return ZERO_OK;
}

ZERO_API int zero_offload_host_update(const float* g, float* w, float* m, float* v, uint16_t* p16, int64_t n,
                                      const zero_hyper* hp, int64_t t, int decay, int path)
{
    if (n < 0 || (n > 0 && (!g || !w || !m || !v || !p16)) || !hp || t < 1 || path < 0 || path > 2)
        return ZERO_ERR_ARG;
    const bool avx2 = cpu_has_avx2();
    if (path == 2 && !avx2) return ZERO_ERR_ARG;
    const AdamFn f = (path == 2 || (path == 0 && avx2)) ? zh_adam_avx2 : zh_adam_base;
    const ZhCoef c = make_coef(hp, t);
    DefaultFpEnv env;
    f(g, w, m, v, p16, n, &c, decay ? hp->weight_decay : 0.0f);
    return ZERO_OK;
}

ZERO_API void zero_offload_destroy(zero_offload_handle* h) { release(h); }

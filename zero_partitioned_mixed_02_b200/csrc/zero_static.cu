// zero_step_static: the two-pass stage 1/2 step for callers that cannot
// allocate device memory. Its scratch (fp32 reduced gradients, the overflow
// word, the pointer and run tables) lives in one file-scope __device__ array,
// so the call itself allocates nothing. See include/zero.h for the contract.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "zero.h"
#include "zero_internal.h"

#define ZERO_API extern "C" __attribute__((visibility("default")))

namespace {

// Scratch layout: [0, 256) overflow word | grad pointer table | replica
// pointer table | run table | fp32 reduced gradients.
constexpr size_t kFlagOff = 0;
constexpr size_t kGradTabOff = 256;
constexpr size_t kOutTabOff = kGradTabOff + 8 * ZERO_STATIC_MAX_ND;
constexpr size_t kRunTabOff = kOutTabOff + 8 * ZERO_STATIC_MAX_ND;
constexpr size_t kRedOff = 8192;
constexpr size_t kScratchBytes = kRedOff + 4 * (size_t)ZERO_STATIC_MAX_PSI;
static_assert(kRunTabOff + sizeof(zk::SegDesc) * ZERO_STATIC_MAX_ND <= kRedOff, "run table overlaps");

// One copy per device that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};        // device address of g_static_scratch, per device
int g_occ[kMaxDevices][2] = {};           // resident blocks per SM: reduce, update
int g_sms[kMaxDevices] = {};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// beta^n as the n-fold double product 1.0 * beta * ... * beta, the same
// definition as the handle path's bias corrections. The caller passes t, so
// the products are kept between calls: a call continues from the last one's
// products when its betas are the same and its n has not gone backwards, and
// starts again from 1.0 otherwise. The loop also ends as soon as neither
// product changes any more (a beta of 1, a product of 0, or the smallest
// subnormal on which a beta below one settles), which bounds a large first t
// to a few million multiplications; the values are those of the plain loop.
struct Powers {
    double b1 = -1.0, b2 = -1.0;
    int64_t n = 0;
    double p1 = 1.0, p2 = 1.0;
};
Powers g_pow;  // guarded by g_mu

void beta_powers(double b1, double b2, int64_t n, double* p1, double* p2)
{
    std::lock_guard<std::mutex> lock(g_mu);
    Powers& c = g_pow;
    if (c.b1 != b1 || c.b2 != b2 || c.n > n) {
        c = Powers{};
        c.b1 = b1;
        c.b2 = b2;
    }
    while (c.n < n) {
        const double q1 = c.p1 * b1, q2 = c.p2 * b2;
        if (q1 == c.p1 && q2 == c.p2) {  // a fixed point: every further factor leaves both unchanged
            c.n = n;
            break;
        }
        c.p1 = q1;
        c.p2 = q2;
        ++c.n;
    }
    *p1 = c.p1;
    *p2 = c.p2;
}

// The host-side name of a __device__ array is not its device address; the
// address is looked up once per device, with that device current.
cudaError_t setup(int dev, void** scratch)
{
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        const int smem = zk::step_smem_bytes(ZERO_STATIC_MAX_ND, ZERO_STATIC_MAX_ND);
        e = zk::occupancy(zk::K_REDUCE, smem, &g_occ[dev][0]);
        if (e == cudaSuccess) e = zk::occupancy(zk::K_UPDATE, smem, &g_occ[dev][1]);
        if (e != cudaSuccess) return e;
        g_scratch[dev] = p;
    }
    *scratch = g_scratch[dev];
    return cudaSuccess;
}

// Same cut as the handle path: the vector body starts on a line of the
// gradient index; head and ragged tail go to scalar chunks.
void add_run(zk::SegDesc* runs, int* n, int64_t* chunks, int64_t begin, int64_t len)
{
    if (len <= 0) return;
    zk::SegDesc d{};
    d.grad_begin = d.state_begin = d.out_begin = begin;
    d.len = len;
    d.decay = 1;
    int64_t head = (zk::kLineElems - begin % zk::kLineElems) % zk::kLineElems;
    if (head > len) head = len;
    const int64_t quads = (len - head) / zk::kQuad;
    d.head = (int)head;
    d.tail = (int)(len - head - quads * zk::kQuad);
    d.chunk_begin = *chunks;
    *chunks += (quads + zk::kQuadsPerChunk - 1) / zk::kQuadsPerChunk + (d.head + d.tail + 31) / 32;
    runs[(*n)++] = d;
}

}  // namespace

ZERO_API int zero_step_static(int64_t psi, int32_t nd, const uint16_t* const* grads, float* master,
                              float* m, float* v, uint16_t* const* replicas, float loss_scale,
                              const zero_hyper* hp, int64_t* t, void* stream, int* skipped)
{
    if (skipped) *skipped = 0;
    if (psi < 1 || psi > ZERO_STATIC_MAX_PSI || nd < 1 || nd > ZERO_STATIC_MAX_ND) return ZERO_ERR_ARG;
    if (!grads || !master || !m || !v || !replicas || !hp || !t || *t < 0 || *t == INT64_MAX) return ZERO_ERR_ARG;
    if (!(loss_scale > 0.0f) || !std::isfinite(loss_scale)) return ZERO_ERR_ARG;
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->beta1) || !std::isfinite(hp->beta2) ||
        !std::isfinite(hp->eps) || !std::isfinite(hp->weight_decay))
        return ZERO_ERR_ARG;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v)) return ZERO_ERR_ALIGN;
    for (int k = 0; k < nd; ++k) {
        if (!grads[k] || !replicas[k]) return ZERO_ERR_ARG;
        if (!aligned16(grads[k]) || !aligned16(replicas[k])) return ZERO_ERR_ALIGN;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZERO_ERR_CUDA;
    void* scratch = nullptr;
    if (setup(dev, &scratch) != cudaSuccess) return ZERO_ERR_CUDA;
    char* base = static_cast<char*>(scratch);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // host copies of the tables (pageable; each copy is staged before it returns)
    const uint16_t* grad_tab[ZERO_STATIC_MAX_ND];
    uint16_t* out_tab[ZERO_STATIC_MAX_ND];
    zk::SegDesc runs[ZERO_STATIC_MAX_ND];
    int n_runs = 0;
    int64_t chunks = 0;
    const int64_t p = (psi + nd - 1) / nd;
    for (int r = 0; r < nd; ++r) {
        grad_tab[r] = grads[r];
        out_tab[r] = replicas[r];
        const int64_t b = std::min<int64_t>((int64_t)r * p, psi);
        add_run(runs, &n_runs, &chunks, b, std::min<int64_t>(b + p, psi) - b);
    }

    // the array keeps the last call's contents: clear the overflow word
    cudaError_t e = cudaMemsetAsync(base + kFlagOff, 0, 2 * sizeof(unsigned), s);  // overflow, error words
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(base + kGradTabOff, grad_tab, nd * sizeof(void*), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(base + kOutTabOff, out_tab, nd * sizeof(void*), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(base + kRunTabOff, runs, n_runs * sizeof(zk::SegDesc), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return ZERO_ERR_CUDA;

    zk::StepArgs a{};
    a.segs = reinterpret_cast<const zk::SegDesc*>(base + kRunTabOff);
    a.n_segs = n_runs;
    a.n_chunks = chunks;
    a.grads = reinterpret_cast<const uint16_t* const*>(base + kGradTabOff);
    a.outs = reinterpret_cast<uint16_t* const*>(base + kOutTabOff);
    a.nd = nd;
    a.n_out = nd;
    a.w_in = master;
    a.m_in = m;
    a.v_in = v;
    a.w_out = master;  // the update pass works in place
    a.m_out = m;
    a.v_out = v;
    a.red = reinterpret_cast<float*>(base + kRedOff);
    a.flag = reinterpret_cast<unsigned*>(base + kFlagOff);
    a.err = a.flag + 1;
    a.grad_len = a.state_len = a.out_len = psi;
    a.call_id = 1;
    a.c.inv_scale = (float)(1.0 / (double)loss_scale);
    a.c.lr = hp->lr;
    a.c.b1 = hp->beta1;
    a.c.b2 = hp->beta2;
    a.c.omb1 = 1.0f - hp->beta1;
    a.c.omb2 = 1.0f - hp->beta2;
    a.c.eps = hp->eps;
    a.c.wd = hp->weight_decay;
    double p1, p2;  // beta^(t+1) as the (t+1)-fold double product
    beta_powers((double)hp->beta1, (double)hp->beta2, *t + 1, &p1, &p2);
    a.c.bc1 = (float)(1.0 - p1);
    a.c.bc2 = (float)(1.0 - p2);

    const int64_t want = std::max<int64_t>(1, (chunks + zk::kThreads / 32 - 1) / (zk::kThreads / 32));
    const int g0 = (int)std::min<int64_t>(want, (int64_t)g_sms[dev] * std::max(1, g_occ[dev][0]));
    const int g1 = (int)std::min<int64_t>(want, (int64_t)g_sms[dev] * std::max(1, g_occ[dev][1]));
    e = zk::launch_step(zk::K_REDUCE, a, g0, s);
    if (e == cudaSuccess) e = zk::launch_step(zk::K_UPDATE, a, g1, s);
    unsigned words[2] = {0, 0};  // overflow word, error word (bounds-checked build)
    if (e == cudaSuccess) e = cudaMemcpyAsync(words, base + kFlagOff, sizeof(words), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return ZERO_ERR_CUDA;
    if (words[1] != 0) return ZERO_ERR_INTERNAL;
    const unsigned flag = words[0];
    if (flag == a.call_id) {
        if (skipped) *skipped = 1;
        return ZERO_SKIPPED;
    }
    *t = *t + 1;
    return ZERO_OK;
}

// Internal interface between the host ABI (zero_abi.cu) and the kernels
// (zero_kernels.cu). Not installed; the public boundary is include/zero.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace zk {

constexpr int kThreads = 256;  // threads per block of every kernel
// Vector work moves "quads" of 4 consecutive elements: 8 bytes of fp16, 16 of
// fp32. A warp chunk is 64 quads (256 elements); lane L takes quads L and
// L + 32, so each warp instruction touches one contiguous, sector-aligned run
// (256 B of fp16, 512 B of fp32) and a lane keeps 8 elements in flight.
constexpr int kQuad = 4;
constexpr int kQuadsPerChunk = 64;
constexpr int kChunkElems = kQuad * kQuadsPerChunk;
// Vector bodies start on a multiple of kLineElems gradient elements: one
// 128-byte line of fp16 (two of fp32). Every warp chunk then covers whole
// 32-byte sectors, so no sector is written in halves by two different warps
// (a partial-sector write costs the memory system a read-modify-write).
constexpr int kLineElems = 64;

// One contiguous run of elements. A run is a piece of one rank's partition
// (stage 1/2) or one rank's chunk of one tensor (stage 3). Three index spaces:
// the gradient buffers (grad), the state arrays (state), the fp16 output
// buffers (out). The run is cut, relative to the gradient index, into a scalar
// head up to the first multiple of kLineElems, a body of quads, and a scalar
// tail (< kQuad). Work is handed out in warp chunks: ceil(quads / 64) vector
// chunks, then ceil((head + tail) / 32) scalar chunks.
struct alignas(16) SegDesc {
    long long grad_begin;
    long long state_begin;
    long long out_begin;
    long long len;
    long long chunk_begin;  // first chunk of this run in the launch's chunk numbering
    int head;               // scalar elements before the body
    int tail;               // scalar elements after the body
    int decay;              // 1: weight decay applies to the run; 0: excluded tensor
    int pad;
};
static_assert(sizeof(SegDesc) == 64, "SegDesc layout");

// Per-step binary32 constants, computed on the host (or, for the
// asynchronous step, partly on the device from the control block).
struct Coef {
    float inv_scale, lr, b1, b2, omb1, omb2, bc1, bc2, eps, wd;
};

// Device-resident control block of the asynchronous step: everything the host
// would otherwise decide between steps.
struct alignas(16) Ctrl {
    double p1, p2;       // beta1^t, beta2^t as t-fold double products
    long long t;         // committed steps
    long long skipped;   // steps skipped since the asynchronous run began
    float scale;         // current loss scale
    float growth;        // dynamic loss scaling: growth factor,
    float backoff;       //   back-off factor,
    float b1, b2;        // betas the products use
    int interval;        //   good steps before growth,
    int good;            //   current run of good steps
    int cur;             // live state buffer
    int fused;           // 1: a step writes the other buffer, switched on commit
    // the next step's binary32 constants, written by zero_async_begin and by
    // each commit (ctrl_next_constants), so that the step kernel loads three
    // values instead of deriving them in double in every thread
    float inv_scale, bc1, bc2;
};
static_assert(sizeof(Ctrl) == 80, "Ctrl layout");

// inv_scale = (float)(1 / (double)scale); bc_k = (float)(1 - beta_k^(t+1)),
// beta_k^(t+1) the (t+1)-fold double product continued from p_k: the same
// operations as the synchronous step's host code, so the results are equal.
__host__ __device__ inline void ctrl_next_constants(Ctrl* c)
{
    const double p1 = c->p1 * (double)c->b1;
    const double p2 = c->p2 * (double)c->b2;
    c->bc1 = (float)(1.0 - p1);
    c->bc2 = (float)(1.0 - p2);
    c->inv_scale = (float)(1.0 / (double)c->scale);
}

struct StepArgs {
    const SegDesc* segs;
    int n_segs;
    long long n_chunks;
    const uint16_t* const* grads;  // device table, nd entries
    uint16_t* const* outs;         // device table, n_out entries
    int nd;
    int n_out;
    const float* w_in;
    const float* m_in;
    const float* v_in;
    float* w_out;
    float* m_out;
    float* v_out;
    float* red;                    // two-pass: reduced unscaled gradients (state order)
    const float* master_init;      // init: initial master weights (gradient order)
    unsigned* flag;                // overflow word: holds the id of the last call that overflowed
    unsigned call_id;
    Coef c;
    // asynchronous step: when ctrl is set the kernel takes inv_scale, bc1,
    // bc2 and the in/out state buffers (from st) from the control block
    const Ctrl* ctrl;
    float* st[2][3];
    unsigned* err;                 // kernel error word (roll-back condition)
    // element extents of the buffers (grads and master_init; state arrays and
    // red; outputs), checked by the bounds-checked build (ZK_BOUNDS_CHECK)
    long long grad_len, state_len, out_len;
    // without an fp32 master: the output the weight is read from (K_UPDATE,
    // K_STEP_FUSED), and how many of the last outputs K_STEP_FUSED leaves
    // unwritten (the fused bfloat16 step keeps the last output, the backup
    // K_REPLICA restores from or brings up to date; 0 elsewhere)
    int w_src;
    int keep_last;
};

struct GatherArgs {
    const SegDesc* segs;  // grad_begin = index into src, out_begin = index into dst
    int n_segs;
    long long n_chunks;
    const uint16_t* src;
    uint16_t* dst;
    unsigned* err;                // error word (bounds-checked build)
    long long src_len, dst_len;   // element extents (bounds-checked build)
};

// ---- the TMA-staged fused step ----
// A run of the TMA path: its body [head, len - tail) starts on a line of the
// gradient index and is a multiple of 8 elements, cut into tiles of the shape's
// elements; head and tail elements are scalar items handled from global
// memory. Every index space is in 16-byte phase with the gradient index.
struct alignas(16) TmaRun {
    long long grad_begin;
    long long state_begin;
    long long out_begin;
    long long len;
    long long tile_begin;  // first tile of the body in the launch's tile numbering
    long long scal_begin;  // first scalar item in the launch's scalar numbering
    int head;
    int tail;
    int decay;             // as SegDesc::decay
    int pad;
};
static_assert(sizeof(TmaRun) == 64, "TmaRun layout");

// Two shapes of the TMA kernel. Stage 1/2 with its Nd replica writes is
// store-heavy: many consumer warps (one CTA of 32 warps per SM) and a single
// stage, released as soon as the warps have read it, so the next tile's loads
// overlap the arithmetic and the stores. Few output streams (stage 3, the rank
// view): a deeper pipeline of two stages keeps more loads in flight.
struct TmaShape {
    int warps;   // consumer warps; one more warp produces
    int stages;  // input stages
    int tile;    // elements per tile: one quad per consumer thread
};
constexpr TmaShape kTmaWide{31, 1, 31 * 32 * 4};
constexpr TmaShape kTmaDeep{20, 2, 20 * 32 * 4};
inline TmaShape tma_shape(int n_out) { return n_out >= 4 ? kTmaWide : kTmaDeep; }
constexpr int kTmaMaxNd = 16;  // ranks whose tiles fit the stages (deep shape at 16: 226,304 B)

struct TmaArgs {
    StepArgs b;             // pointers, tables, constants, flag (segs unused)
    const TmaRun* runs;
    int n_runs;
    long long n_tiles;
    long long n_scal;
    unsigned* err;          // set when a bounded wait gives up
    unsigned wait_rounds;   // try_wait rounds before a wait gives up
    long long hold_tile;    // test hook: this tile is never armed (-1: none)
};

// ---- the two-pass step with TMA staging (ZERO_VARIANT_TWO_PASS_TMA) ----
constexpr int kPassReduce = 0;  // Nd gradient slices in, the reduced gradient out
constexpr int kPassUpdate = 1;  // reduced gradient, m, v, weight in; m, v, (master,) parameters out
// the reduce pass has Nd input streams and one output: the deeper shape; the
// update pass is store-heavy with many outputs: the shape of the fused step
inline TmaShape tma_pass_shape(int mode, int n_out) { return mode == kPassReduce ? kTmaDeep : tma_shape(n_out); }

// try_wait rounds (each may suspend about a microsecond) before a wait of the
// TMA kernels gives up: a few seconds, far beyond any legitimate wait.
constexpr unsigned kTmaWaitRounds = 1u << 22;
// Error-word bits set by the in-place update pass of the two-pass TMA step
// (its failed waits; every other kernel uses the bits below 64).
constexpr int kErrUpdateShift = 6;
constexpr unsigned kErrUpdate = 7u << kErrUpdateShift;

enum Kernel : int {
    K_STEP_FUSED = 0,  // reduce + unscale + flag + Adam into the next buffer + fp16 write-back
    K_REDUCE = 1,      // two-pass, pass 1: reduce + unscale + flag into red
    K_UPDATE = 2,      // two-pass, pass 2: flag check, Adam in place + fp16 write-back
    K_CAST = 3,        // fp16 write-back of the current master (overflow roll-back)
    K_INIT = 4,        // master = master_init, m = v = 0, fp16 write-back
    K_GATHER = 5,      // stage-3 layer gather
    K_CAST_IF = 6,     // K_CAST only if the step overflowed (asynchronous step)
    K_REPLICA = 7,     // fused bfloat16 step: on overflow (or a failed wait) copy the last output
                       // over the others, else copy output 0 into the last one
    K_COUNT = 8
};

// Blocks per SM the kernel reaches with `smem` bytes of dynamic shared memory
// (0 for a kind not built for the format). bf16: the bfloat16 step without an
// fp32 master (kinds K_REDUCE, K_UPDATE, K_CAST, K_INIT; state = m and v only,
// the weight read back from the first output).
cudaError_t occupancy(Kernel k, int smem, int* blocks_per_sm, bool bf16 = false);
cudaError_t launch_step(Kernel k, const StepArgs& a, int grid, cudaStream_t s, bool bf16 = false);
cudaError_t launch_gather(const GatherArgs& a, int grid, cudaStream_t s);
cudaError_t launch_copy(void* dst, const void* src, size_t bytes, int grid, cudaStream_t s);
// Asynchronous step: commit or roll back on the device (one thread).
cudaError_t launch_commit(Ctrl* ctrl, unsigned* flag, const unsigned* err, cudaStream_t s);
// TMA-staged fused step: one-time attribute set-up and blocks per SM for the
// shape and nd ranks, launch.
cudaError_t tma_prepare(TmaShape shape, int nd, bool bf16, int* blocks_per_sm);
cudaError_t launch_step_tma(TmaShape shape, const TmaArgs& a, int grid, cudaStream_t s, bool bf16);
// Two-pass step with TMA staging: attribute set-up and blocks per SM of the
// two passes (bf16: the bfloat16 codec without master), launch of one pass.
// Both use TmaArgs; the update pass returns at once if the overflow word holds
// the call's id or the error word is set.
cudaError_t tma_pass_prepare(int nd, int n_out, bool bf16, int* occ_reduce, int* occ_update);
cudaError_t launch_pass_tma(int mode, const TmaArgs& a, int grid, cudaStream_t s, bool bf16);
int step_smem_bytes(int nd, int n_out);

}  // namespace zk

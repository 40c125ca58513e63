// Host side of libzero: validation, the partitioner and descriptor tables, the
// memory ledger, and the C ABI declared in include/zero.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <utility>
#include <vector>

#include "zero.h"
#include "zero_internal.h"
#include "zero_layout.h"
#include "zero_nvtx.h"

#define ZERO_API extern "C" __attribute__((visibility("default")))

using zl::Layout;
using zl::split;
using zl::Unit;

namespace {

constexpr int64_t kAlign = 256;
constexpr int64_t kMaxPsi = int64_t(1) << 42;

int64_t align_up(int64_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// fused variants: one pass into a second state buffer, roll-back by re-cast;
// two-pass variants: reduce into a scratch, then update in place
bool is_fused(int variant) { return variant == ZERO_VARIANT_FUSED || variant == ZERO_VARIANT_FUSED_TMA; }
bool is_tma(int variant) { return variant == ZERO_VARIANT_FUSED_TMA || variant == ZERO_VARIANT_TWO_PASS_TMA; }

// Cut a run at the first line-aligned gradient index and give it its chunks.
void add_run(std::vector<zk::SegDesc>& v, int64_t* chunks, int64_t grad_begin, int64_t state_begin,
             int64_t out_begin, int64_t len, int decay = 1)
{
    if (len <= 0) return;
    zk::SegDesc d{};
    d.decay = decay;
    d.grad_begin = grad_begin;
    d.state_begin = state_begin;
    d.out_begin = out_begin;
    d.len = len;
    int64_t head = (zk::kLineElems - (grad_begin % zk::kLineElems)) % zk::kLineElems;
    if (head > len) head = len;
    const int64_t quads = (len - head) / zk::kQuad;
    d.head = (int)head;
    d.tail = (int)(len - head - quads * zk::kQuad);
    d.chunk_begin = *chunks;
    const int64_t vec = (quads + zk::kQuadsPerChunk - 1) / zk::kQuadsPerChunk;
    *chunks += vec + (d.head + d.tail + 31) / 32;
    v.push_back(d);
}

}  // namespace

int zl::build_layout(const zero_config* cfg, Layout* L)
{
    if (!cfg) return ZERO_ERR_ARG;
    if (cfg->psi < 1 || cfg->psi > kMaxPsi) return ZERO_ERR_ARG;
    if (cfg->nd < 1 || cfg->nd > ZERO_MAX_ND) return ZERO_ERR_ARG;
    if (cfg->stage < 1 || cfg->stage > 3) return ZERO_ERR_ARG;
    if (cfg->variant != ZERO_VARIANT_FUSED && cfg->variant != ZERO_VARIANT_TWO_PASS &&
        cfg->variant != ZERO_VARIANT_FUSED_TMA && cfg->variant != ZERO_VARIANT_TWO_PASS_TMA)
        return ZERO_ERR_ARG;
    if (cfg->n_tensors < 0) return ZERO_ERR_ARG;
    if (cfg->precision != ZERO_PRECISION_FP16 && cfg->precision != ZERO_PRECISION_BF16) return ZERO_ERR_ARG;
    // without a master the fused step needs a second copy of the old weights
    // to roll back to: the last replica of emulated stage 1/2 ranks (Nd >= 2);
    // anything else runs the two-pass step only
    if (cfg->precision == ZERO_PRECISION_BF16 && is_fused(cfg->variant) &&
        !(cfg->rank_view < 0 && cfg->stage <= 2 && cfg->nd >= 2))
        return ZERO_ERR_ARG;
    if (cfg->rank_view < -1 || cfg->rank_view >= cfg->nd) return ZERO_ERR_ARG;
    // a stage-3 rank writes only its own fp16 shard
    if (cfg->rank_view >= 0 && cfg->stage == 3 && cfg->view_outputs > 1) return ZERO_ERR_ARG;
    if (cfg->reserved != 0) return ZERO_ERR_ARG;
    if (cfg->rank_view < 0 ? cfg->view_outputs != 0
                           : (cfg->view_outputs != 0 && cfg->view_outputs != 1 && cfg->view_outputs != cfg->nd))
        return ZERO_ERR_ARG;
    if (cfg->stage == 3 && cfg->n_tensors == 0) return ZERO_ERR_ARG;
    if (cfg->n_tensors > 0 && !cfg->tensors) return ZERO_ERR_ARG;

    L->psi = cfg->psi;
    L->nd = cfg->nd;
    L->stage = cfg->stage;
    L->view = cfg->rank_view;
    L->variant = cfg->variant;
    L->bf16 = cfg->precision == ZERO_PRECISION_BF16;
    const int nd = cfg->nd;
    if (cfg->n_tensors > 0) {
        int64_t sum = 0;
        int32_t prev_unit = 0;
        for (int i = 0; i < cfg->n_tensors; ++i) {
            const zero_tensor& t = cfg->tensors[i];
            if (t.numel < 1 || (t.flags & ~ZERO_TENSOR_NO_DECAY) != 0 || t.unit < 0) return ZERO_ERR_ARG;
            if (i == 0 ? t.unit != 0 : (t.unit != prev_unit && t.unit != prev_unit + 1)) return ZERO_ERR_ARG;
            prev_unit = t.unit;
            sum += t.numel;
            if (sum > kMaxPsi) return ZERO_ERR_ARG;
            L->numel.push_back(t.numel);
            L->unit_of.push_back(t.unit);
            L->decay_of.push_back((t.flags & ZERO_TENSOR_NO_DECAY) ? 0 : 1);
        }
        if (sum != cfg->psi) return ZERO_ERR_ARG;
        L->n_units = prev_unit + 1;
    } else {
        L->numel.push_back(cfg->psi);
        L->unit_of.push_back(0);
        L->decay_of.push_back(1);
        L->n_units = 1;
    }
    L->P = (cfg->psi + nd - 1) / nd;

    // ---- partitions and the step's run table ----
    L->shard_begin.assign(nd, 0);
    L->shard_len.assign(nd, 0);
    if (cfg->stage <= 2) {
        // flat spans of equal decay (consecutive tensors with the same flag
        // merge); a partition is cut where it crosses from one span to the next
        std::vector<std::pair<int64_t, int>> span_end;  // (end, decay)
        int64_t flat = 0;
        for (size_t t = 0; t < L->numel.size(); ++t) {
            flat += L->numel[t];
            if (!span_end.empty() && span_end.back().second == L->decay_of[t])
                span_end.back().first = flat;
            else
                span_end.push_back({flat, L->decay_of[t]});
        }
        // runs of the flat range [b, e): grad and state indices are flat - base
        auto add_partition = [&](int64_t b, int64_t e, int64_t base) {
            int64_t x = b, span_begin = 0;
            for (const auto& sp : span_end) {
                const int64_t lo = std::max(x, span_begin), hi = std::min(e, sp.first);
                if (hi > lo) {
                    add_run(L->step_segs, &L->step_chunks, lo - base, lo - base, lo, hi - lo, sp.second);
                    x = hi;
                }
                span_begin = sp.first;
            }
        };
        if (cfg->rank_view < 0) {
            for (int r = 0; r < nd; ++r) {
                int64_t b, e;
                split(cfg->psi, nd, r, &b, &e);
                L->shard_begin[r] = b;
                L->shard_len[r] = e - b;
                add_partition(b, e, 0);
            }
            L->state_elems = cfg->psi;
            L->grad_len = cfg->psi;
            L->n_out = nd;
        } else {
            int64_t b, e;
            split(cfg->psi, nd, cfg->rank_view, &b, &e);
            L->shard_len[cfg->rank_view] = e - b;
            add_partition(b, e, b);
            L->state_elems = e - b;
            L->grad_len = e - b;
            L->n_out = cfg->view_outputs == nd ? nd : 1;
        }
    } else {
        // stage 3: every tensor split per rank; rank r's shard is its chunks
        // in tensor order, shards back to back in rank order. The single-rank
        // view (rank r of a real job) keeps rank r's runs only, its state and
        // shard indexed from 0; gradients stay full-length (flat index).
        const int view = cfg->rank_view;
        int64_t pos = 0;
        for (int r = 0; r < nd; ++r) {
            L->shard_begin[r] = pos;
            int64_t off = 0, q = 0;
            for (size_t t = 0; t < L->numel.size(); ++t) {
                int64_t b, e;
                split(L->numel[t], nd, r, &b, &e);
                if (view < 0)
                    add_run(L->step_segs, &L->step_chunks, off + b, pos + q, pos + q, e - b, L->decay_of[t]);
                else if (r == view)
                    add_run(L->step_segs, &L->step_chunks, off + b, q, q, e - b, L->decay_of[t]);
                q += e - b;
                off += L->numel[t];
            }
            L->shard_len[r] = q;
            pos += q;
        }
        L->state_elems = view < 0 ? cfg->psi : L->shard_len[view];
        L->grad_len = cfg->psi;
        L->n_out = 1;  // the fp16 shard array

        // gather runs, unit by unit: tensor order, rank order within a tensor
        L->units.assign(L->n_units, Unit{});
        std::vector<int64_t> tensor_off(L->numel.size() + 1, 0);
        for (size_t t = 0; t < L->numel.size(); ++t) tensor_off[t + 1] = tensor_off[t] + L->numel[t];
        // position of rank r's chunk of tensor t inside the state arrays
        std::vector<int64_t> chunk_pos(L->numel.size() * (size_t)nd);
        for (int r = 0; r < nd; ++r) {
            int64_t q = L->shard_begin[r];
            for (size_t t = 0; t < L->numel.size(); ++t) {
                int64_t b, e;
                split(L->numel[t], nd, r, &b, &e);
                chunk_pos[t * nd + r] = q;
                q += e - b;
            }
        }
        size_t t = 0;
        for (int u = 0; u < L->n_units; ++u) {
            Unit& U = L->units[u];
            U.seg0 = (int64_t)L->gather_segs.size();
            U.flat_begin = tensor_off[t];
            int64_t chunks = 0;
            U.rank_run0 = (int64_t)L->rank_gather.size();
            while (t < L->numel.size() && L->unit_of[t] == u) {
                for (int r = 0; r < nd; ++r) {
                    int64_t b, e;
                    split(L->numel[t], nd, r, &b, &e);
                    if (view < 0)
                        add_run(L->gather_segs, &chunks, chunk_pos[t * nd + r],
                                0, tensor_off[t] - U.flat_begin + b, e - b);
                    // the same copies by source rank (the rank gather's
                    // table, and the plan zero_gather_plan reports)
                    if (e > b) {
                        zg::Run g{};
                        g.src_begin = chunk_pos[t * nd + r] - L->shard_begin[r];
                        g.out_begin = tensor_off[t] - U.flat_begin + b;
                        g.len = e - b;
                        g.tile_begin = U.rank_tiles;
                        g.rank = r;
                        U.rank_tiles += zg::tiles_of(e - b);
                        L->rank_gather.push_back(g);
                    }
                }
                U.numel += L->numel[t];
                ++t;
            }
            U.n_segs = (int64_t)L->gather_segs.size() - U.seg0;
            U.n_chunks = chunks;
            U.rank_n_runs = (int64_t)L->rank_gather.size() - U.rank_run0;
            L->transient_elems = std::max(L->transient_elems, U.numel);
        }
    }

    // ---- TMA run tables: the same runs, bodies cut at 8-element multiples ----
    // Tiles are numbered per table for one tile size: the fused kernel's
    // shape, or for the two-pass TMA variant the update pass's (tma_runs) and
    // the reduce pass's (tma_runs_r).
    if (is_tma(cfg->variant) && nd <= zk::kTmaMaxNd) {
        bool ok = true;
        for (const zk::SegDesc& d : L->step_segs)
            if ((d.state_begin - d.grad_begin) % 4 != 0 || (d.out_begin - d.grad_begin) % 8 != 0) ok = false;
        auto table = [&](int tile, std::vector<zk::TmaRun>& out, int64_t* tiles, int64_t* scal) {
            for (const zk::SegDesc& d : L->step_segs) {
                zk::TmaRun t{};
                t.decay = d.decay;
                t.grad_begin = d.grad_begin;
                t.state_begin = d.state_begin;
                t.out_begin = d.out_begin;
                t.len = d.len;
                int64_t head = (zk::kLineElems - d.grad_begin % zk::kLineElems) % zk::kLineElems;
                if (head > d.len) head = d.len;
                const int64_t body = (d.len - head) / 8 * 8;
                t.head = (int)head;
                t.tail = (int)(d.len - head - body);
                t.tile_begin = *tiles;
                t.scal_begin = *scal;
                *tiles += (body + tile - 1) / tile;
                *scal += t.head + t.tail;
                out.push_back(t);
            }
        };
        if (ok) {
            if (is_fused(cfg->variant)) {
                L->tma_shape = zk::tma_shape(L->n_out);
            } else {
                L->tma_shape = zk::tma_pass_shape(zk::kPassUpdate, L->n_out);
                L->tma_shape_r = zk::tma_pass_shape(zk::kPassReduce, L->n_out);
                table(L->tma_shape_r.tile, L->tma_runs_r, &L->tma_tiles_r, &L->tma_scal_r);
            }
            table(L->tma_shape.tile, L->tma_runs, &L->tma_tiles, &L->tma_scal);
            L->tma_ok = !L->tma_runs.empty();
        }
    }

    // ---- workspace layout ----
    int64_t off = 0;
    L->off_flag = off;
    off += kAlign;
    L->off_grad_tab = off;
    off += align_up((int64_t)nd * 8);
    L->off_out_tab = off;
    off += align_up((int64_t)std::max(L->n_out, 1) * 8);
    L->off_step_segs = off;
    off += align_up((int64_t)std::max<size_t>(L->step_segs.size(), 1) * sizeof(zk::SegDesc));
    if (L->tma_ok) {
        L->off_tma_runs = off;
        off += align_up((int64_t)L->tma_runs.size() * sizeof(zk::TmaRun));
        if (!L->tma_runs_r.empty()) {
            L->off_tma_runs_r = off;
            off += align_up((int64_t)L->tma_runs_r.size() * sizeof(zk::TmaRun));
        }
    }
    if (cfg->stage == 3) {
        // the Nd shard addresses, then the Nd shard lengths (a rank of a real
        // job: the ranks' shards; emulated ranks: their places in the shard array)
        L->off_shard_tab = off;
        off += align_up((int64_t)nd * 16);
        L->off_rank_gather = off;
        off += align_up((int64_t)std::max<size_t>(L->rank_gather.size(), 1) * sizeof(zg::Run));
    }
    const int n_buf = is_fused(cfg->variant) ? 2 : 1;
    for (int b = 0; b < n_buf; ++b)
        for (int k = 0; k < 3; ++k) {
            if (k == 0 && L->bf16) continue;  // no master: the parameters are the weights
            L->off_state[b][k] = off;
            off += align_up(L->state_elems * 4);
        }
    if (!is_fused(cfg->variant)) {
        L->off_reduced = off;
        off += align_up(L->state_elems * 4);
    }
    if (cfg->stage == 3) {
        L->off_shard16 = off;
        off += align_up(L->state_elems * 2);
    }
    L->total = off;
    return ZERO_OK;
}

namespace {

void fill_ledger(const Layout& L, zero_ledger* out)
{
    std::memset(out, 0, sizeof(*out));
    // [P1] "Where 16 bytes per parameter comes from": 2 + 2 + K, K = 12;
    // [P2] "The Mathematics": M_states(p, Nd). Without fp32 master weights
    // ([P3] "Why parameter count is not training memory") K = 8: m and v.
    const int64_t Ki = L.bf16 ? 8 : 12;
    const double psi = (double)L.psi, nd = (double)L.nd, K = (double)Ki;
    out->formula_bytes[0] = (2.0 + 2.0 + K) * psi;
    out->formula_bytes[1] = 4.0 * psi + K * psi / nd;
    out->formula_bytes[2] = 2.0 * psi + (2.0 + K) * psi / nd;
    out->formula_bytes[3] = (2.0 + 2.0 + K) * psi / nd;
    int64_t max_part = 0, max_shard = 0;
    for (int r = 0; r < L.nd; ++r) {
        int64_t b, e;
        split(L.psi, L.nd, r, &b, &e);
        max_part = std::max(max_part, e - b);
        int64_t s = 0;
        for (int64_t n : L.numel) {
            int64_t cb, ce;
            split(n, L.nd, r, &cb, &ce);
            s += ce - cb;
        }
        max_shard = std::max(max_shard, s);
    }
    out->exact_bytes[0] = (4 + Ki) * L.psi;
    out->exact_bytes[1] = 4 * L.psi + Ki * max_part;
    out->exact_bytes[2] = 2 * L.psi + (2 + Ki) * max_part;
    out->exact_bytes[3] = (4 + Ki) * max_shard;
    // ring collectives: each rank sends everything but the chunk it keeps
    const int64_t rs = (int64_t)L.nd * L.psi - L.psi;
    out->comm_elements[0] = rs;
    out->comm_elements[1] = rs;
    out->comm_elements[2] = 2 * rs;
    out->comm_elements[3] = 2 * rs;
    out->comm_elements[4] = 2 * rs;
    out->comm_elements[5] = 3 * rs;
    out->allreduce_buffer_bytes = 4 * L.psi;
    out->transient_bytes = L.stage == 3 ? 2 * L.transient_elems : 0;
    out->peak_stage3_bytes = out->exact_bytes[3] + 2 * L.transient_elems;
    out->workspace_bytes = L.total;
    out->partition_len = L.P;
    out->state_elems = L.state_elems;
    out->grad_len = L.grad_len;
    for (int b = 0; b < 2; ++b) {
        out->off_master[b] = L.off_state[b][0];
        out->off_m[b] = L.off_state[b][1];
        out->off_v[b] = L.off_state[b][2];
    }
    out->off_shard16 = L.off_shard16;
    out->off_reduced = L.off_reduced;
    out->n_units = L.stage == 3 ? L.n_units : 0;
    out->n_out = L.stage == 3 ? 0 : L.n_out;
}

}  // namespace

struct zero_handle {
    Layout L;
    char* ws = nullptr;
    int device = 0;
    int sms = 0;
    int occ[zk::K_COUNT] = {};
    zk::SegDesc* d_step_segs = nullptr;
    zk::TmaRun* d_tma_runs = nullptr;
    bool use_tma = false;  // TMA variant and its kernel fits on this device
    int occ_tma = 0;       // fused kernel, or the update pass of the two-pass TMA variant
    zk::TmaRun* d_tma_runs_r = nullptr;  // two-pass TMA variant: the reduce pass's table
    int occ_tma_r = 0;
    // stage 3: the layer gather from the Nd ranks' shards (a real rank: the
    // ranks' shards, peer-mapped; emulated ranks: places in the shard array)
    const uint16_t** d_shard_tab = nullptr;
    int64_t* d_shard_len = nullptr;
    zg::Run* d_rank_gather = nullptr;
    int occ_gather_ranks = 0;
    std::vector<const uint16_t*> shard_tab;  // host copy of what d_shard_tab holds
    bool shard_tab_valid = false;
    int64_t hold_tile = -1;  // test hook for the bounded waits (zero_test_hold_tile)
    unsigned hold_rounds = 0;
    int64_t hold_update_tile = -1;  // the same for the update pass (zero_test_hold_update_tile)
    unsigned hold_update_rounds = 0;
    bool async = false;      // between zero_async_begin and zero_async_end
    float async_b1 = 0.0f, async_b2 = 0.0f;
    zk::Ctrl ctrl_host{};    // staging copy of the control block
    zk::Ctrl* d_ctrl = nullptr;
    const uint16_t** d_grad_tab = nullptr;
    uint16_t** d_out_tab = nullptr;
    unsigned* d_flag = nullptr;
    std::vector<const uint16_t*> grad_tab;  // host copy of what d_grad_tab holds
    bool grad_tab_valid = false;
    std::vector<uint16_t*> out_tab;
    int cur = 0;  // live state buffer (fused variant)
    int64_t t = 0;
    unsigned call_id = 0;
    unsigned host_flag[2] = {0, 0};  // overflow word, kernel error word
    int last_cuda = 0;
    bool pending = false;  // launched, not yet committed
    int64_t pending_t = 0;
    int pending_next = 0;
    zk::StepArgs args{};   // arguments of the pending launch
    // beta^t products for the last t computed (t-fold double products)
    float bc_b1 = -1.0f, bc_b2 = -1.0f;
    int64_t bc_t = -1;
    double bc_p1 = 1.0, bc_p2 = 1.0;

    float* state(int buf, int k) const
    {
        return L.off_state[buf][k] < 0 ? nullptr : reinterpret_cast<float*>(ws + L.off_state[buf][k]);
    }
};

namespace {

int cuda_fail(zero_handle* h, cudaError_t e);

// The TMA-staged step with arguments a: the fused kernel, or the reduce and
// update passes (a.red set by the caller). hold_tile / wait_rounds: the test
// hook, applied to the first launch only.
// passes of a two-pass step to enqueue (the fused step is one pass)
constexpr int kRunReduce = 1, kRunUpdate = 2, kRunBoth = 3;
cudaError_t launch_tma_step(zero_handle* h, const zk::StepArgs& a, int64_t hold_tile, unsigned wait_rounds,
                            cudaStream_t s, int passes = kRunBoth);

// A single-rank-view handle that writes every rank's replica is rank r of a
// real job: the ranks agree on overflow between zero_step_launch and
// zero_step_commit. A two-pass step updates in place, so its update pass must
// wait for that agreement: zero_step_launch enqueues the reduce pass only and
// zero_step_commit the update pass.
// a rank of a real job: its outputs are the other ranks' replicas (stage 1/2)
// or its shard of a sharded job (stage 3); it agrees with the other ranks on
// overflow between launch and commit
bool real_rank(const Layout& L) { return L.view >= 0 && (L.n_out > 1 || L.stage == 3); }

bool defers_update(const Layout& L) { return real_rank(L) && !is_fused(L.variant); }

// The fused step without a master reads the weight from the last replica and
// writes all the others; K_REPLICA then completes or restores them.
void set_replica_roles(const Layout& L, zk::StepArgs& a)
{
    if (is_fused(L.variant) && L.bf16) {
        a.w_src = a.n_out - 1;
        a.keep_last = 1;
    }
}

int cuda_fail(zero_handle* h, cudaError_t e)
{
    if (h) h->last_cuda = (int)e;
    return ZERO_ERR_CUDA;
}

int grid_for(const zero_handle* h, zk::Kernel k, int64_t chunks)
{
    const int64_t warps_per_block = zk::kThreads / 32;
    const int64_t want = std::max<int64_t>(1, (chunks + warps_per_block - 1) / warps_per_block);
    const int64_t cap = (int64_t)h->sms * std::max(1, h->occ[k]);
    return (int)std::min(want, cap);
}

// The error word and the buffers' element extents every kernel argument
// carries (checked by the bounds-checked build).
void set_extents(const zero_handle* h, zk::StepArgs& a)
{
    const Layout& L = h->L;
    a.err = h->d_flag + 1;
    a.grad_len = L.grad_len;
    a.state_len = L.state_elems;
    a.out_len = L.stage == 3 ? L.state_elems : L.psi;
}

// The kernel-error word after a synchronising call (only the bounds-checked
// build sets it outside the steps): ZERO_ERR_INTERNAL, cleared, if it is set.
int check_error_word(zero_handle* h, cudaStream_t s)
{
    unsigned word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, h->d_flag + 1, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(h, e);
    if (word == 0) return ZERO_OK;
    e = cudaMemsetAsync(h->d_flag + 1, 0, sizeof(unsigned), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e == cudaSuccess ? ZERO_ERR_INTERNAL : cuda_fail(h, e);
}

// (double)b^t as the t-fold product, continued from the previous call when
// possible (same multiplications in the same order as a fresh loop).
void bias_corrections(zero_handle* h, float b1, float b2, int64_t t, float* bc1, float* bc2)
{
    if (!(b1 == h->bc_b1 && b2 == h->bc_b2 && h->bc_t >= 0 && h->bc_t <= t)) {
        h->bc_b1 = b1;
        h->bc_b2 = b2;
        h->bc_t = 0;
        h->bc_p1 = 1.0;
        h->bc_p2 = 1.0;
    }
    while (h->bc_t < t) {
        h->bc_p1 = h->bc_p1 * (double)b1;
        h->bc_p2 = h->bc_p2 * (double)b2;
        ++h->bc_t;
    }
    *bc1 = (float)(1.0 - h->bc_p1);
    *bc2 = (float)(1.0 - h->bc_p2);
}

}  // namespace

namespace {

cudaError_t launch_tma_step(zero_handle* h, const zk::StepArgs& a, int64_t hold_tile, unsigned wait_rounds,
                            cudaStream_t s, int passes)
{
    const Layout& L = h->L;
    zk::TmaArgs ta{};
    ta.b = a;
    ta.err = h->d_flag + 1;
    ta.wait_rounds = wait_rounds;
    ta.hold_tile = hold_tile;
    if (is_fused(L.variant)) {
        ta.runs = h->d_tma_runs;
        ta.n_runs = (int)L.tma_runs.size();
        ta.n_tiles = L.tma_tiles;
        ta.n_scal = L.tma_scal;
        const int64_t cap = (int64_t)h->sms * h->occ_tma;
        const int64_t want = std::max<int64_t>(1, std::max(L.tma_tiles, (L.tma_scal + 255) / 256));
        return zk::launch_step_tma(L.tma_shape, ta, (int)std::min(want, cap), s, L.bf16);
    }
    if (passes & kRunReduce) {
        ta.runs = h->d_tma_runs_r;
        ta.n_runs = (int)L.tma_runs_r.size();
        ta.n_tiles = L.tma_tiles_r;
        ta.n_scal = L.tma_scal_r;
        const int64_t cap = (int64_t)h->sms * h->occ_tma_r;
        const int64_t want = std::max<int64_t>(1, std::max(L.tma_tiles_r, (L.tma_scal_r + 255) / 256));
        const cudaError_t e = zk::launch_pass_tma(zk::kPassReduce, ta, (int)std::min(want, cap), s, L.bf16);
        if (e != cudaSuccess) return e;
    }
    if (!(passes & kRunUpdate)) return cudaSuccess;
    ta.runs = h->d_tma_runs;
    ta.n_runs = (int)L.tma_runs.size();
    ta.n_tiles = L.tma_tiles;
    ta.n_scal = L.tma_scal;
    ta.hold_tile = h->hold_update_tile;
    ta.wait_rounds = h->hold_update_tile >= 0 ? h->hold_update_rounds : zk::kTmaWaitRounds;
    h->hold_update_tile = -1;
    const int64_t cap = (int64_t)h->sms * h->occ_tma;
    const int64_t want = std::max<int64_t>(1, std::max(L.tma_tiles, (L.tma_scal + 255) / 256));
    return zk::launch_pass_tma(zk::kPassUpdate, ta, (int)std::min(want, cap), s, L.bf16);
}

}  // namespace

ZERO_API int zero_state_bytes(const zero_config* cfg, zero_ledger* out)
{
    if (!out) return ZERO_ERR_ARG;
    Layout L;
    const int rc = build_layout(cfg, &L);
    if (rc != ZERO_OK) return rc;
    fill_ledger(L, out);
    return ZERO_OK;
}

ZERO_API int zero_rank_shard(const zero_config* cfg, int32_t rank, int64_t* state_begin, int64_t* len)
{
    if (!state_begin || !len) return ZERO_ERR_ARG;
    Layout L;
    const int rc = build_layout(cfg, &L);
    if (rc != ZERO_OK) return rc;
    if (rank < 0 || rank >= L.nd) return ZERO_ERR_ARG;
    if (L.view >= 0) {  // the handle holds the viewed rank's shard alone, from 0
        *state_begin = 0;
        *len = rank == L.view ? L.state_elems : 0;
        return ZERO_OK;
    }
    *state_begin = L.shard_begin[rank];
    *len = L.shard_len[rank];
    return ZERO_OK;
}

ZERO_API int zero_gather_plan(const zero_config* cfg, int32_t unit, zero_gather_run* runs, int64_t cap,
                             int64_t* n_runs)
{
    if (!n_runs) return ZERO_ERR_ARG;
    Layout L;
    const int rc = build_layout(cfg, &L);
    if (rc != ZERO_OK) return rc;
    if (L.stage != 3) return ZERO_ERR_STAGE;
    if (unit < 0 || unit >= L.n_units) return ZERO_ERR_ARG;
    const Unit& U = L.units[unit];
    *n_runs = U.rank_n_runs;
    if (!runs) return ZERO_OK;
    if (cap < U.rank_n_runs) return ZERO_ERR_ARG;
    for (int64_t i = 0; i < U.rank_n_runs; ++i) {
        const zg::Run& g = L.rank_gather[U.rank_run0 + i];
        runs[i].src_begin = g.src_begin;
        runs[i].out_begin = g.out_begin;
        runs[i].len = g.len;
        runs[i].src_rank = g.rank;
        runs[i].reserved = 0;
    }
    return ZERO_OK;
}

ZERO_API int zero_unit_range(const zero_config* cfg, int32_t unit, int64_t* flat_begin, int64_t* numel)
{
    if (!flat_begin || !numel) return ZERO_ERR_ARG;
    Layout L;
    const int rc = build_layout(cfg, &L);
    if (rc != ZERO_OK) return rc;
    if (L.stage != 3) return ZERO_ERR_STAGE;
    if (unit < 0 || unit >= L.n_units) return ZERO_ERR_ARG;
    *flat_begin = L.units[unit].flat_begin;
    *numel = L.units[unit].numel;
    return ZERO_OK;
}

ZERO_API int zero_init(const zero_config* cfg, void* workspace, size_t workspace_bytes,
                       const float* master_init, uint16_t* const* param_bufs, void* stream,
                       zero_handle** out)
{
    const zk::NvtxRange nvtx_range("zero_init");
    if (!out) return ZERO_ERR_ARG;
    *out = nullptr;
    zero_handle* h = new (std::nothrow) zero_handle();
    if (!h) return ZERO_ERR_INTERNAL;
    int rc = build_layout(cfg, &h->L);
    if (rc != ZERO_OK) {
        delete h;
        return rc;
    }
    const Layout& L = h->L;
    // master_init may be NULL only when this handle owns no element (an
    // empty partition in the single-rank view)
    if (!workspace || (!master_init && L.state_elems > 0)) rc = ZERO_ERR_ARG;
    else if (!aligned16(workspace) || !aligned16(master_init)) rc = ZERO_ERR_ALIGN;
    else if ((int64_t)workspace_bytes < L.total) rc = ZERO_ERR_WORKSPACE;
    if (rc == ZERO_OK && L.stage <= 2) {
        if (!param_bufs) {
            rc = ZERO_ERR_ARG;
        } else {
            for (int k = 0; k < L.n_out && rc == ZERO_OK; ++k) {
                if (!param_bufs[k]) rc = ZERO_ERR_ARG;
                else if (!aligned16(param_bufs[k])) rc = ZERO_ERR_ALIGN;
            }
        }
    }
    if (rc != ZERO_OK) {
        delete h;
        return rc;
    }
    h->ws = static_cast<char*>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaGetDevice(&h->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->device);
    const int smem = zk::step_smem_bytes(L.nd, L.n_out);
    for (int k = 0; k < zk::K_COUNT && e == cudaSuccess; ++k)
        e = zk::occupancy((zk::Kernel)k, k == zk::K_GATHER ? 0 : smem, &h->occ[k], L.bf16);
    if (e != cudaSuccess) {
        rc = cuda_fail(h, e);
        delete h;
        return rc;
    }
    h->d_flag = reinterpret_cast<unsigned*>(h->ws + L.off_flag);
    h->d_ctrl = reinterpret_cast<zk::Ctrl*>(h->ws + L.off_flag + 64);
    h->d_grad_tab = reinterpret_cast<const uint16_t**>(h->ws + L.off_grad_tab);
    h->d_out_tab = reinterpret_cast<uint16_t**>(h->ws + L.off_out_tab);
    h->d_step_segs = reinterpret_cast<zk::SegDesc*>(h->ws + L.off_step_segs);
    if (L.tma_ok) {
        h->d_tma_runs = reinterpret_cast<zk::TmaRun*>(h->ws + L.off_tma_runs);
        if (is_fused(L.variant)) {
            e = zk::tma_prepare(L.tma_shape, L.nd, L.bf16, &h->occ_tma);
            h->occ_tma_r = h->occ_tma;
        } else {
            h->d_tma_runs_r = reinterpret_cast<zk::TmaRun*>(h->ws + L.off_tma_runs_r);
            e = zk::tma_pass_prepare(L.nd, L.n_out, L.bf16, &h->occ_tma_r, &h->occ_tma);
        }
        if (e != cudaSuccess) {
            rc = cuda_fail(h, e);
            delete h;
            return rc;
        }
        h->use_tma = h->occ_tma >= 1 && h->occ_tma_r >= 1;
    }
    if (L.off_shard_tab >= 0) {
        h->d_shard_tab = reinterpret_cast<const uint16_t**>(h->ws + L.off_shard_tab);
        h->d_shard_len = reinterpret_cast<int64_t*>(h->ws + L.off_shard_tab + 8 * (int64_t)L.nd);
        h->d_rank_gather = reinterpret_cast<zg::Run*>(h->ws + L.off_rank_gather);
        e = zg::occupancy(&h->occ_gather_ranks);
        if (e != cudaSuccess) {
            rc = cuda_fail(h, e);
            delete h;
            return rc;
        }
    }
    if (L.stage <= 2)
        h->out_tab.assign(param_bufs, param_bufs + L.n_out);
    else
        h->out_tab.assign(1, reinterpret_cast<uint16_t*>(h->ws + L.off_shard16));

    e = cudaMemsetAsync(h->ws + L.off_flag, 0, 256, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(h->d_out_tab, h->out_tab.data(), h->out_tab.size() * sizeof(uint16_t*),
                            cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && !L.step_segs.empty())
        e = cudaMemcpyAsync(h->d_step_segs, L.step_segs.data(), L.step_segs.size() * sizeof(zk::SegDesc),
                            cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && L.tma_ok)
        e = cudaMemcpyAsync(h->d_tma_runs, L.tma_runs.data(), L.tma_runs.size() * sizeof(zk::TmaRun),
                            cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && !L.tma_runs_r.empty())
        e = cudaMemcpyAsync(h->d_tma_runs_r, L.tma_runs_r.data(), L.tma_runs_r.size() * sizeof(zk::TmaRun),
                            cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && h->d_shard_tab && L.view < 0) {
        // emulated ranks: shard r starts at its place in the handle's own shard array
        const uint16_t* base = reinterpret_cast<const uint16_t*>(h->ws + L.off_shard16);
        h->shard_tab.resize(L.nd);
        for (int r = 0; r < L.nd; ++r) h->shard_tab[r] = base + L.shard_begin[r];
        h->shard_tab_valid = true;
        e = cudaMemcpyAsync(h->d_shard_tab, h->shard_tab.data(), L.nd * sizeof(uint16_t*), cudaMemcpyHostToDevice, s);
    }
    if (e == cudaSuccess && h->d_shard_len)
        e = cudaMemcpyAsync(h->d_shard_len, L.shard_len.data(), L.nd * sizeof(int64_t), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && h->d_rank_gather && !L.rank_gather.empty())
        e = cudaMemcpyAsync(h->d_rank_gather, L.rank_gather.data(), L.rank_gather.size() * sizeof(zg::Run),
                            cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && L.step_chunks > 0) {
        zk::StepArgs a{};
        a.segs = h->d_step_segs;
        a.n_segs = (int)L.step_segs.size();
        a.n_chunks = L.step_chunks;
        a.outs = h->d_out_tab;
        a.n_out = (int)h->out_tab.size();
        a.nd = L.nd;
        a.w_out = h->state(0, 0);
        a.m_out = h->state(0, 1);
        a.v_out = h->state(0, 2);
        a.master_init = master_init;
        a.flag = h->d_flag;
        set_extents(h, a);
        e = zk::launch_step(zk::K_INIT, a, grid_for(h, zk::K_INIT, L.step_chunks), s, L.bf16);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        rc = cuda_fail(h, e);
        delete h;
        return rc;
    }
    rc = check_error_word(h, s);
    if (rc != ZERO_OK) {
        delete h;
        return rc;
    }
    *out = h;
    return ZERO_OK;
}

ZERO_API int zero_step_launch(zero_handle* h, const uint16_t* const* grads, float loss_scale,
                              const zero_hyper* hp, void* stream)
{
    const zk::NvtxRange nvtx_range("zero_step_launch");
    if (!h || !grads || !hp) return ZERO_ERR_ARG;
    if (h->pending || h->async) return ZERO_ERR_ARG;  // uncommitted launch, or an asynchronous run is open
    if (!(loss_scale > 0.0f) || !std::isfinite(loss_scale)) return ZERO_ERR_ARG;
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->beta1) || !std::isfinite(hp->beta2) ||
        !std::isfinite(hp->eps) || !std::isfinite(hp->weight_decay))
        return ZERO_ERR_ARG;
    const Layout& L = h->L;
    for (int k = 0; k < L.nd; ++k) {
        if (!grads[k]) return ZERO_ERR_ARG;
        if (!aligned16(grads[k])) return ZERO_ERR_ALIGN;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (!h->grad_tab_valid || !std::equal(grads, grads + L.nd, h->grad_tab.begin())) {
        h->grad_tab.assign(grads, grads + L.nd);
        e = cudaMemcpyAsync(h->d_grad_tab, h->grad_tab.data(), L.nd * sizeof(uint16_t*),
                            cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return cuda_fail(h, e);
        h->grad_tab_valid = true;
    }
    if (++h->call_id == 0) ++h->call_id;  // 0 is the flag's initial value

    const int64_t t_new = h->t + 1;
    zk::StepArgs& a = h->args;
    a = zk::StepArgs{};
    a.segs = h->d_step_segs;
    a.n_segs = (int)L.step_segs.size();
    a.n_chunks = L.step_chunks;
    a.grads = h->d_grad_tab;
    a.outs = h->d_out_tab;
    a.nd = L.nd;
    a.n_out = (int)h->out_tab.size();
    a.flag = h->d_flag;
    a.call_id = h->call_id;
    set_extents(h, a);
    a.c.inv_scale = (float)(1.0 / (double)loss_scale);
    a.c.lr = hp->lr;
    a.c.b1 = hp->beta1;
    a.c.b2 = hp->beta2;
    a.c.omb1 = 1.0f - hp->beta1;
    a.c.omb2 = 1.0f - hp->beta2;
    a.c.eps = hp->eps;
    a.c.wd = hp->weight_decay;
    bias_corrections(h, hp->beta1, hp->beta2, t_new, &a.c.bc1, &a.c.bc2);

    const bool fused = is_fused(L.variant);
    const int nxt = fused ? 1 - h->cur : h->cur;
    set_replica_roles(L, a);
    a.w_in = h->state(h->cur, 0);
    a.m_in = h->state(h->cur, 1);
    a.v_in = h->state(h->cur, 2);
    a.w_out = h->state(nxt, 0);
    a.m_out = h->state(nxt, 1);
    a.v_out = h->state(nxt, 2);
    if (L.step_chunks > 0) {
        const int passes = defers_update(L) ? kRunReduce : kRunBoth;
        if (h->use_tma) {
            if (!fused) a.red = reinterpret_cast<float*>(h->ws + L.off_reduced);
            e = launch_tma_step(h, a, h->hold_tile, h->hold_tile >= 0 ? h->hold_rounds : zk::kTmaWaitRounds, s,
                                passes);
            h->hold_tile = -1;
        } else if (fused) {
            e = zk::launch_step(zk::K_STEP_FUSED, a, grid_for(h, zk::K_STEP_FUSED, L.step_chunks), s, L.bf16);
        } else {
            a.red = reinterpret_cast<float*>(h->ws + L.off_reduced);
            e = zk::launch_step(zk::K_REDUCE, a, grid_for(h, zk::K_REDUCE, L.step_chunks), s, L.bf16);
            if (e == cudaSuccess && (passes & kRunUpdate))
                e = zk::launch_step(zk::K_UPDATE, a, grid_for(h, zk::K_UPDATE, L.step_chunks), s, L.bf16);
        }
        if (e != cudaSuccess) return cuda_fail(h, e);
    }
    h->pending = true;
    h->pending_t = t_new;
    h->pending_next = nxt;
    return ZERO_OK;
}

ZERO_API int zero_step_commit(zero_handle* h, void* stream, int* skipped)
{
    const zk::NvtxRange nvtx_range("zero_step_commit");
    if (skipped) *skipped = 0;
    if (!h || !h->pending) return ZERO_ERR_ARG;
    h->pending = false;
    const Layout& L = h->L;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (defers_update(L) && L.step_chunks > 0) {
        // the update pass, after the ranks' agreement on the flag words (it
        // returns at once if the agreed words say overflow or a failed wait)
        if (h->use_tma)
            e = launch_tma_step(h, h->args, -1, zk::kTmaWaitRounds, s, kRunUpdate);
        else
            e = zk::launch_step(zk::K_UPDATE, h->args, grid_for(h, zk::K_UPDATE, L.step_chunks), s, L.bf16);
        if (e != cudaSuccess) return cuda_fail(h, e);
    }
    // a copy into pageable host memory returns once the stream has reached it
    e = cudaMemcpyAsync(h->host_flag, h->d_flag, 2 * sizeof(unsigned), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(h, e);
    const bool kernel_error = h->host_flag[1] != 0;
    if (is_fused(L.variant) && L.bf16 && L.step_chunks > 0) {
        // without a master: bring the last replica up to date, or on overflow
        // restore the others from it (the kernel reads the same words)
        e = zk::launch_step(zk::K_REPLICA, h->args, grid_for(h, zk::K_REPLICA, L.step_chunks), s, true);
        if (e != cudaSuccess) return cuda_fail(h, e);
    }
    if (h->host_flag[0] == h->call_id || kernel_error) {
        // Overflow (or a kernel that gave up a wait): the state buffers do not
        // switch (fused) or were never written (two-pass). The fused pass
        // already wrote fp16 parameters, so rewrite them from the unchanged
        // master (without a master the replica pass above restored them).
        if (is_fused(L.variant) && !L.bf16 && L.step_chunks > 0) {
            zk::StepArgs a = h->args;
            a.w_in = h->state(h->cur, 0);
            e = zk::launch_step(zk::K_CAST, a, grid_for(h, zk::K_CAST, L.step_chunks), s);
            if (e != cudaSuccess) return cuda_fail(h, e);
        }
        if (kernel_error) {
            e = cudaMemsetAsync(h->d_flag + 1, 0, sizeof(unsigned), s);
            if (e == cudaSuccess) e = cudaStreamSynchronize(s);
            if (e != cudaSuccess) return cuda_fail(h, e);
            // the in-place update pass gave up part of the way: nothing to roll back
            return (h->host_flag[1] & zk::kErrUpdate) ? ZERO_ERR_PARTIAL : ZERO_ERR_INTERNAL;
        }
        if (skipped) *skipped = 1;
        return ZERO_SKIPPED;
    }
    h->t = h->pending_t;
    h->cur = h->pending_next;
    return ZERO_OK;
}

ZERO_API int zero_step(zero_handle* h, const uint16_t* const* grads, float loss_scale,
                       const zero_hyper* hp, void* stream, int* skipped)
{
    if (skipped) *skipped = 0;
    const int rc = zero_step_launch(h, grads, loss_scale, hp, stream);
    if (rc != ZERO_OK) return rc;
    return zero_step_commit(h, stream, skipped);
}

ZERO_API int zero_async_begin(zero_handle* h, const uint16_t* const* grads, const zero_scaler* sc,
                              float beta1, float beta2, void* stream)
{
    if (!h || !grads || !sc || h->pending || h->async) return ZERO_ERR_ARG;
    // a rank of a real job agrees with the other ranks through launch/commit
    if (real_rank(h->L)) return ZERO_ERR_ARG;
    if (!(sc->init_scale > 0.0f) || !std::isfinite(sc->init_scale) || !(sc->growth_factor >= 1.0f) ||
        !std::isfinite(sc->growth_factor) || !(sc->backoff_factor > 0.0f) || !(sc->backoff_factor <= 1.0f) ||
        sc->growth_interval < 1 || !std::isfinite(beta1) || !std::isfinite(beta2))
        return ZERO_ERR_ARG;
    const Layout& L = h->L;
    for (int k = 0; k < L.nd; ++k) {
        if (!grads[k]) return ZERO_ERR_ARG;
        if (!aligned16(grads[k])) return ZERO_ERR_ALIGN;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    h->grad_tab.assign(grads, grads + L.nd);
    cudaError_t e = cudaMemcpyAsync(h->d_grad_tab, h->grad_tab.data(), L.nd * sizeof(uint16_t*),
                                    cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(h, e);
    h->grad_tab_valid = true;
    zk::Ctrl& c = h->ctrl_host;
    c = zk::Ctrl{};
    c.p1 = 1.0;
    c.p2 = 1.0;
    for (int64_t k = 0; k < h->t; ++k) {  // the t-fold products
        c.p1 = c.p1 * (double)beta1;
        c.p2 = c.p2 * (double)beta2;
    }
    c.t = h->t;
    c.scale = sc->init_scale;
    c.growth = sc->growth_factor;
    c.backoff = sc->backoff_factor;
    c.b1 = beta1;
    c.b2 = beta2;
    c.interval = sc->growth_interval;
    c.cur = h->cur;
    c.fused = is_fused(L.variant);
    zk::ctrl_next_constants(&c);
    e = cudaMemcpyAsync(h->d_ctrl, &c, sizeof(zk::Ctrl), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(h->d_flag, 0, sizeof(unsigned), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(h, e);
    h->async = true;
    h->async_b1 = beta1;
    h->async_b2 = beta2;
    return ZERO_OK;
}

ZERO_API int zero_step_async(zero_handle* h, const zero_hyper* hp, void* stream)
{
    const zk::NvtxRange nvtx_range("zero_step_async");
    if (!h || !hp || !h->async) return ZERO_ERR_ARG;
    if (hp->beta1 != h->async_b1 || hp->beta2 != h->async_b2) return ZERO_ERR_ARG;
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->eps) || !std::isfinite(hp->weight_decay))
        return ZERO_ERR_ARG;
    const Layout& L = h->L;
    if (L.step_chunks == 0) return ZERO_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    zk::StepArgs a{};
    a.segs = h->d_step_segs;
    a.n_segs = (int)L.step_segs.size();
    a.n_chunks = L.step_chunks;
    a.grads = h->d_grad_tab;
    a.outs = h->d_out_tab;
    a.nd = L.nd;
    a.n_out = (int)h->out_tab.size();
    a.flag = h->d_flag;
    set_extents(h, a);
    a.call_id = 1;  // the commit kernel clears the word after every step
    a.c.lr = hp->lr;
    a.c.b1 = hp->beta1;
    a.c.b2 = hp->beta2;
    a.c.omb1 = 1.0f - hp->beta1;
    a.c.omb2 = 1.0f - hp->beta2;
    a.c.eps = hp->eps;
    a.c.wd = hp->weight_decay;
    a.ctrl = h->d_ctrl;
    const int nb = is_fused(L.variant) ? 2 : 1;
    for (int b = 0; b < 2; ++b)
        for (int k = 0; k < 3; ++k) a.st[b][k] = h->state(b < nb ? b : 0, k);
    const bool fused = is_fused(L.variant);
    set_replica_roles(L, a);
    cudaError_t e;
    if (h->use_tma) {
        if (!fused) a.red = reinterpret_cast<float*>(h->ws + L.off_reduced);
        e = launch_tma_step(h, a, -1, zk::kTmaWaitRounds, s);
    } else if (fused) {
        e = zk::launch_step(zk::K_STEP_FUSED, a, grid_for(h, zk::K_STEP_FUSED, L.step_chunks), s, L.bf16);
    } else {
        a.red = reinterpret_cast<float*>(h->ws + L.off_reduced);
        e = zk::launch_step(zk::K_REDUCE, a, grid_for(h, zk::K_REDUCE, L.step_chunks), s, L.bf16);
        if (e == cudaSuccess)
            e = zk::launch_step(zk::K_UPDATE, a, grid_for(h, zk::K_UPDATE, L.step_chunks), s, L.bf16);
    }
    // the fused passes wrote fp16 parameters: rewrite them from the unchanged
    // master if the step overflowed (the kernel returns at once otherwise);
    // without a master the replica pass restores or completes them
    if (e == cudaSuccess && fused && L.bf16)
        e = zk::launch_step(zk::K_REPLICA, a, grid_for(h, zk::K_REPLICA, L.step_chunks), s, true);
    else if (e == cudaSuccess && fused)
        e = zk::launch_step(zk::K_CAST_IF, a, grid_for(h, zk::K_CAST, L.step_chunks), s);
    if (e == cudaSuccess) e = zk::launch_commit(h->d_ctrl, h->d_flag, h->d_flag + 1, s);
    return e == cudaSuccess ? ZERO_OK : cuda_fail(h, e);
}

ZERO_API int zero_async_end(zero_handle* h, void* stream, zero_async_state* out)
{
    if (!h || !h->async) return ZERO_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    zk::Ctrl c{};
    unsigned err = 0;
    cudaError_t e = cudaMemcpyAsync(&c, h->d_ctrl, sizeof(zk::Ctrl), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&err, h->d_flag + 1, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(h, e);
    h->async = false;
    h->t = c.t;
    h->cur = c.cur;
    h->bc_b1 = h->async_b1;  // continue the host's products where the device left them
    h->bc_b2 = h->async_b2;
    h->bc_t = c.t;
    h->bc_p1 = c.p1;
    h->bc_p2 = c.p2;
    if (out) {
        out->t = c.t;
        out->skipped = c.skipped;
        out->loss_scale = c.scale;
        out->good_steps = c.good;
    }
    if (err != 0) {
        e = cudaMemsetAsync(h->d_flag + 1, 0, sizeof(unsigned), s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_fail(h, e);
        return (err & zk::kErrUpdate) ? ZERO_ERR_PARTIAL : ZERO_ERR_INTERNAL;
    }
    return ZERO_OK;
}

namespace {

// One layer unit from the Nd shards the handle's table points to, with the
// copy kernel of zero_gather_ranks.cu.
int launch_rank_gather(zero_handle* h, const Unit& U, uint16_t* out, cudaStream_t s)
{
    if (U.rank_tiles == 0) return ZERO_OK;
    const Layout& L = h->L;
    zg::Args g{};
    g.runs = h->d_rank_gather + U.rank_run0;
    g.n_runs = (int)U.rank_n_runs;
    g.nd = L.nd;
    g.n_tiles = U.rank_tiles;
    g.shards = h->d_shard_tab;
    g.shard_len = h->d_shard_len;
    g.dst = out;
    g.dst_len = U.numel;
    g.err = h->d_flag + 1;
    const int64_t cap = (int64_t)h->sms * std::max(h->occ_gather_ranks, 1);
    const cudaError_t e = zg::launch(g, (int)std::min(U.rank_tiles, cap), s);
    return e == cudaSuccess ? ZERO_OK : cuda_fail(h, e);
}

}  // namespace

ZERO_API int zero_gather_layer(zero_handle* h, int32_t unit, uint16_t* out, void* stream)
{
    const zk::NvtxRange nvtx_range("zero_gather_layer");
    if (!h || h->pending) return ZERO_ERR_ARG;
    const Layout& L = h->L;
    if (L.stage != 3) return ZERO_ERR_STAGE;
    if (L.view >= 0) return ZERO_ERR_ARG;  // a rank's handle gathers with zero_gather_layer_ranks
    if (unit < 0 || unit >= L.n_units || !out) return ZERO_ERR_ARG;
    if (!aligned16(out)) return ZERO_ERR_ALIGN;
    const Unit& U = L.units[unit];
    return launch_rank_gather(h, U, out, static_cast<cudaStream_t>(stream));
}

ZERO_API int zero_gather_layer_ranks(zero_handle* h, int32_t unit, const uint16_t* const* shards, uint16_t* out,
                                    void* stream)
{
    const zk::NvtxRange nvtx_range("zero_gather_layer_ranks");
    if (!h || h->pending) return ZERO_ERR_ARG;
    const Layout& L = h->L;
    if (L.stage != 3) return ZERO_ERR_STAGE;
    if (L.view < 0 || !h->d_shard_tab) return ZERO_ERR_ARG;  // emulated ranks: zero_gather_layer
    if (unit < 0 || unit >= L.n_units || !out || !shards) return ZERO_ERR_ARG;
    if (!aligned16(out)) return ZERO_ERR_ALIGN;
    for (int k = 0; k < L.nd; ++k) {
        if (!shards[k] && L.shard_len[k] > 0) return ZERO_ERR_ARG;
        if (!aligned16(shards[k])) return ZERO_ERR_ALIGN;
    }
    const Unit& U = L.units[unit];
    if (U.rank_tiles == 0) return ZERO_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!h->shard_tab_valid || !std::equal(shards, shards + L.nd, h->shard_tab.begin())) {
        h->shard_tab.assign(shards, shards + L.nd);
        const cudaError_t e = cudaMemcpyAsync(h->d_shard_tab, h->shard_tab.data(), L.nd * sizeof(uint16_t*),
                                              cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return cuda_fail(h, e);
        h->shard_tab_valid = true;
    }
    return launch_rank_gather(h, U, out, s);
}

ZERO_API int zero_set_state(zero_handle* h, const float* master, const float* m, const float* v, int64_t t,
                           void* stream)
{
    const zk::NvtxRange nvtx_range("zero_set_state");
    if (!h || h->pending || h->async || t < 0) return ZERO_ERR_ARG;
    const Layout& L = h->L;
    const size_t bytes = (size_t)L.state_elems * sizeof(float);
    // without a master (bfloat16) the parameters live in the outputs; a
    // non-NULL master is then written to them, rounded to bfloat16
    if (L.state_elems > 0 && ((!master && !L.bf16) || !m || !v)) return ZERO_ERR_ARG;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v)) return ZERO_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const float* src[3] = {master, m, v};
    cudaError_t e = cudaSuccess;
    for (int k = 0; k < 3 && e == cudaSuccess && bytes > 0; ++k) {
        float* dst = h->state(h->cur, k);
        if (dst && dst != src[k]) e = cudaMemcpyAsync(dst, src[k], bytes, cudaMemcpyDeviceToDevice, s);
    }
    if (e == cudaSuccess && L.step_chunks > 0 && master) {
        // the 16-bit parameters follow the restored master
        zk::StepArgs a{};
        a.segs = h->d_step_segs;
        a.n_segs = (int)L.step_segs.size();
        a.n_chunks = L.step_chunks;
        a.outs = h->d_out_tab;
        a.n_out = (int)h->out_tab.size();
        a.nd = L.nd;
        a.w_in = L.bf16 ? master : h->state(h->cur, 0);
        a.flag = h->d_flag;
        set_extents(h, a);
        e = zk::launch_step(zk::K_CAST, a, grid_for(h, zk::K_CAST, L.step_chunks), s, L.bf16);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(h, e);
    const int rc = check_error_word(h, s);
    if (rc != ZERO_OK) return rc;
    h->t = t;
    h->bc_t = -1;  // recompute the bias-correction products for the new t
    return ZERO_OK;
}

ZERO_API int zero_current_state(const zero_handle* h, float** master, float** m, float** v, int64_t* t)
{
    if (!h || h->async) return ZERO_ERR_ARG;
    if (master) *master = h->state(h->cur, 0);
    if (m) *m = h->state(h->cur, 1);
    if (v) *v = h->state(h->cur, 2);
    if (t) *t = h->t;
    return ZERO_OK;
}

ZERO_API int zero_stream_copy(void* dst, const void* src, size_t bytes, void* stream)
{
    if (!dst || !src || bytes % 16 != 0) return ZERO_ERR_ARG;
    if (!aligned16(dst) || !aligned16(src)) return ZERO_ERR_ALIGN;
    if (bytes == 0) return ZERO_OK;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return ZERO_ERR_CUDA;
    const cudaError_t e = zk::launch_copy(dst, src, bytes, sms * 8, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ZERO_OK : ZERO_ERR_CUDA;
}

ZERO_API int zero_test_hold_tile(zero_handle* h, int64_t tile, uint32_t wait_rounds)
{
    if (!h || tile < 0 || wait_rounds == 0) return ZERO_ERR_ARG;
    h->hold_tile = tile;
    h->hold_rounds = wait_rounds;
    return ZERO_OK;
}

ZERO_API int zero_test_hold_update_tile(zero_handle* h, int64_t tile, uint32_t wait_rounds)
{
    if (!h || tile < 0 || wait_rounds == 0) return ZERO_ERR_ARG;
    if (h->L.variant != ZERO_VARIANT_TWO_PASS_TMA || !h->use_tma) return ZERO_ERR_ARG;
    h->hold_update_tile = tile;
    h->hold_update_rounds = wait_rounds;
    return ZERO_OK;
}

ZERO_API int zero_flag_words(zero_handle* h, uint32_t** words)
{
    if (!h || !words) return ZERO_ERR_ARG;
    *words = h->d_flag;
    return ZERO_OK;
}

ZERO_API int zero_uses_tma(const zero_handle* h) { return h ? (h->use_tma ? 1 : 0) : ZERO_ERR_ARG; }

ZERO_API int zero_last_cuda_error(const zero_handle* h) { return h ? h->last_cuda : 0; }

ZERO_API const char* zero_error_string(int code)
{
    switch (code) {
        case ZERO_OK: return "ok";
        case ZERO_SKIPPED: return "step skipped: non-finite unscaled gradient";
        case ZERO_ERR_ARG: return "invalid argument";
        case ZERO_ERR_ALIGN: return "device pointer not 16-byte aligned";
        case ZERO_ERR_STAGE: return "call not valid for this ZeRO stage";
        case ZERO_ERR_WORKSPACE: return "workspace too small";
        case ZERO_ERR_CUDA: return "CUDA error";
        case ZERO_ERR_INTERNAL: return "internal error";
        case ZERO_ERR_PARTIAL: return "update pass gave up part of the way: state partly updated, restore it";
        default: return "unknown error code";
    }
}

ZERO_API void zero_destroy(zero_handle* h) { delete h; }

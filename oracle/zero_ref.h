/*
 * Oracle for the ZeRO partitioned mixed-precision Adam step -- C interface.
 *
 * TEST INFRASTRUCTURE. This is a plain, slow, single-threaded CPU statement of
 * what the step computes, written from the pages' text. Only the test suite,
 * the package's smoke check and the benchmark's CPU-baseline leg may load it.
 * The product path (the CUDA library) never calls it and shares no code,
 * header, table or constant with it.
 *
 * Pages cited in this file:
 *   [P1] "Your 7.5B model's weights fit in 15 GB. Training state was 120 GB per
 *        GPU" (blog.teqners.com)
 *   [P2] "Engine Room", chapter 10 "ZeRO and the Memory Tricks"
 *        (hoshank.vercel.app)
 *   [P3] "DeepSpeed ZeRO: account for every training state" (chenhuiyu.github.io)
 *
 * fp16 values travel as their IEEE binary16 bit patterns (uint16_t).
 */
#ifndef ZERO_REF_H
#define ZERO_REF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Adam / AdamW hyper-parameters, all binary32. */
typedef struct zr_hyper {
    float lr;
    float beta1;
    float beta2;
    float eps;
    float weight_decay; /* decoupled, multiplied by lr; 0 gives plain Adam */
} zr_hyper;

/* ---- binary16 conversions (round to nearest, ties to even) ---- */
float    zr_f32_from_f16(uint16_t h);
uint16_t zr_f16_from_f32(float x);
uint16_t zr_f16_from_f64(double x);
void     zr_f32_from_f16_array(const uint16_t* h, float* out, int64_t n);
void     zr_f16_from_f32_array(const float* x, uint16_t* out, int64_t n);
/* One direct fp16 update w16 <- fp16(w16 + fp16(dw)), the update the pages say
 * fp16 cannot absorb ([P1] "Why you can't just delete the fp32 copies"). */
uint16_t zr_direct_f16_update(uint16_t w16, float dw);
void     zr_direct_f16_update_array(const uint16_t* w16, const float* dw, uint16_t* out, int64_t n);

/* ---- bfloat16 conversions (round to nearest, ties to even) ---- */
float    zr_f32_from_bf16(uint16_t h);
uint16_t zr_bf16_from_f32(float x);
uint16_t zr_bf16_from_f64(double x);
void     zr_f32_from_bf16_array(const uint16_t* h, float* out, int64_t n);
void     zr_bf16_from_f32_array(const float* x, uint16_t* out, int64_t n);

/* ---- partitions ---- */
/* Stage 1/2: rank r of nd owns flat [r*P, min((r+1)*P, psi)), P = ceil(psi/nd). */
void zr_partition(int64_t psi, int32_t nd, int32_t r, int64_t* begin, int64_t* end);
/* Stage 3: every tensor of n elements is split the same way, per tensor. */
void zr_chunk(int64_t n, int32_t nd, int32_t r, int64_t* begin, int64_t* end);
/* Stage 3: number of elements in rank r's shard (its chunks of all tensors). */
int64_t zr_shard_len(int32_t n_tensors, const int64_t* numel, int32_t nd, int32_t r);

/* ---- step scalars ---- */
/* bc_k = 1 - beta_k^t, with beta_k^t the t-fold double product of (double)beta_k,
 * rounded once to binary32. */
void  zr_bias_corrections(float beta1, float beta2, int64_t t, float* bc1, float* bc2);
/* 1/loss_scale computed in double and rounded once to binary32. */
float zr_inv_scale(float loss_scale);

/* ---- the step ---- */
/* Plain data parallelism, the result ZeRO must reproduce: every rank all-reduces
 * (sums, rank order 0..nd-1, in binary32) the nd fp16 gradients, unscales, and
 * runs the identical mixed-precision Adam update on the full vector.  One copy
 * of the replicated state is enough.  Returns 1 (and changes nothing, t
 * included) if any unscaled reduced gradient is not finite, else 0. */
int zr_dp_step(int64_t n, int32_t nd, const uint16_t* const* grads,
               float* w, float* m, float* v, uint16_t* p16,
               float loss_scale, const zr_hyper* hp, int64_t* t);

/* zr_dp_step with decoupled weight decay only where decay[i] != 0 (decay may
 * be NULL: every element decays); elements with decay[i] == 0 are updated with
 * weight decay 0. */
int zr_dp_step_masked(int64_t n, int32_t nd, const uint16_t* const* grads,
                      float* w, float* m, float* v, uint16_t* p16,
                      float loss_scale, const zr_hyper* hp, const uint8_t* decay,
                      int64_t* t);

/* A BF16 setup without fp32 master weights: nd bfloat16 gradients summed in
 * binary32 in rank order and unscaled, the same skip rule, then per element
 * w = fp32(w16); Adam on (w, m, v) as in zr_dp_step (decay mask as in
 * zr_dp_step_masked); w16 = bf16(w). Returns 1 on overflow (nothing changes). */
int zr_bf16_step(int64_t n, int32_t nd, const uint16_t* const* grads, uint16_t* w16,
                 float* m, float* v, float loss_scale, const zr_hyper* hp,
                 const uint8_t* decay, int64_t* t);

/* ZeRO stage 1/2 with nd ranks: reduce-scatter, a global overflow flag,
 * Adam on each rank's own partition of master/m/v, then an all-gather of the
 * fp16 partitions into every rank's replica.  w_sh[r], m_sh[r], v_sh[r] hold
 * rank r's partition; replicas[r] is rank r's full fp16 parameter vector. */
int zr_zero12_step(int64_t psi, int32_t nd, const uint16_t* const* grads,
                   float* const* w_sh, float* const* m_sh, float* const* v_sh,
                   uint16_t* const* replicas,
                   float loss_scale, const zr_hyper* hp, int64_t* t);

/* ZeRO stage 3 with nd ranks: every tensor is split into nd chunks; rank r's
 * shard is its chunks of all tensors in tensor order.  Rank r keeps fp16
 * parameters (p_sh[r]) only for its shard. */
int zr_zero3_step(int32_t n_tensors, const int64_t* numel, int32_t nd,
                  const uint16_t* const* grads,
                  float* const* w_sh, float* const* m_sh, float* const* v_sh,
                  uint16_t* const* p_sh,
                  float loss_scale, const zr_hyper* hp, int64_t* t);

/* Stage 3 on-demand gather of one layer unit: the unit's tensors, in tensor
 * order, each rebuilt whole from the nd ranks' chunks, packed back to back.
 * Returns the number of elements written. */
int64_t zr_zero3_gather(int32_t n_tensors, const int64_t* numel, const int32_t* unit_of,
                        int32_t nd, int32_t unit, const uint16_t* const* p_sh,
                        uint16_t* out);

/* ---- dynamic loss scaling (not on the pages; the usual reading) ----
 * After a skipped (overflowing) step the scale is multiplied by `backoff` and
 * the run of good steps restarts; after `interval` consecutive good steps it
 * is multiplied by `growth` (kept if that would overflow binary32). */
void zr_scaler_update(float* scale, int32_t* good, int overflow, float growth, float backoff,
                      int32_t interval);

/* ---- memory and communication ledger ---- */
/* Per-rank model-state bytes from the pages' formulas:
 * out = {16 psi, 4 psi + 12 psi/nd, 2 psi + 14 psi/nd, 16 psi/nd}. */
void zr_ledger_formula(double psi, double nd, double out[4]);
/* Same quantities in exact integer bytes for the rank holding the most state
 * (rank 0 under the ceil split).  If n_tensors > 0 the stage-3 figure uses the
 * per-tensor chunks, else the flat partition. */
void zr_ledger_exact(int64_t psi, int32_t nd, int32_t n_tensors, const int64_t* numel,
                     int64_t out[4]);
/* Elements sent per step, summed over all ranks, by ring collectives:
 * out = {reduce-scatter, all-gather, DP all-reduce, stage 1, stage 2, stage 3}. */
void zr_comm_elements(int64_t psi, int32_t nd, int64_t out[6]);

#ifdef __cplusplus
}
#endif
#endif

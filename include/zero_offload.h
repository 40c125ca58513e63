/*
 * zero_offload.h -- the offloaded step of libzero: the same ZeRO stage 1/2/3
 * step as zero.h, with the fp32 master weights and Adam moments kept in host
 * memory and the Adam update run by the host's cores.
 *
 * The operation ([P2] "Engine Room" ch. 10, "ZeRO and the Memory Tricks" --
 * "The Breakthrough": ZeRO-Offload keeps the fp16 parameters and the forward
 * and backward compute on the GPU and moves the fp32 states and the Adam
 * update to the host CPU and its RAM; it changes where the terms of the memory
 * formula live, not the formula; [P3] "DeepSpeed ZeRO: account for every
 * training state" -- "Offload trades capacity against movement": offload
 * lowers GPU residency at the price of transfers and host-side update time).
 *
 * One step computes exactly what zero_step computes (zero.h), element for
 * element and bit for bit:
 *   1. device: the rank-ordered fp32 sum of the Nd fp16 gradients, times
 *      inv_scale, over every owned element; one overflow flag for the step.
 *      If any unscaled gradient is inf or NaN the step is skipped (nothing
 *      changes, t included) and ZERO_SKIPPED is returned.
 *   2. per chunk of the state (state order, chunk_elems elements): the device
 *      computes the unscaled reduced gradient again and copies it to the host
 *      (4 bytes per element); the host updates master, m, v with Adam and
 *      rounds the new master to fp16; the fp16 chunk is copied back (2 bytes
 *      per element) and written to every output (stage 1/2: the Nd replicas;
 *      stage 3: the fp16 shards). Chunks are pipelined: while the host updates
 *      chunk k, chunk k+1 travels to the host and chunk k-1 to the device.
 * Reading: the pages list the gradient reduction among what moves to the
 * host; with Nd ranks the cross-rank sum is the reduce-scatter collective,
 * which stays on the device here, and what crosses PCIe is the reduced
 * partition (one vector), not the Nd gradients.
 *
 * Memory (all owned by the caller):
 *   - device workspace: tables, the overflow word, and per pipeline slot one
 *     fp32 and one fp16 chunk (zero_offload_ledger.device_bytes);
 *   - host state: master, m, v as three consecutive fp32 arrays of
 *     state_elems elements (ordinary host memory; 12 bytes per element);
 *   - host staging: page-locked memory (cudaHostAlloc or a pinned torch
 *     tensor) for the chunks in flight (host_staging_bytes).
 * Stage 3 keeps its fp16 shards in the caller's buffer param_bufs[0] (state
 * order, state_elems elements); zero_offload_gather_layer rebuilds a layer
 * unit from them as zero_gather_layer does.
 *
 * The library creates four CUDA streams and some events per handle (no device
 * memory); zero_offload_destroy releases them. Conventions of zero.h apply
 * (16-byte aligned device pointers, ordering on `stream`, one thread per
 * handle). Error codes are zero.h's.
 */
#ifndef ZERO_OFFLOAD_H
#define ZERO_OFFLOAD_H

#include <stddef.h>
#include <stdint.h>

#include "zero.h"

#ifdef __cplusplus
extern "C" {
#endif

#define ZERO_OFFLOAD_SLOTS 3                      /* chunks in flight per direction */
#define ZERO_OFFLOAD_DEFAULT_CHUNK (1LL << 22)    /* largest default chunk (elements) */

typedef struct zero_offload_ledger {
    int64_t state_elems;        /* elements of each host state array */
    int64_t host_state_bytes;   /* 12 * state_elems: master, m, v */
    int64_t host_staging_bytes; /* page-locked staging */
    int64_t device_bytes;       /* device workspace */
    int64_t chunk_elems;        /* elements per pipeline chunk */
    int64_t n_chunks;
    int64_t d2h_bytes_per_step; /* 4 * state_elems (reduced fp32 gradient) */
    int64_t h2d_bytes_per_step; /* 2 * state_elems (fp16 parameters) */
    int64_t device_state_bytes; /* per-rank model-state bytes left on the device,
                                   the formula's fp16 terms without the K term:
                                   stage 1: 2 psi + 2 psi; stage 2: 2 psi +
                                   2 P; stage 3: 4 S (P the largest partition,
                                   S the largest stage-3 shard) */
    int32_t n_out;              /* fp16 outputs written per element */
    int32_t reserved;
} zero_offload_ledger;

typedef struct zero_offload_handle zero_offload_handle;

/* Sizes for cfg (same rules as zero_state_bytes; variant is ignored;
 * precision must be ZERO_PRECISION_FP16).
 * chunk_elems: 0 = the default, min(ZERO_OFFLOAD_DEFAULT_CHUNK,
 * max(2^20, state_elems / 8 rounded up to 256)), capped by the state rounded up
 * to 256; else a multiple of 256 in [256, 2^30]. Host only. ZERO_OK or
 * ZERO_ERR_ARG. */
int zero_offload_bytes(const zero_config* cfg, int64_t chunk_elems, zero_offload_ledger* out);

/* Create a handle. master_init: HOST array of the initial fp32 master weights
 * in gradient order (grad_len elements: psi, or the partition for a rank view).
 * host_state: 3 * state_elems floats (the library writes master, m = v = 0).
 * param_bufs: stage 1/2 as in zero_init (Nd replicas, or 1 for a rank view,
 * each psi fp16 elements); stage 3: one device buffer of state_elems fp16
 * elements for the shards. The initial fp16 parameters are written to them on
 * `stream` before the call returns. n_threads: host threads of the update
 * (1..256; the calling thread is one of them).
 * Errors: ZERO_ERR_ARG (bad config, sizes, NULL, n_threads, staging not
 * page-locked), ZERO_ERR_ALIGN (device pointer or staging not 16-byte
 * aligned), ZERO_ERR_WORKSPACE (a buffer smaller than the ledger says),
 * ZERO_ERR_CUDA. */
int zero_offload_init(const zero_config* cfg, int64_t chunk_elems, void* device_ws, size_t device_bytes,
                      void* host_staging, size_t staging_bytes, float* host_state, const float* master_init,
                      uint16_t* const* param_bufs, int n_threads, void* stream, zero_offload_handle** out);

/* One step. grads: Nd device pointers as in zero_step. Returns after the host
 * update of every chunk; the fp16 outputs are complete when the work enqueued
 * on `stream` by the call is. ZERO_OK, ZERO_SKIPPED, ZERO_ERR_ARG,
 * ZERO_ERR_ALIGN or ZERO_ERR_CUDA (after which the handle refuses further
 * steps: the host state may be partly updated). */
int zero_offload_step(zero_offload_handle* h, const uint16_t* const* grads, float loss_scale,
                      const zero_hyper* hp, void* stream);

/* Stage 3: write layer unit `unit`'s full fp16 weights into `out` (device),
 * exactly as zero_gather_layer (zero.h): the unit's tensors in tensor order,
 * each rebuilt from the Nd ranks' chunks in the shard buffer. Ordered on
 * `stream` (after a step when the step's work on that stream is). ZERO_OK,
 * ZERO_ERR_STAGE (stage 1/2), ZERO_ERR_ARG, ZERO_ERR_ALIGN, ZERO_ERR_CUDA. */
int zero_offload_gather_layer(zero_offload_handle* h, int32_t unit, uint16_t* out, void* stream);

/* Checkpoint / resume: replace the host state with master, m, v (HOST
 * arrays of state_elems floats in state order, e.g. saved from
 * zero_offload_state) and the step count t, and rewrite the fp16 parameters
 * from the restored master on `stream` (complete when the call returns).
 * ZERO_OK, ZERO_ERR_ARG (NULL array with state_elems > 0, t < 0, or a handle
 * refusing steps), ZERO_ERR_CUDA. */
int zero_offload_set_state(zero_offload_handle* h, const float* master, const float* m, const float* v,
                           int64_t t, void* stream);

/* Host pointers to the live state (state order) and the step count. */
int zero_offload_state(zero_offload_handle* h, const float** master, const float** m, const float** v,
                       int64_t* t);

/* The host update alone, on caller host arrays: n elements of w, m, v, p16
 * updated from the unscaled gradient g with the bias corrections of step t
 * (t >= 1) and weight decay hp->weight_decay if decay != 0, else 0.
 * path: 0 = the one zero_offload_step uses on this CPU, 1 = portable code,
 * 2 = AVX2 + F16C (ZERO_ERR_ARG where the CPU lacks them). Host only; used to
 * check the host arithmetic without a GPU. */
int zero_offload_host_update(const float* g, float* w, float* m, float* v, uint16_t* p16, int64_t n,
                             const zero_hyper* hp, int64_t t, int decay, int path);

/* Release the handle, its streams, events and threads (the caller's memory
 * stays the caller's). Waits for the handle's device work. NULL is ignored. */
void zero_offload_destroy(zero_offload_handle* h);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_OFFLOAD_H */

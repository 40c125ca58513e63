/*
 * zero_peer.h -- peer buffers for rank r of a real Nd-rank data-parallel job:
 * how one rank's step reaches the other ranks' gradients and fp16 parameters.
 *
 * The operation these calls serve ([P1] "The part that sounds too good:
 * communication"; [P2] "ZeRO and the Memory Tricks" -- "The Breakthrough"):
 * stage 1/2 replace the gradient all-reduce by a reduce-scatter (rank r needs
 * partition r of every rank's gradient) and an all-gather of the updated fp16
 * partitions (every rank needs partition r of rank r's parameters). With one
 * process per GPU and the GPUs joined by NVLink/NVSwitch, rank r's handle
 * (zero_config.rank_view = r, view_outputs = Nd; zero.h) does both inside its
 * step: it loads partition r of the Nd gradients straight from the ranks'
 * memory and stores its new fp16 partition straight into the Nd ranks'
 * parameter buffers. These calls give it those addresses.
 *
 *   exporting rank:  zero_peer_export(buf, bytes, &desc)  -> send desc to the others
 *   importing rank:  zero_peer_open(&desc, &ptr)           -> ptr addresses buf
 *                    ... steps ...
 *                    zero_peer_close(&desc, ptr)
 *
 * A descriptor is plain bytes (send it with any transport: an all-gather of
 * the process group, a file, a socket). It names the CUDA allocation holding
 * the buffer (an IPC handle of the CUDA runtime), the buffer's byte offset in
 * that allocation and its length, and the exporting process. Buffers carved
 * out of a larger allocation (a caching allocator's segment) are fine: the
 * offset is found from the allocation's address range.
 *
 * Opening a descriptor exported by the calling process itself returns the
 * exported address unchanged and maps nothing, so a rank may open the whole
 * exchanged list, its own entry included. Opening several buffers of one
 * allocation maps it once (reference counted per allocation and device);
 * zero_peer_close unmaps it when the last of them is closed.
 *
 * Ordering is the caller's: before rank r's step reads the gradients every
 * rank must have finished writing its own, and no rank may read its
 * parameter buffer before every rank's step (and commit) has finished writing
 * into it. An NCCL all-reduce of one word on the step's stream, or a stream
 * synchronise plus a host barrier, gives both. The exporter must keep the
 * buffer allocated until every importer has closed it.
 *
 * Conventions: the calls act on the calling thread's current CUDA device; a
 * buffer on another GPU becomes addressable through peer access, which the
 * mapping enables. A descriptor of the calling process is returned as is:
 * peer access between that process's own devices is the caller's affair.
 * Errors: ZERO_ERR_ARG (NULL pointers, a zero or oversized length, memory that
 * is not device memory, a range outside its allocation, a descriptor with a
 * bad magic word or misaligned fields, a pointer that no open mapping of that
 * descriptor returned), ZERO_ERR_ALIGN (buffer not 16-byte aligned),
 * ZERO_ERR_CUDA (the IPC call or the address query failed, e.g. for memory
 * mapped by the virtual-memory API, which has no IPC handle, or a driver
 * without IPC). zero_peer_last_cuda_error returns the code of the last such
 * failure: a CUDA runtime error code, or for the address query the driver
 * API's result code. Thread safe.
 */
#ifndef ZERO_PEER_H
#define ZERO_PEER_H

#include <stddef.h>
#include <stdint.h>

#include "zero.h"

#ifdef __cplusplus
extern "C" {
#endif

#define ZERO_PEER_MAGIC 0x5A505231u /* "ZPR1" */

typedef struct zero_peer_desc {
    uint32_t magic;          /* ZERO_PEER_MAGIC */
    int32_t device;          /* the exporter's device ordinal (its own numbering) */
    uint64_t process;        /* random token of the exporting process */
    uint64_t offset;         /* byte offset of the buffer in its allocation */
    uint64_t bytes;          /* the buffer's length in bytes */
    uint64_t address;        /* the buffer's address in the exporting process */
    unsigned char ipc[64];   /* the allocation's CUDA IPC memory handle */
} zero_peer_desc;            /* 104 bytes, no padding */

/* Describe the device buffer [dev_ptr, dev_ptr + bytes) of this process for
 * other processes. dev_ptr: device memory of the current device, 16-byte
 * aligned; bytes > 0. */
int zero_peer_export(const void* dev_ptr, size_t bytes, zero_peer_desc* out);

/* Map a buffer described by zero_peer_export (in this or another process) and
 * return its address in this process in *dev_ptr. */
int zero_peer_open(const zero_peer_desc* desc, void** dev_ptr);

/* Release what zero_peer_open(desc) returned as dev_ptr. */
int zero_peer_close(const zero_peer_desc* desc, void* dev_ptr);

/* Number of allocations currently mapped by zero_peer_open (for tests). */
int zero_peer_open_count(void);

/* CUDA error code of the last failed peer call of any thread (0 if none). */
int zero_peer_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_PEER_H */

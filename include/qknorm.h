/*
 * qknorm.h -- C ABI of libqknorm.so: QK-Norm (RMSNorm of query and key
 * activations) in place on a fused QKV activation buffer, on NVIDIA B200
 * (sm_100a).
 *
 * Buffer layout ("combined QKV projection" lesson, GQA section: one fused
 * projection output split by head into Q, K and V widths).  The activation
 * is a row-major [T, row_stride] array of bf16 or fp32 in device memory:
 *
 *     columns [0, Hq*D)              Q   (Hq heads of head_dim D)
 *     columns [Hq*D, (Hq+Hk)*D)      K   (Hk heads)
 *     columns [(Hq+Hk)*D, W)         V   (Hk heads), W = (Hq + 2*Hk) * D
 *     columns [W, row_stride)        padding
 *
 * Both entry points overwrite the Q and K columns of every row with their
 * normalised values and never read or write V or the padding.
 *
 * Arithmetic: elements are widened to fp32, sums of squares accumulate in
 * fp32, the inverse RMS is 1/sqrt(S/L + eps) in fp32 (L = normalised length,
 * eps inside the square root; S/L is formed as S times 1/L rounded to fp32),
 * and each output, (x * rinv) * gamma per head and (x * gamma) * rinv
 * layerwise, is rounded once to the storage type: round to nearest even for
 * bf16 and fp16, and for FP8 E4M3 round to nearest even saturating to +-448.
 *
 * Common arguments
 *   qkv         device pointer to the fused buffer; 16-byte aligned.
 *   dtype       QKN_BF16, QKN_FP32, QKN_FP16 or QKN_FP8_E4M3 (storage type
 *               of qkv).
 *   T           number of tokens (rows), >= 0; T == 0 returns QKN_OK and
 *               launches nothing (qkv may then be NULL).
 *   Hq, Hk      query / key head counts, >= 0, Hq + Hk >= 1.
 *   D           head_dim: 64, 128 or 256.
 *   row_stride  elements between consecutive rows, >= W; row_stride *
 *               sizeof(element) must be a multiple of 16 bytes.
 *   gamma_q/k   fp32 device pointers, 16-byte aligned; gamma_k may be NULL
 *               when Hk == 0 and gamma_q may be NULL when Hq == 0.
 *   eps         finite, >= 0.
 *   stream      a cudaStream_t passed as void* (NULL = legacy default stream).
 *
 * Ownership and execution: every pointer is owned by the caller and must
 * stay valid until the work on `stream` completes.  The library allocates
 * no memory and keeps no per-call state; calls are asynchronous and
 * stream-ordered, and the caller synchronises.  Entry points are safe to call
 * from several host threads, except that calls of qknorm_layerwise_noalloc
 * share one scratch array per device and must be ordered on one stream (see
 * there).
 *
 * Errors: each entry point returns QKN_OK or a negative qkn_status and
 * launches nothing when an argument is rejected.  Validation touches no CUDA
 * API, so it runs on a host without a GPU.  QKN_ERR_CUDA means a CUDA runtime
 * call (device query or kernel launch) failed on this call;
 * qknorm_last_cuda_error() then returns that cudaError_t for the calling
 * thread.
 */
#ifndef QKNORM_H
#define QKNORM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QKN_BF16 = 0,     /* bfloat16                                            */
    QKN_FP32 = 1,     /* IEEE binary32                                       */
    QKN_FP16 = 2,     /* IEEE binary16                                       */
    QKN_FP8_E4M3 = 3  /* FP8 E4M3 (bias 7, no infinities, max finite 448)    */
} qkn_dtype;

typedef enum {
    QKN_OK = 0,
    QKN_ERR_NULL = -1,        /* a required pointer is NULL                     */
    QKN_ERR_SHAPE = -2,       /* negative sizes, no heads, row_stride < W       */
    QKN_ERR_ALIGN = -3,       /* qkv, gamma or row_stride bytes not 16-aligned  */
    QKN_ERR_NSHARDS = -4,     /* nshards not in {1,2,4,8} or not dividing heads */
    QKN_ERR_UNSUPPORTED = -5, /* dtype or head_dim not built, token too wide    */
    QKN_ERR_CUDA = -6,        /* CUDA runtime error on this call                */
    QKN_ERR_EPS = -7,         /* eps negative or not finite                     */
    QKN_ERR_TOO_LARGE = -8    /* T beyond qknorm_layerwise_noalloc's scratch    */
} qkn_status;

/*
 * Per-head QK-Norm (Qwen3 style).  Source: sglang PR #13189 "Add
 * turbomind_rms_norm to accelerate QK norm in Qwen3 models", Motivation and
 * Modifications (an RMSNorm whose hidden_size is head_dim), with the RMSNorm
 * definition of the SwiftQK review (pith.science verdict for arXiv
 * 2608.09160, core_discovery).  For every token t and head h < Hq + Hk, the
 * D-element row x at columns [h*D, (h+1)*D) becomes
 *     y_j = x_j * g_j / sqrt(sum_j(x_j^2) / D + eps),
 * with g = gamma_q[0..D) for query heads (h < Hq) and gamma_k[0..D) for key
 * heads.
 */
int qknorm_per_head(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D, int64_t row_stride,
                    const float *gamma_q, const float *gamma_k, float eps, void *stream);

/*
 * Layerwise QK-Norm in the SwiftQK form.  Sources: SwiftQK abstract
 * (newx.sg paper page: under tensor parallelism the normalisation factor of
 * layerwise QK-Norm depends on the full hidden vector, so ranks exchange only
 * scalar statistics) and the SwiftQK review (key_machinery: the per-rank
 * factor is replaced by 1/sqrt((sum_r S_local,r)/H + eps)).  Per token, the
 * q vector (columns [0, Hq*D), weight gamma_q[0..Hq*D)) and the k vector
 * (columns [Hq*D, (Hq+Hk)*D), weight gamma_k[0..Hk*D)) are each split into
 * nshards contiguous head-aligned slices (tensor-parallel split by head, the
 * lesson's follow-up); each slice's fp32 partial sum of squares S_r is
 * formed from that slice alone, the partials are combined as scalars, and
 * every element is scaled by 1/sqrt(S / L + eps) with L the FULL vector
 * length.  nshards is 1, 2, 4 or 8 and must divide both Hq and Hk.  All
 * shards run inside one kernel on one GPU; there is no cross-GPU traffic.
 * The reduction is a fixed tree whose subtrees are the shards, so the output
 * is bit-identical for every valid nshards.  A token's heads are split over
 * a thread-block cluster of 1, 2, 4 or 8 blocks (C, which must divide
 * Hq + Hk); each block keeps S = 2 tokens' worth of its heads staged in
 * shared memory (S = 3 for FP8 on inputs long enough for the x * gamma
 * overlap), so S * (Hq + Hk) / C * D * sizeof(element) + 8 * (Hq + Hk) + 16
 * bytes must fit the device's opt-in shared memory per block (227 KiB on
 * B200) for the cluster size chosen, else QKN_ERR_UNSUPPORTED.  The blocks of
 * a cluster pass head partials to one another through distributed shared
 * memory and wait for them on transaction barriers; each such wait gives up
 * after 2 seconds, which can only happen if the GPU misbehaves, and is then
 * counted (see qknorm_wait_timeouts) while the kernel runs to its end with
 * wrong results.  Such a call still returns QKN_OK, because the wait runs
 * after the call has returned: a caller that must know reads
 * qknorm_wait_timeouts before the call and again after synchronising with
 * it, and treats the outputs of a call during which the count grew as wrong.
 */
int qknorm_layerwise(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D, int64_t row_stride,
                     const float *gamma_q, const float *gamma_k, float eps, int nshards,
                     void *stream);

/*
 * Tensor-parallel layerwise QK-Norm, the two rank-local steps.  Sources: the
 * SwiftQK review (key_machinery and core_discovery: each rank reduces its
 * shard to a local sum of squares, the ranks exchange only these scalars, and
 * every element is scaled by the global factor 1/sqrt(S_global/H + eps)) and
 * the "combined QKV projection" lesson (tensor-parallel follow-up: each rank
 * holds its share of the Q heads and of the K/V heads).  A rank's buffer is
 * the fused QKV of its own heads: Hq query heads and Hk key/value heads here
 * are this rank's counts, in the layout described at the top.
 *
 * qknorm_layerwise_partials writes, for every token t, the fp32 sum of
 * squares of this rank's q columns to partials[2t] and of its k columns to
 * partials[2t+1] (0 when the rank has no such heads).  partials is
 * caller-owned device memory of 2*T floats, 8-byte aligned; qkv is only read.
 * The sums use the same fixed reduction tree as qknorm_layerwise.
 *
 * The caller then sums the partials over the ranks (for instance one
 * all-reduce of 2*T floats) and calls qknorm_layerwise_apply with the sums:
 * it scales this rank's q columns by gamma_q[j] / sqrt(sums[2t]/len_q + eps)
 * and its k columns by gamma_k[j] / sqrt(sums[2t+1]/len_k + eps), in place,
 * where len_q and len_k are the FULL q and k vector lengths over all ranks
 * (at least Hq*D and Hk*D, at most 2^24, else QKN_ERR_SHAPE) and gamma_q /
 * gamma_k this rank's slices (Hq*D and Hk*D floats).  sums is 2*T floats,
 * 8-byte aligned.  With a single rank, the two calls give exactly the output
 * of qknorm_layerwise.  Arguments and errors are otherwise those above.
 */
int qknorm_layerwise_partials(const void *qkv, int dtype, int64_t T, int Hq, int Hk, int D,
                              int64_t row_stride, float *partials, void *stream);

int qknorm_layerwise_apply(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D,
                           int64_t row_stride, const float *gamma_q, const float *gamma_k,
                           const float *sums, int64_t len_q, int64_t len_k, float eps,
                           void *stream);

/*
 * Layerwise QK-Norm that allocates nothing (no counterpart in the paper: it
 * exists for callers, not for the method).  Some callers cannot allocate GPU
 * memory when they call in: a runtime that hands out memory only from its
 * own fixed pool, an embedding application that forbids allocations on its
 * hot path, or code that runs while an allocator lock is held.  This entry
 * point gives them the result of qknorm_layerwise(..., nshards = 1, ...) -- same
 * arguments except nshards -- computed with the two tensor-parallel steps
 * above for a single rank, whose partial sums live in a static device array
 * inside the library instead of caller memory.  The caller still passes and
 * owns qkv and the weights.
 *
 * Limits and sharing:
 * - T may be at most 65536 (the array holds 2 * 65536 floats, 512 KiB, which
 *   every GPU that loads the library keeps until the process exits); larger T
 *   returns QKN_ERR_TOO_LARGE and launches nothing.
 * - The first call on a device looks up the array's device address (with that
 *   device current) and caches it; make that first call before any stream
 *   capture on the device.
 * - All calls share the one array per device.  Calls whose work overlaps on
 *   the GPU (other streams, or other host threads' streams) race on it and
 *   give wrong results; calls ordered on one stream are fine.  Every partial
 *   sum a call reads is written earlier in that same call, so leftovers from
 *   an earlier call never leak into a result.
 */
int qknorm_layerwise_noalloc(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D,
                             int64_t row_stride, const float *gamma_q, const float *gamma_k,
                             float eps, void *stream);

/*
 * Tensor-parallel layerwise QK-Norm with the scalar exchange inside the
 * kernel, as SwiftQK does it.  Sources: the SwiftQK abstract (ranks exchange
 * only scalar statistics instead of gathering the hidden vectors) and the
 * SwiftQK review (key_machinery: warp 0 of each block writes the partial sums
 * to the peers' buffers and waits on flags, and the weight multiplication
 * overlaps the exchange; major_comments[0]: the wait must not deadlock;
 * major_comments[2]: the ordering of flag and payload).
 *
 * A group of `world` ranks (1, 2, 4 or 8) holds every token; each rank holds
 * Hq query and Hk key/value heads of it in the fused layout described at the
 * top (its share, split by head).  One call per rank, with the same T and the
 * same sequence of calls on every rank: each block stages a token, forms its
 * heads' fp32 partial sums of squares and the rank's two sums (q, k) with the
 * fixed tree of qknorm_layerwise, stores them into every rank's receive
 * buffer, forms x * gamma while the other ranks' sums arrive, reads the world
 * ranks' sums back from its own buffer, combines them in a fixed pairwise
 * tree in rank order (every rank gets the same bits), and scales its columns
 * in place by 1/sqrt(S / L + eps) with L = Hq*D*world (q) or Hk*D*world (k).
 * gamma_q / gamma_k are this rank's slices (Hq*D and Hk*D floats).
 *
 * The exchange: each of a rank's partial sums travels as one 8-byte word
 * {fp32 value, 32-bit call tag}, written with a single point-to-point peer
 * store (one destination per store, no collective library) into the receive
 * buffer of each rank, which lives in that rank's device memory and is
 * mapped into the others with CUDA IPC.  A reader polls its own buffer until every rank's word of the token
 * carries the current call's tag.  Calls alternate between two halves of the
 * buffer, so the buffer is never cleared between calls.  The call's sequence
 * number (which picks the half and the tag) is kept in the communicator's
 * device memory and advanced by each launch, so the calls can be captured in
 * a CUDA graph and replayed.
 *
 * Waits: the blocks of one token on different ranks wait for one another.
 * Blocks take tokens in the same order on every rank, and a launch never has
 * more blocks per rank than fit resident at once; a launch that serves
 * several ranks of a local group, whose blocks wait on one another, is
 * cooperative (all blocks resident, or it fails with QKN_ERR_CUDA rather than
 * start partly), while a rank on its own GPU is launched like the other
 * kernels (its blocks wait only on other GPUs).  Each wait gives up after the
 * communicator's time limit; the first give-up of a call is counted
 * (qknorm_tp_comm_errors, and qknorm_wait_timeouts) and stops every other
 * wait of that call on this rank, so a call whose peer never comes ends
 * after about one time limit with wrong outputs instead of hanging.  Check
 * qknorm_tp_comm_errors after synchronising to detect it.
 *
 * qknorm_tp_comm_create: set up this process's rank on the current device:
 *   allocates its receive buffer (2 * max_tokens * world * 16 bytes plus 256,
 *   zeroed; max_tokens in [1, 2^24]) and writes its CUDA IPC handle (64 bytes,
 *   caller-owned) to ipc_handle.  timeout_s (0 < t <= 3600) is the time limit
 *   of each wait.  Returns QKN_ERR_NSHARDS for a bad world or rank.
 * qknorm_tp_comm_connect: ipc_handles holds the world ranks' handles in rank
 *   order (world * 64 bytes, as exchanged by the caller, e.g. an all-gather);
 *   opens the other ranks' buffers.  Every rank must be created before any
 *   connects.  A world of 1 needs no connect.
 * qknorm_tp_comm_create_local: a group of `world` ranks emulated on the
 *   current device (all receive buffers local; no IPC); one call of
 *   qknorm_layerwise_tp_p2p then serves every rank in one launch.
 * qknorm_tp_comm_destroy: unmaps and frees.  Every rank must first have
 *   finished its last call (synchronise, then meet at a barrier), since peers
 *   store into this rank's buffer.
 * qknorm_layerwise_tp_p2p: qkv, gamma_q and gamma_k are host arrays of device
 *   pointers, one entry per rank the communicator serves (1, or world for a
 *   local group, in rank order).  QKN_ERR_TOO_LARGE if T > max_tokens;
 *   QKN_ERR_UNSUPPORTED if not connected, the current device is not the
 *   communicator's, or the token is too wide for one block of at most 576
 *   threads with gamma in registers.
 *   Other arguments and errors as qknorm_layerwise.
 * qknorm_tp_comm_errors: waits of this communicator that gave up, since it was
 *   created (a blocking copy; synchronise with the calls first).
 */
typedef struct qkn_tp_comm qkn_tp_comm;

int qknorm_tp_comm_create(int world, int rank, int64_t max_tokens, double timeout_s,
                          qkn_tp_comm **comm, void *ipc_handle);
int qknorm_tp_comm_connect(qkn_tp_comm *comm, const void *ipc_handles);
int qknorm_tp_comm_create_local(int world, int64_t max_tokens, double timeout_s,
                                qkn_tp_comm **comm);
int qknorm_tp_comm_destroy(qkn_tp_comm *comm);
int qknorm_tp_comm_errors(qkn_tp_comm *comm, unsigned int *count);
int qknorm_layerwise_tp_p2p(qkn_tp_comm *comm, void *const *qkv, int dtype, int64_t T, int Hq,
                            int Hk, int D, int64_t row_stride, const float *const *gamma_q,
                            const float *const *gamma_k, float eps, void *stream);

/* Static English text for a qkn_status value (never NULL). */
const char *qknorm_status_string(int status);

/* cudaError_t of the calling thread's last QKN_ERR_CUDA (0 if none). */
int qknorm_last_cuda_error(void);

/* Number of in-kernel waits on the current device that gave up since the
 * library was loaded (see qknorm_layerwise); 0 in correct operation.  Copies
 * one device counter to *count with a blocking copy on the legacy default
 * stream, so the work queued before it has finished.  QKN_ERR_NULL if count
 * is NULL, QKN_ERR_CUDA if the copy fails. */
int qknorm_wait_timeouts(unsigned int *count);

/* ABI version: 100 * major + minor (1.01 added QKN_FP16 and QKN_FP8_E4M3, 1.02 the
 * tensor-parallel layerwise steps, 1.03 qknorm_wait_timeouts, 1.04
 * qknorm_layerwise_noalloc and QKN_ERR_TOO_LARGE, 1.05 the in-kernel
 * tensor-parallel exchange: qknorm_tp_comm_* and qknorm_layerwise_tp_p2p). */
int qknorm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QKNORM_H */

/*
 * rra.h - C ABI of the RRAttention prefill hot path on NVIDIA B200 (sm_100a).
 *
 * The path (RRAttention: "Dynamic Block Sparse Attention via Per-Head Round-Robin Shifts for
 * Long-Context Inference", abstract; and the research summary of the same paper, "Summary" and
 * "Key points"):
 *
 *   1. estimate  - in every stride of S tokens head h scores the one query at in-stride offset
 *                  (h + shift) mod S against the stride-summed keys, takes a causal softmax over
 *                  the stride-level scores, and sums the probabilities into B x B blocks.
 *   2. select    - per head and query-block row keep the smallest set of key blocks whose mass
 *                  reaches tau (the find_blocks rule of the XAttention review, section 3), plus
 *                  the diagonal block.
 *   3. attention - causal block-sparse attention over the kept blocks (GQA, online softmax).
 *
 * Conventions shared by every entry point
 *   - Tensors are row-major and contiguous: Q [batch, heads_q, seqlen, head_dim],
 *     K and V [batch, heads_kv, seqlen, head_dim], O like Q; all bf16.
 *   - GQA: query head h reads KV head h / (heads_q / heads_kv).
 *   - Block masses `mass` (fp32) and kept lists `kept_idx` (int32) are packed lower triangles,
 *     one per (batch, head): block row I occupies entries [I(I+1)/2, I(I+1)/2 + I + 1), entry J
 *     belongs to key block J. NB = seqlen / block rows; NB(NB+1)/2 entries per (batch, head).
 *     A kept row lists its key blocks in ascending order; unused entries hold -1.
 *     `kept_cnt` int32 [batch, heads_q, NB] is the length of each kept row.
 *   - Each estimated block row sums to 1: mass(I, J) = (1/m) sum over the m = block/stride
 *     sampled queries i of row I of the stride-softmax probabilities of the strides in block J.
 *   - All pointers are DEVICE pointers, 16-byte aligned, owned by the caller, except the host
 *     buffers of rra_prefill_host. The library never allocates or frees memory (rra_prefill_host
 *     creates two streams and a few events once per device); all work is enqueued on `stream` (a
 *     cudaStream_t; NULL = legacy default stream) and returns without synchronising, except
 *     rra_check_device_status.
 *   - Argument errors are reported before anything is enqueued. A failed launch returns
 *     RRA_ERR_CUDA. Kernels never trap: a device-side wait that exceeds its time limit, or an
 *     invalid kept list met by the attention kernel, sets a sticky error word in the workspace,
 *     which rra_check_device_status reads and clears.
 *   - An empty problem (batch == 0 or seqlen == 0) is valid and enqueues nothing.
 */
#ifndef RRA_H_
#define RRA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RRA_OK = 0,
  RRA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, inconsistent shape, bad tau, bad list */
  RRA_ERR_UNSUPPORTED = 2,    /* valid but not implemented: block != 128, head_dim, stride */
  RRA_ERR_WORKSPACE = 3,      /* workspace smaller than rra_workspace_bytes() */
  RRA_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed */
  RRA_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up waiting on a barrier (see status word) */
} rra_status;

typedef struct {
  int batch;          /* b >= 0 */
  int heads_q;        /* Hq >= 1 */
  int heads_kv;       /* Hkv >= 1, Hq % Hkv == 0 */
  int seqlen;         /* L >= 0, L % block == 0 */
  int head_dim;       /* d in {64, 128} */
  int block;          /* B; 128 is the only supported block size */
  int stride;         /* S in {4, 8, 16, 32}; must divide B */
  int shift;          /* round-robin shift; any integer, reduced mod S */
  float tau;          /* (0, 1]; tau >= 1 keeps every causal block */
  float softmax_scale;/* applied to q.k in both the estimate and the attention; <= 0 means
                         1/sqrt(head_dim) */
} rra_params;

typedef struct CUstream_st *rra_stream_t;   /* same type as cudaStream_t */

/* Bytes of device workspace needed by rra_estimate / rra_sparse_attn / rra_prefill for these
 * parameters on the CURRENT device (it depends on the device's SM count). Returns 0 if the
 * parameters are invalid. The workspace must be zero-filled once before its first use (this
 * clears the error word); afterwards the library keeps it consistent itself. One workspace must
 * not be used by two calls that may run concurrently. */
size_t rra_workspace_bytes(const rra_params *p);

/* Step 1 (estimate). q, k: bf16 inputs. mass: fp32 output, [b, Hq, NB(NB+1)/2] packed rows
 * summing to 1. The pooled keys and the per-row partial sums live in the workspace. */
rra_status rra_estimate(const rra_params *p, const void *q, const void *k, float *mass,
                        void *workspace, size_t workspace_bytes, rra_stream_t stream);

/* Steps 1 and 2: rra_estimate followed by rra_select on its masses, in one call. mass may be
 * NULL (then the masses live in the workspace, which rra_workspace_bytes accounts for);
 * kept_idx / kept_cnt as rra_select writes them. */
rra_status rra_estimate_select(const rra_params *p, const void *q, const void *k, float *mass,
                               int32_t *kept_idx, int32_t *kept_cnt, void *workspace,
                               size_t workspace_bytes, rra_stream_t stream);

/* Step 1, alternative estimator (the XAttention review, sections 2-3: antidiagonal scoring
 * with stride-level softmax): the same mass output and layout as rra_estimate, but the
 * stride-level score of query stride i against key stride j is the sum of the S logits on the
 * antidiagonal of that S x S sub-block, sum_{t<S} q_{iS+t} . k_{jS+S-1-t}, every head scoring
 * all of its queries (params->shift is ignored). Causal softmax over strides j <= i and block
 * sums as in rra_estimate; select and attention are unchanged. Same workspace as rra_estimate.
 * It costs S times the estimate's tensor-core work, and provides the comparison point for the
 * pattern-search time. */
rra_status rra_estimate_xattn(const rra_params *p, const void *q, const void *k, float *mass,
                              void *workspace, size_t workspace_bytes, rra_stream_t stream);

/* Step 2 (select). mass: fp32 [b, Hq, NB(NB+1)/2] (any non-negative values; negative or NaN
 * entries count as 0). For each row: sort J descending by mass (ties: smaller J first), keep the
 * shortest prefix whose running sum, accumulated in fp64, reaches tau * (fp64 row sum), add the
 * diagonal J = I, emit ascending. tau >= 1 keeps every block. Outputs kept_idx, kept_cnt. */
rra_status rra_select(const rra_params *p, const float *mass, int32_t *kept_idx,
                      int32_t *kept_cnt, rra_stream_t stream);

/* Step 3 (attention). out[b, h, t, :] = softmax over the keys u of the kept blocks of t's block
 * row with u <= t of (softmax_scale * q_t . k_u), applied to v; bf16 output, fp32 accumulation.
 * Any kept list is accepted (it need not contain the diagonal); a query with no key gets 0.
 * List entries that are out of [0, I] or not strictly ascending are skipped and flag
 * RRA_ERR_INVALID_ARG in the workspace error word. */
rra_status rra_sparse_attn(const rra_params *p, const void *q, const void *k, const void *v,
                           const int32_t *kept_idx, const int32_t *kept_cnt, void *out,
                           void *workspace, size_t workspace_bytes, rra_stream_t stream);

/* Steps 1-3 back to back on one stream. mass may be NULL (then it lives in the workspace,
 * which rra_workspace_bytes accounts for). kept_idx / kept_cnt are outputs. */
rra_status rra_prefill(const rra_params *p, const void *q, const void *k, const void *v,
                       void *out, float *mass, int32_t *kept_idx, int32_t *kept_cnt,
                       void *workspace, size_t workspace_bytes, rra_stream_t stream);

/* Steps 1-3 on HOST inputs and output, with the copies overlapped with the compute. It has no
 * counterpart in the paper: it is a convenience of this library. q_host, k_host, v_host and
 * out_host are host buffers in the layouts of rra_prefill; pinned (page-locked) memory lets the
 * copies run asynchronously. q_dev, k_dev, v_dev, out_dev are device staging buffers of the same
 * sizes, kept_idx / kept_cnt device outputs as in rra_prefill; the masses stay in the workspace,
 * which must hold rra_workspace_bytes(p).
 * The problem is cut into up to 32 chunks. With batch == 1 a chunk is a group of query heads
 * within one KV head, or whole KV heads when there are more than 32; the KV head's K and V are
 * copied with its first group. Otherwise a chunk is a group of batch rows. Each chunk is an
 * independent sub-problem, because every step is per (batch row, head); a chunk of heads runs
 * with the round-robin shift advanced by its
 * first query head, so every head samples the offset it would sample in the whole problem, and
 * the results equal rra_prefill's. Chunk c's host-to-device copies run on an internal stream,
 * its estimate, select and attention on `stream` once they have landed, and its output copy on
 * a second internal stream, so chunk c+1's inputs and chunk c-1's output cross PCIe while chunk
 * c computes. Each copy is one cudaMemcpyAsync. The call is asynchronous: `stream` completes
 * after the last output copy, and the staging buffers are used only after the work already on
 * `stream`. The internal streams and events are created on the first call on each device (make
 * it before any stream capture) and kept until exit; calls on one device must not overlap.
 * Errors as for rra_prefill. */
rra_status rra_prefill_host(const rra_params *p, const void *q_host, const void *k_host,
                            const void *v_host, void *out_host, void *q_dev, void *k_dev,
                            void *v_dev, void *out_dev, int32_t *kept_idx, int32_t *kept_cnt,
                            void *workspace, size_t workspace_bytes, rra_stream_t stream);

/* Step 1 (estimate) for callers that cannot allocate device memory. It has no counterpart in
 * the paper: it is a convenience of this library. Same inputs, output and validation as
 * rra_estimate, but no workspace argument: the scratch lives in a fixed 48 MiB array inside the
 * library's device image, which every device that loads the library keeps until the process
 * exits. Meant for callers whose device memory is owned by a pool that forbids new
 * allocations, or that must avoid cudaMalloc / cudaFree because those calls can synchronise the
 * device. Problems whose rra_workspace_bytes exceeds 48 MiB return RRA_ERR_WORKSPACE before
 * anything is enqueued (on a 148-SM B200: a 32-query-head, 8-KV-head, d = 128 layer at S = 8 fits
 * up to 23K tokens). All calls share the one array: calls whose kernels may overlap on the GPU
 * (other streams, other threads) race, so serialise them. The first call on each device looks
 * up the array's device address and clears its status word; make it before any stream capture
 * begins. Device-side errors (an expired barrier wait) go to the array's sticky status word,
 * which rra_static_scratch_status reads and clears. Allocates nothing. */
rra_status rra_estimate_static_scratch(const rra_params *p, const void *q, const void *k,
                                       float *mass, rra_stream_t stream);

/* Device status of the fixed scratch array used by rra_estimate_static_scratch, which has no
 * workspace a caller could hand to rra_check_device_status. No counterpart in the paper either.
 * Synchronises `stream`, reads the array's sticky error word and clears it; returns as
 * rra_check_device_status does (RRA_ERR_DEVICE_TIMEOUT if a barrier wait of an earlier
 * static-scratch call expired: that call's masses are then undefined, and calls made since
 * returned without computing). raw_word may be NULL. Allocates nothing. */
rra_status rra_static_scratch_status(rra_stream_t stream, uint32_t *raw_word);

/* Synchronises `stream`, reads the workspace error word and clears it. Returns RRA_OK,
 * RRA_ERR_DEVICE_TIMEOUT (a barrier wait expired), RRA_ERR_INVALID_ARG (a kept list was
 * invalid) or RRA_ERR_CUDA. If raw_word is non-NULL the raw word is stored there. */
rra_status rra_check_device_status(void *workspace, rra_stream_t stream, uint32_t *raw_word);

/* Time limit of the kernels' device-side barrier waits, in nanoseconds, for every call made
 * after it in this process (default 4 s; 0 restores the default). A diagnostic and test hook:
 * a very short limit makes a kernel give up waiting, drain the copies and MMAs it has in flight,
 * set RRA_ERR_DEVICE_TIMEOUT in the status word and return, which is how the timeout path is
 * exercised without a real hang. */
void rra_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code. */
const char *rra_status_string(rra_status s);

/* Library version, e.g. "rra 0.1 sm_100a". */
const char *rra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RRA_H_ */

/*
 * fa_b200.h - C ABI of the B200 (sm_100a) exact-attention library libfa_b200.so.
 *
 * Exact scaled-dot-product attention O = softmax(scale * Q K^T [+ causal mask]) V,
 * computed tile by tile with an online softmax so that the N x N score matrix
 * never reaches device memory ("DL101 chapter 9", handsonai.io, section 3.3
 * FlashAttention; "Flash Attention: principle & practice", holysheep.ai,
 * sections 2.1 Online Softmax and 2.2 Tiling).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are contiguous, row-major, in device memory, and 16-byte aligned.
 *    "bf16" arguments are void pointers to IEEE bfloat16 bit patterns.
 *  - Q, K, V, O, dO, dQ, dK, dV are [B, H, N, d] (batch, head, sequence, head
 *    dimension; the multi-head layout of "DL101 chapter 9", section 3).
 *    LSE and D are [B, H, N] float32.  The ragged-batch entry points
 *    (_varlen) take sequences packed token-major, [total, heads, d], and the
 *    paged decode takes page pools; each states its layout.
 *  - Supported head dimensions: d = 64 and d = 128 (fa_fwd_fp8: 128).  Any
 *    N >= 0 (ragged tails are masked inside the kernels).
 *  - Key / value tensors may have fewer heads than queries (Hkv dividing H;
 *    the _gqa, _ext, _varlen, _paged and _fp8 entry points): query head h
 *    attends key / value head h / (H / Hkv) ("DL101 chapter 9", sections 3.1
 *    MQA and 3.2 GQA).
 *  - scale multiplies Q K^T before the softmax; callers normally pass
 *    1/sqrt(d) ("DL101 chapter 9", section 1.1).
 *  - Causal masking keeps key j for query i iff j <= i + Nk - Nq (diagonal
 *    included; with Nq = Nk = N simply j <= i).  With Nq != Nk (the _ext
 *    entry points) the Nq queries are the last Nq positions of the Nk-token
 *    sequence, i.e. a chunk of new tokens over a cache ("DL101 chapter 9",
 *    section 1.1: token t attends K_{<=t}).  A query that sees no key
 *    (only when Nq > Nk) gets O = 0 and LSE = -inf.
 *  - LSE is the natural-log log-sum-exp of the row's scaled, masked scores:
 *    LSE_i = ln sum_j exp(scale * q_i . k_j).
 *  - The caller allocates and owns every buffer, workspaces included.  The
 *    library allocates no device memory; it keeps only per-process state
 *    (a driver entry point, device properties and a device error word).
 *  - All calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL
 *    is the legacy default stream).  Argument errors are reported before any
 *    launch and leave the outputs untouched.  A failed launch returns
 *    FA_ERR_CUDA.  A kernel whose bounded wait expired records FA_ERR_TIMEOUT
 *    in the device error word (read it with fa_get_device_error); kernels
 *    never trap.
 *  - The current CUDA device must be the one that holds the buffers.
 *  - No C++ exception crosses this interface.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fa_stream_t; /* same type as cudaStream_t */
typedef struct CUevent_st* fa_event_t;   /* same type as cudaEvent_t  */

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer      */
    FA_ERR_UNSUPPORTED = 2,  /* head dimension other than 64 / 128, no sm_100   */
    FA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required      */
    FA_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed             */
    FA_ERR_TIMEOUT = 5,      /* a kernel's bounded wait expired (device word)   */
    FA_ERR_BOUNDS = 6        /* debug build only: a kernel's bounds check failed
                                and the access was skipped (device word)        */
} fa_status;

/*
 * Forward pass.  "DL101 chapter 9", section 3.3 (tiled FlashAttention:
 * running max m and sum l, O <- O*c + P V, final O / l) and "Flash Attention:
 * principle & practice", section 2.1 (online softmax).
 *   q, k, v : bf16 [B, H, N, d], read only.
 *   o       : bf16 [B, H, N, d], written.
 *   lse     : float32 [B, H, N], written; may be NULL when not needed.
 *   causal  : 0 or 1.
 * Returns FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED or FA_ERR_CUDA.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, int causal, float scale,
                 fa_stream_t stream);

/*
 * Grouped-query forward ("DL101 chapter 9", sections 3.1 MQA and 3.2 GQA):
 * k and v are bf16 [B, Hkv, N, d] and query head h of batch b attends key /
 * value head h / (H / Hkv) of that batch.  Hkv must divide H; Hkv = H is
 * fa_fwd, Hkv = 1 multi-query attention.  Everything else as fa_fwd.
 */
fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int Hkv, int N, int d, int causal, float scale,
                     fa_stream_t stream);

/*
 * Forward with separate query and key lengths, grouped heads allowed (the
 * non-square Lq x Lk problem of "DL101 chapter 9", section 3.3):
 *   q       : bf16 [B, H, Nq, d], read only.
 *   k, v    : bf16 [B, Hkv, Nk, d], read only.
 *   o       : bf16 [B, H, Nq, d], written.
 *   lse     : float32 [B, H, Nq], written; may be NULL.
 * Nq, Nk >= 0 with Nq + Nk < 2^31.  Causal masking is bottom-right aligned
 * (see the conventions above).  Nk = 0 writes O = 0 and LSE = -inf.
 * Pointers to arrays of zero size may be NULL.
 * fa_fwd_gqa(..., N, ...) is fa_fwd_ext(..., N, N, ...).  Returns as fa_fwd.
 */
fa_status fa_fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     fa_stream_t stream);

/*
 * Forward over a ragged batch: B sequences of different lengths packed
 * without padding (each sequence is the attention problem of its own rows;
 * "DL101 chapter 9", section 3.3 for Lq x Lk).
 *   q            : bf16 [total_q, H, d], token-major: the rows of sequence b
 *                  are cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1; read only.
 *   k, v         : bf16 [total_k, Hkv, d], likewise with cu_seqlens_k.
 *   o            : bf16 [total_q, H, d], written.
 *   lse          : float32 [H, total_q], written; may be NULL.
 *   cu_seqlens_q,
 *   cu_seqlens_k : int32 [B + 1] in DEVICE memory: 0, then the running sums
 *                  of the lengths, ending at total_q / total_k.  A sequence
 *                  whose range leaves the packed array is treated as empty.
 *   max_seqlen_q : host upper bound of the query lengths (sizes the launch).
 *                  A longer sequence records FA_ERR_INVALID_ARG in the device
 *                  error word and its rows past max_seqlen_q are not written.
 * Causal masking is bottom-right aligned per sequence (query i of a sequence
 * keeps key j iff j <= i + Lk_b - Lq_b).  A sequence with no keys gets O = 0,
 * LSE = -inf.  Pointers to empty arrays may be NULL.  Returns as fa_fwd.
 */
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k,
                        int B, int H, int Hkv, int total_q, int total_k, int max_seqlen_q,
                        int d, int causal, float scale, fa_stream_t stream);

/*
 * Forward with 8-bit float inputs (e4m3, OCP FP8): the FP8 path the pages
 * mention for FlashAttention-3 ("Flash Attention La Gi?", FlashAttention-3).
 * The pages give no scaling convention; here each input tensor carries one
 * descale factor (real value = stored e4m3 value x factor), the products run
 * on the tensor core's 8-bit path with f32 accumulation, and the softmax
 * probabilities are rounded to e4m3 before the P V product (relative error
 * up to 2^-4 per probability, so O carries a few percent relative error).
 *   q       : e4m3 [B, H, Nq, 128] (bytes), read only.
 *   k       : e4m3 [B, Hkv, Nk, 128], read only.
 *   vt      : e4m3 [B, Hkv, 128, Nk]: V transposed (row r holds component r
 *             of every value), read only.  Nk must be a multiple of 16.
 *   q_scale, k_scale, v_scale : the descale factors.
 *   o       : bf16 [B, H, Nq, 128], written (real, descaled values).
 *   lse     : float32 [B, H, Nq], written; may be NULL.
 *   d       : must be 128.
 * Masking, grouping, scale and errors as fa_fwd_ext; FA_ERR_UNSUPPORTED for
 * d != 128 or Nk not a multiple of 16.
 */
fa_status fa_fwd_fp8(const void* q, const void* k, const void* vt, void* o, float* lse,
                     float q_scale, float k_scale, float v_scale,
                     int B, int H, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     fa_stream_t stream);

/*
 * Bytes of device workspace fa_bwd needs: D = rowsum(dO * O) and
 * log2(e) * LSE as float32 [B, H, Np] with Np = N rounded up to a multiple
 * of 128, the float32 dQ accumulator [B, H, N, d] and one uint32
 * completion counter per (b, h), each region 256-byte aligned.  Returns 0
 * for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass with recomputation ("Flash Attention La Gi?", thienlv.com,
 * Recomputation: scores are recomputed from Q, K, V and the saved LSE
 * instead of being stored).  Gradients of sum(O * dO):
 *   dV = P^T dO, dP = dO V^T, D = rowsum(dO * O), dS = P * (dP - D),
 *   dQ = scale dS K, dK = scale dS^T Q.
 *   q, k, v, o, dout : bf16 [B, H, N, d], read only (o and lse from fa_fwd).
 *   lse              : float32 [B, H, N], read only.
 *   dq, dk, dv       : bf16 [B, H, N, d], written.
 *   workspace        : device buffer of at least fa_bwd_workspace_size bytes,
 *                      256-byte aligned, owned by the caller; contents on
 *                      entry are ignored, on exit unspecified.
 * Returns FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE or
 * FA_ERR_CUDA.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o,
                 const void* dout, const float* lse, void* dq, void* dk, void* dv,
                 void* workspace, size_t ws_bytes,
                 int B, int H, int N, int d, int causal, float scale,
                 fa_stream_t stream);

/*
 * Grouped-query backward: k, v, dk, dv are [B, Hkv, N, d]; the gradient of a
 * shared key / value head is the sum over its H / Hkv query heads.  The
 * workspace is fa_bwd_workspace_size(B, H, N, d).  Everything else as fa_bwd.
 */
fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                     void* workspace, size_t ws_bytes,
                     int B, int H, int Hkv, int N, int d, int causal, float scale,
                     fa_stream_t stream);

/*
 * Backward with separate query and key lengths (the inverse of fa_fwd_ext):
 *   q, o, dout : bf16 [B, H, Nq, d], read only;  lse : float32 [B, H, Nq].
 *   k, v       : bf16 [B, Hkv, Nk, d], read only.
 *   dq         : bf16 [B, H, Nq, d], written.
 *   dk, dv     : bf16 [B, Hkv, Nk, d], written.
 *   workspace  : fa_bwd_workspace_size(B, H, Nq, d) bytes (not needed when
 *                Nq or Nk is 0).
 * Queries with LSE = -inf (they saw no key) contribute nothing.  Nq = 0
 * writes dK = dV = 0; Nk = 0 writes dQ = 0.  Pointers to arrays of zero size
 * may be NULL.  Returns as fa_bwd.
 */
fa_status fa_bwd_ext(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                     void* workspace, size_t ws_bytes,
                     int B, int H, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     fa_stream_t stream);

/*
 * Bytes of device workspace fa_bwd_varlen needs: D and log2(e) * LSE as
 * float32 [H, P] (every sequence's rows in their own padded segment, P about
 * total_q + 132 B), then the float32 dQ accumulator [total_q, H, d], each
 * region 256-byte aligned.  Returns 0 for invalid sizes.
 */
size_t fa_bwd_varlen_workspace_size(int B, int H, int total_q, int d);

/*
 * Backward over a ragged batch (the inverse of fa_fwd_varlen; recomputation
 * as fa_bwd):
 *   q, o, dout   : bf16 [total_q, H, d] token-major, read only.
 *   lse          : float32 [H, total_q] from fa_fwd_varlen, read only.
 *   k, v         : bf16 [total_k, Hkv, d], read only.
 *   dq           : bf16 [total_q, H, d], written.
 *   dk, dv       : bf16 [total_k, Hkv, d], written (zero for keys that no
 *                  query sees and for rows outside every sequence).
 *   cu_seqlens_q,
 *   cu_seqlens_k : int32 [B + 1] in device memory, as fa_fwd_varlen.
 *   max_seqlen_k : host upper bound of the key lengths (sizes the launch).
 *   workspace    : fa_bwd_varlen_workspace_size(B, H, total_q, d) bytes,
 *                  256-byte aligned, owned by the caller.
 * Returns FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE or
 * FA_ERR_CUDA.
 */
fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        const int* cu_seqlens_q, const int* cu_seqlens_k,
                        void* workspace, size_t ws_bytes,
                        int B, int H, int Hkv, int total_q, int total_k, int max_seqlen_k,
                        int d, int causal, float scale, fa_stream_t stream);

/*
 * Bytes of device workspace fa_decode needs for the split-KV partials
 * (per batch, head and split: running max, running sum and an unnormalised
 * d-vector, float32) for caches of capacity Lmax.  Returns 0 for invalid
 * sizes.
 */
size_t fa_decode_workspace_size(int B, int H, int Lmax, int d);

/*
 * KV-cache decode: one new query per (batch, head) attends the cached keys
 * and values at positions 0 .. seqlens[b]-1 ("DL101 chapter 9", section 1.1
 * Key/Value Caching), split over chunks of the cache whose partial softmax
 * states are merged afterwards with the rescale-and-add rule of "Flash
 * Attention: principle & practice", section 2.1.
 *   q       : bf16 [B, H, d], read only.
 *   kcache,
 *   vcache  : bf16 [B, H, Lmax, d], read only; rows at or beyond seqlens[b]
 *             are never read.
 *   seqlens : int32 [B] in DEVICE memory, 0 <= seqlens[b] <= Lmax (values
 *             outside are clamped to that range).
 *   o       : bf16 [B, H, d], written (zeros where seqlens[b] == 0).
 *   lse     : float32 [B, H], written (-inf where seqlens[b] == 0); may be NULL.
 *   workspace : at least fa_decode_workspace_size(B, H, Lmax, d) bytes,
 *             256-byte aligned, owned by the caller.
 * Returns FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE or
 * FA_ERR_CUDA.
 */
fa_status fa_decode(const void* q, const void* kcache, const void* vcache,
                    const int* seqlens, void* o, float* lse,
                    int B, int H, int Lmax, int d, float scale,
                    void* workspace, size_t ws_bytes, fa_stream_t stream);

/*
 * Grouped-query decode: kcache and vcache are [B, Hkv, Lmax, d] and query
 * head h reads cache head h / (H / Hkv).  The workspace is
 * fa_decode_workspace_size(B, H, Lmax, d).  Everything else as fa_decode.
 */
fa_status fa_decode_gqa(const void* q, const void* kcache, const void* vcache,
                        const int* seqlens, void* o, float* lse,
                        int B, int H, int Hkv, int Lmax, int d, float scale,
                        void* workspace, size_t ws_bytes, fa_stream_t stream);

/*
 * Decode over a paged KV cache.  The pages name PagedAttention without
 * describing it; this is the addressing it implies: the cache of every
 * sequence is a list of fixed-size pages drawn from one pool, so sequences
 * grow without reserving Lmax rows each.  The arithmetic is fa_decode's
 * ("DL101 chapter 9", section 1.1; split-KV merge of "Flash Attention:
 * principle & practice", section 2.1).
 *   kpages,
 *   vpages      : bf16 [num_pages, Hkv, page_size, d], read only; row r of
 *                 head h of pool page p holds the key / value of one position.
 *   block_table : int32 [B, pages_per_seq] in DEVICE memory: position j of
 *                 sequence b lives in row j % page_size of pool page
 *                 block_table[b][j / page_size].  Entries past a sequence's
 *                 last page are never read.  An entry outside
 *                 [0, num_pages) is never dereferenced: its positions count
 *                 as masked and FA_ERR_INVALID_ARG is recorded in the device
 *                 error word (read it with fa_get_device_error).
 *   seqlens     : int32 [B], device; clamped to [0, pages_per_seq * page_size].
 *   page_size   : a power of two from 1 to 65536.
 *   workspace   : fa_decode_workspace_size(B, H, pages_per_seq * page_size, d).
 * q, o, lse, scale and the grouping Hkv as fa_decode_gqa.  Returns
 * FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE or
 * FA_ERR_CUDA.
 */
fa_status fa_decode_paged(const void* q, const void* kpages, const void* vpages,
                          const int* block_table, const int* seqlens, void* o, float* lse,
                          int B, int H, int Hkv, int page_size, int pages_per_seq,
                          int num_pages, int d, float scale,
                          void* workspace, size_t ws_bytes, fa_stream_t stream);

/*
 * Size in bytes of the device array that fa_decode_static uses as scratch
 * (16 MiB, held by every device that loads the library until exit).
 */
#define FA_DECODE_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * fa_decode without a caller-provided workspace, for callers that cannot
 * call cudaMalloc (a plug-in whose host program owns nearly all device memory
 * through its own pool, or a latency-critical loop that must not trigger the
 * device-wide synchronisation an allocation can cause).  The pages have no
 * counterpart: this is an interface convenience, not part of the method.
 *   Arguments, layouts, ownership and results are those of fa_decode, minus
 *   workspace / ws_bytes.  The split-KV partials go to a library-owned device
 *   array of FA_DECODE_STATIC_SCRATCH_BYTES bytes; a problem whose
 *   fa_decode_workspace_size(B, H, Lmax, d) exceeds that returns
 *   FA_ERR_WORKSPACE before any launch.  Allocates nothing.
 *   The first call on a device looks up the array's device address (with
 *   that device current); make it before any stream capture.  All calls
 *   share the array: calls that overlap on the GPU race and must be
 *   serialised by the caller.
 * Returns FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE or
 * FA_ERR_CUDA.
 */
fa_status fa_decode_static(const void* q, const void* kcache, const void* vcache,
                           const int* seqlens, void* o, float* lse,
                           int B, int H, int Lmax, int d, float scale,
                           fa_stream_t stream);

/*
 * Measurement hook.  With non-NULL events, every later call records `start`
 * on its stream just before launching its dominant kernel and `stop` just
 * after it: the attention kernel of fa_fwd*, the main kernel of fa_bwd*
 * (not the D = rowsum(dO o O) preprocess or the dQ conversion), the split-KV
 * kernel of fa_decode* (not the combine).  cudaEventElapsedTime(start, stop)
 * then times that kernel alone.  The events are created and owned by the
 * caller; pass NULL, NULL to turn the hook off.  Process-wide and not
 * thread-safe.  Always returns FA_OK.
 */
fa_status fa_set_timing_events(fa_event_t start, fa_event_t stop);

/*
 * Work-distribution override, for tests and measurements that must exercise
 * one particular schedule.  It changes only how work is spread over the SMs,
 * never a result.  Process-wide (it applies to every later call on every
 * device and host thread) until changed again.
 *   fwd_schedule : FA_SCHEDULE_AUTO lets the library choose per call;
 *                  FA_SCHEDULE_GRID launches the forward with one CTA per
 *                  256-row query tile; FA_SCHEDULE_PERSISTENT launches about
 *                  one CTA per SM (at most a third of the tiles), each looping
 *                  over several tiles.
 *   bwd_order    : FA_SCHEDULE_AUTO; FA_SCHEDULE_GRID orders the backward's
 *                  CTAs head-major (a head's key tiles adjacent);
 *                  FA_SCHEDULE_PERSISTENT launches the longest causal key
 *                  tiles of every head first.
 * Returns FA_ERR_INVALID_ARG for any other value (nothing is changed), else
 * FA_OK.
 */
enum {
    FA_SCHEDULE_AUTO = 0,
    FA_SCHEDULE_GRID = 1,
    FA_SCHEDULE_PERSISTENT = 2
};
fa_status fa_set_schedule(int fwd_schedule, int bwd_order);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word.  Returns FA_OK, FA_ERR_TIMEOUT (a kernel gave up a bounded wait and
 * returned without finishing) or FA_ERR_CUDA (the synchronisation failed).
 */
fa_status fa_get_device_error(fa_stream_t stream);

/*
 * Self-check of the failure detection behind FA_ERR_TIMEOUT ("FlashAttention:
 * Fast and Memory-Efficient Exact Attention with IO-Awareness" fixes no
 * failure model; this is the library's own).  Launches one CTA that waits,
 * with the same bounded waits as the attention kernels (a single-thread wait
 * and a warp-collective one), on an mbarrier that nothing arrives on.  After
 * the wait limit (2 s) both give up: the device error word becomes
 * FA_ERR_TIMEOUT and 2 is added to *gave_up (a device int, 4-byte aligned,
 * owned by the caller), and the kernel returns; the context stays usable.
 * Returns FA_ERR_INVALID_ARG for a null or misaligned pointer,
 * FA_ERR_UNSUPPORTED off sm_100, FA_ERR_CUDA if the launch fails.
 */
fa_status fa_check_bounded_wait(int* gave_up, fa_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char* fa_status_string(fa_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */

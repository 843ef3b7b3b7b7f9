/*
 * fa_b200.h -- exact attention forward for B200 (sm_100a), C ABI.
 *
 * Computes, for every query row of every head,
 *
 *     O   = softmax(scale * Q K^T + bias + mask) V
 *     LSE = log( sum_j exp(scale * q.k_j + bias_j) )   (natural log, fp32)
 *
 * tile by tile with an online softmax, so the score matrix never reaches
 * device memory.  The operation and its arguments follow these passages of
 * the source pages:
 *
 *   - "FlashAttention-4" (H3 runtime), API: [batch, sequence, heads, head_dim]
 *     layout, matching fp16/bf16 Q/K/V, and an error instead of a silent
 *     change of kernel for anything unsupported.
 *   - "flashrt/fa4-cute-runtime", Functions: the forward returns (out, lse);
 *     forward_static writes into a caller-preallocated out; seqused_k is a
 *     device int32 tensor holding the valid K/V length of a padded buffer;
 *     pack_gqa packs the query heads that share one K/V head.
 *   - "mgoin/tml-fa4", argument contract: varlen q [total_q, Hq, D],
 *     k/v [total_k, Hkv, D], cu_seqlens int32 [B+1] whose last entry is the
 *     total; rel_bias [total_q, Hq, rel_extent] in q's order and dtype with
 *     rel_extent a multiple of 128; the distance d = i + (k_len - q_len) - j,
 *     score += rel_bias[cu_seqlens_q[b] + i, h, d] when 0 <= d < rel_extent;
 *     in causal mode d == 0 is the query's own key (keys with d < 0 masked).
 *   - "mgoin/tml-fa4" (split-KV combine) and "FlashAttention-4 backend for
 *     Blackwell #1235" (split over keys merged through the LSE): the
 *     split-KV entry point.
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers of the current CUDA device, owned by
 *     the caller.  The library allocates no device memory and never
 *     synchronises the stream: a call only enqueues work on `stream`
 *     (a cudaStream_t; NULL means the legacy default stream) and returns.
 *   - Element type `dt` applies to q, k, v, out and rel_bias alike.
 *   - head_dim D must be a multiple of 8 from 16 to 256 ("FlashAttention-4
 *     backend for Blackwell #1235" uses head dims 16 and 64 and gives FA4's
 *     range on SM100 in steps of 8; "flashrt/fa4-cute-runtime" the
 *     D48/D72/D128 family and D256); Hq must be a multiple of Hkv; query
 *     head h reads K/V head h / (Hq / Hkv).
 *   - q, k, v, out and rel_bias must be 16-byte aligned and contiguous in the
 *     documented layout.  cu_seqlens and seqused_k are device int32 arrays.
 *   - The library receives pointers and sizes only, so it cannot check that
 *     a buffer holds the elements its layout implies for the sizes passed
 *     (out and q: B*Sq*Hq*D, or total_q*Hq*D; lse: B*Hq*Sq, or Hq*total_q;
 *     rel_bias: B*Sq*Hq*rel_extent, or total_q*Hq*rel_extent; seqused_k: B;
 *     cu_seqlens: B+1).  A smaller buffer is read or written out of bounds
 *     on the device.  The Python binding checks these extents before every
 *     call.
 *   - softmax_scale <= 0 selects 1 / sqrt(D).
 *   - A query row with no admissible key gets O = 0 and LSE = -inf.
 *   - K/V rows that a call reads but masks (beyond seqused_k, or the padding
 *     of a ragged tile) must hold finite values.
 *   - Errors: invalid arguments return FA_ERR_INVALID or FA_ERR_UNSUPPORTED
 *     before anything is enqueued; a launch failure returns FA_ERR_CUDA.  No
 *     entry point ever falls back to another algorithm.  A message for the
 *     last failure of the calling thread is available from
 *     fa_last_error_message().
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID = 1,        /* malformed arguments (null, shape, alignment) */
  FA_ERR_UNSUPPORTED = 2,    /* well-formed but not served (e.g. D = 100)   */
  FA_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed         */
  FA_ERR_WORKSPACE = 4,      /* split-KV workspace missing or too small      */
  FA_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up waiting (see below)         */
  FA_ERR_DEVICE_INPUT = 6    /* a kernel found device-side input that breaks
                                the contract (cu_seqlens, seqused_k; below)  */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/*
 * Dense forward.
 *   q   [B, Sq, Hq, D]    k, v [B, Sk, Hkv, D]    out [B, Sq, Hq, D]
 *   lse [B, Hq, Sq] float32 (may be NULL when not wanted)
 *   causal: bottom-right aligned (key j admitted iff j <= i + k_len - Sq).
 *   seqused_k: NULL, or device int32 [B] with 0 <= seqused_k[b] <= Sk; batch
 *     entry b then uses keys [0, seqused_k[b]) of its padded K/V rows and
 *     k_len = seqused_k[b] in the causal and bias distance.  The kernel checks
 *     the bound on the device: an entry outside it is skipped (its rows of
 *     out and lse keep their contents) and fa_check_device_error afterwards
 *     returns FA_ERR_DEVICE_INPUT.
 *   rel_bias: NULL, or [B*Sq, Hq, rel_extent] in q's dtype (the dense form of
 *     the varlen layout, rows in q's flattened order), rel_extent % 128 == 0.
 */
fa_status fa_fwd(const void *q, const void *k, const void *v, void *out,
                 float *lse, int B, int Sq, int Sk, int Hq, int Hkv, int D,
                 fa_dtype dt, int causal, float softmax_scale,
                 const int *seqused_k, const void *rel_bias, int rel_extent,
                 void *stream);

/*
 * Variable-length forward ("mgoin/tml-fa4", argument contract).
 *   q [total_q, Hq, D]   k, v [total_k, Hkv, D]   out [total_q, Hq, D]
 *   lse [Hq, total_q] float32 (may be NULL)
 *   cu_seqlens_q, cu_seqlens_k: device int32 [B+1], nondecreasing, first 0,
 *     last total_q / total_k.
 *   max_seqlen_q: the largest q length (it sizes the launch).  max_seqlen_k
 *     is accepted for API parity.
 *   seqused_k: NULL or device int32 [B]; k_len_b = seqused_k[b] (at most the
 *     cu_seqlens_k length).
 *   These device arrays are checked where the kernel reads them: a sequence
 *     whose cu_seqlens entries leave [0, total] or decrease, whose q length
 *     exceeds max_seqlen_q, whose seqused_k entry is outside [0, its k
 *     length], or the last sequence when cu_seqlens does not end at the
 *     totals, is skipped: nothing is read or written for it (its rows of out
 *     and lse keep their contents), and fa_check_device_error afterwards
 *     returns FA_ERR_DEVICE_INPUT.  The other sequences are computed.
 *   rel_bias: NULL or [total_q, Hq, rel_extent], rel_extent % 128 == 0.
 */
fa_status fa_fwd_varlen(const void *q, const void *k, const void *v, void *out,
                        float *lse, const int *cu_seqlens_q,
                        const int *cu_seqlens_k, const int *seqused_k, int B,
                        int max_seqlen_q, int max_seqlen_k, int total_q,
                        int total_k, int Hq, int Hkv, int D, fa_dtype dt,
                        int causal, float softmax_scale, const void *rel_bias,
                        int rel_extent, void *stream);

/*
 * Split-KV forward (decode): keys are cut into num_splits contiguous ranges,
 * each range yields a float32 partial (O normalised over the range, and its
 * LSE) in `workspace`, and a second kernel merges them through the LSE:
 *     lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
 * Arguments as fa_fwd, plus:
 *   num_splits: 0 picks fa_splitkv_default_splits(); otherwise >= 1 (the
 *     effective count can be lower when the ranges, rounded to whole key
 *     tiles, cover Sk sooner).
 *   workspace: device memory of at least fa_splitkv_workspace_bytes(...)
 *     bytes, 16-byte aligned, owned by the caller; its contents on entry do
 *     not matter and are overwritten.
 * A seqused_k entry outside [0, Sk] is reported as in fa_fwd, but here the
 * rows of that batch entry in out and lse are unspecified (the merge reads
 * partials that no kernel wrote).
 */
size_t fa_splitkv_workspace_bytes(int B, int Sq, int Hq, int D, int num_splits);
int fa_splitkv_default_splits(int B, int Sq, int Sk, int Hq, int Hkv, int D,
                              int num_sms);
fa_status fa_fwd_splitkv(const void *q, const void *k, const void *v, void *out,
                         float *lse, int B, int Sq, int Sk, int Hq, int Hkv,
                         int D, fa_dtype dt, int causal, float softmax_scale,
                         const int *seqused_k, const void *rel_bias,
                         int rel_extent, int num_splits, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * Split-KV forward that allocates nothing: no workspace argument, and no
 * device allocation inside the library.  The pages have no counterpart to
 * this entry point; it exists for callers that cannot call cudaMalloc at all
 * and so cannot provide fa_fwd_splitkv's workspace: code that runs where the
 * device allocator belongs to someone else (a host framework's caching
 * allocator or a memory pool sized once at start-up, which the caller must
 * not bypass), or code under a rule of no allocation after initialisation
 * (fixed-latency serving loops, where a cudaMalloc can synchronise the device
 * and stall every stream).
 *
 * The split partials go to a scratch array inside the library of
 * FA_SPLITKV_STATIC_SCRATCH_BYTES bytes, which every GPU that loads the
 * library holds until the process exits.  Arguments are those of
 * fa_fwd_splitkv without the workspace; a problem whose partials
 * (fa_splitkv_workspace_bytes for the split count used) exceed the scratch is
 * rejected with FA_ERR_WORKSPACE before anything is enqueued.
 *
 * The first call on each device looks up the scratch's device address (with
 * that device current) and caches it; make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents; each call writes every partial it reads, so nothing has to start
 * at zero.  Calls whose kernels overlap on the GPU (different streams without
 * ordering between them, or several host threads) race on the array and give
 * wrong results: order them.
 */
#define FA_SPLITKV_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
fa_status fa_fwd_splitkv_static(const void *q, const void *k, const void *v,
                                void *out, float *lse, int B, int Sq, int Sk,
                                int Hq, int Hkv, int D, fa_dtype dt,
                                int causal, float softmax_scale,
                                const int *seqused_k, const void *rel_bias,
                                int rel_extent, int num_splits, void *stream);

/*
 * Score and mask modifiers ("mgoin/tml-fa4" lists mask/score modifiers among
 * the forward paths; the two below are the plain readings this library
 * serves).  With d = i + (k_len - q_len) - j the distance of key j from query
 * row i's diagonal (the distance of the causal and bias rules):
 *   window_left  >= 0: key j is masked when d > window_left (more than
 *                 window_left keys before the diagonal); < 0: no bound.
 *   window_right >= 0: key j is masked when -d > window_right (more than
 *                 window_right keys after the diagonal); < 0: no bound.
 *                 causal mode is window_right = 0 (a larger value is capped).
 *   softcap      >  0: the scaled score s becomes softcap * tanh(s / softcap)
 *                 before rel_bias is added; 0: off.  Must be finite, >= 0.
 * A row whose window holds no key gets O = 0 and LSE = -inf.  Keys outside
 * the window are neither loaded nor multiplied when they fill whole key
 * tiles.  FA_MODS_NONE initialises a struct with no modifier; a NULL pointer
 * means the same.
 */
typedef struct {
  int window_left;
  int window_right;
  float softcap;
} fa_mods;
#define FA_MODS_NONE {-1, -1, 0.0f}

/* fa_fwd, fa_fwd_varlen and fa_fwd_splitkv with modifiers (`mods` may be
 * NULL; it is read during the call only). */
fa_status fa_fwd_ex(const void *q, const void *k, const void *v, void *out,
                    float *lse, int B, int Sq, int Sk, int Hq, int Hkv, int D,
                    fa_dtype dt, int causal, float softmax_scale,
                    const int *seqused_k, const void *rel_bias, int rel_extent,
                    const fa_mods *mods, void *stream);
fa_status fa_fwd_varlen_ex(const void *q, const void *k, const void *v,
                           void *out, float *lse, const int *cu_seqlens_q,
                           const int *cu_seqlens_k, const int *seqused_k,
                           int B, int max_seqlen_q, int max_seqlen_k,
                           int total_q, int total_k, int Hq, int Hkv, int D,
                           fa_dtype dt, int causal, float softmax_scale,
                           const void *rel_bias, int rel_extent,
                           const fa_mods *mods, void *stream);
fa_status fa_fwd_splitkv_ex(const void *q, const void *k, const void *v,
                            void *out, float *lse, int B, int Sq, int Sk,
                            int Hq, int Hkv, int D, fa_dtype dt, int causal,
                            float softmax_scale, const int *seqused_k,
                            const void *rel_bias, int rel_extent,
                            int num_splits, void *workspace,
                            size_t workspace_bytes, const fa_mods *mods,
                            void *stream);

/*
 * Context-parallel attention over key shards ("FlashAttention-4 backend for
 * Blackwell #1235": the returned LSE lets a split over keys be merged outside
 * the kernel; "mgoin/tml-fa4": the split-KV combine).  Each GPU holds one
 * contiguous shard of every sequence's keys and values; the exact result is
 * the LSE-weighted merge of the shards' normalised partials.
 *
 * fa_fwd_shard_partial: the partial of the shard held in k/v [B, Sk, Hkv, D]
 * (dense layout; q [B, Sq, Hq, D] holds all query rows).  Masks and bias use
 * the rows' distances in the WHOLE sequence: k_after (device int32 [B], or
 * NULL for all zero) gives, per sequence, how many of its keys follow this
 * shard, so d = i + (k_len + k_after[b] - q_len) - j with j the key's index
 * within the shard and k_len = Sk (or seqused_k[b]).  Values are clamped to
 * [0, 2^30].  rel_bias, causal and mods are those of the whole problem.
 *   o_part   : device float [B*Sq*Hq][D], packed (token, head) rows, the
 *              normalised partial O of this shard (0 for a row with no key);
 *   lse_part : device float [B*Sq*Hq], its natural-log LSE (-inf, no key).
 *   num_splits, workspace, workspace_bytes: as fa_fwd_splitkv (the shard's
 *              keys are split again inside the GPU and merged into the one
 *              partial); with one split the workspace may be NULL.
 * A shard with Sk = 0 writes O = 0 and LSE = -inf for every row.
 *
 * fa_combine_partials: merges n_parts partials stacked as o_parts
 * [n_parts][B*Sq*Hq][D] and lse_parts [n_parts][B*Sq*Hq] (the shards in any
 * order) into out [B, Sq, Hq, D] of type dt and lse [B, Hq, Sq] (may be
 * NULL).  A row whose partials are all -inf gets O = 0 and LSE = -inf.
 * o_parts and out must be 16-byte aligned.
 */
fa_status fa_fwd_shard_partial(const void *q, const void *k, const void *v,
                               float *o_part, float *lse_part, int B, int Sq,
                               int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                               int causal, float softmax_scale,
                               const int *seqused_k, const int *k_after,
                               const void *rel_bias, int rel_extent,
                               const fa_mods *mods, int num_splits,
                               void *workspace, size_t workspace_bytes,
                               void *stream);
fa_status fa_combine_partials(const float *o_parts, const float *lse_parts,
                              int n_parts, int B, int Sq, int Hq, int D,
                              fa_dtype dt, void *out, float *lse, void *stream);

/*
 * Device-side error word.  Every wait inside the kernels is bounded; a kernel
 * that gives up records code 1 in a device word of the current device and
 * returns without trapping (later waits of any kernel then give up at once,
 * until the word is cleared).  A kernel that finds device-side input breaking
 * the contract (cu_seqlens, seqused_k: see fa_fwd_varlen) records code 2,
 * skips that sequence and computes the others.  This call synchronises the
 * current device, copies the word to *code (0 = none; the codes are bits and
 * may be OR-ed) and, if clear != 0, resets it.  Returns FA_OK,
 * FA_ERR_DEVICE_TIMEOUT when bit 1 was set, FA_ERR_DEVICE_INPUT when only
 * bit 2 was, or FA_ERR_CUDA.
 */
fa_status fa_check_device_error(int *code, int clear);

/*
 * Watchdog self-test: enqueues one thread that waits, bounded by timeout_ns
 * (1 ms to 1 s), on a barrier nothing ever completes.  The wait gives up and
 * records the timeout code in the watchdog word exactly as a stalled kernel
 * would, without trapping; the device stays usable.  A following
 * fa_check_device_error then returns FA_ERR_DEVICE_TIMEOUT (and clears the
 * word when asked).  Returns FA_OK once enqueued.
 */
fa_status fa_watchdog_selftest(unsigned long long timeout_ns, void *stream);

/*
 * Self-test of the softmax's FMA-pipe exponential: y[i] = 2^x[i] computed by
 * the polynomial routine that some of the softmax's exponentials take instead
 * of the MUFU unit (a degree-3 minimax polynomial on [-1/2, 1/2] scaled by an
 * exponent-field add; relative error below 8e-5 for -125 <= x <= 8, results
 * below 2^-125 are not accurate, and x < -126 gives 2^-126).  x and y are
 * device float arrays of n elements.  The pages have no counterpart: it
 * exists so that a test can measure this routine's error on the GPU.
 * Returns FA_OK once enqueued.
 */
fa_status fa_selftest_exp2_fma(const float *x, float *y, long long n, void *stream);

/* Human-readable name of a status; never NULL. */
const char *fa_status_string(fa_status s);

/* Message for the calling thread's last failed call ("" if none). */
const char *fa_last_error_message(void);

/* Library version string. */
const char *fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */

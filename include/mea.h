/*
 * mea.h -- C ABI of libmea: memory-efficient exact attention on B200 (sm_100a).
 *
 * The operation (FlashAttention (2022), sections "L'idea: non scrivere mai la
 * matrice intera" and "Il trucco della softmax che non ha bisogno di vedere
 * tutto"; xFormers tutorial "Come costruire Transformer efficienti in memoria
 * con xFormers ...", section "Impostare xFormers e Validare l'Attenzione
 * Memory-Efficient"):
 *
 *     out = softmax(Q K^T * scale + bias) V,   lse = ln sum_j exp(scale q.k_j + b_j)
 *
 * computed tile by tile with a running max / running sum, so the M x N score
 * matrix never reaches device memory.  The result is exact up to the rounding of
 * fp32 accumulation and of the fp16/bf16 output.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates nothing, keeps no pointer after the call returns and is safe to
 *    call from several host threads.
 *  - Calls are asynchronous on `stream` and never synchronise (except
 *    mea_read_device_status).  Argument errors are detected on the host and
 *    returned before anything is launched; nothing is thrown across the ABI.
 *  - Element types: MEA_F16 or MEA_BF16 for q/k/v/out; lse is fp32.
 *    Accumulation is fp32 throughout.
 *  - Head dimension K must be 64 or 128.  Base pointers must be 16-byte aligned
 *    and every stride a multiple of 8 elements (tensor-memory-accelerator
 *    copies require 16-byte aligned rows); otherwise MEA_ERR_UNSUPPORTED.
 *  - Contents of device-side index arrays (seqstart offsets) are trusted; a
 *    kernel that finds them inconsistent with the host-side sizes records
 *    MEA_ERR_INVALID_ARG in the device status word (see
 *    mea_read_device_status) instead of faulting.
 *  - Every device wait is bounded: a wait that exceeds about two seconds makes
 *    the kernel record MEA_ERR_DEVICE_TIMEOUT and return, never hang.
 */
#ifndef MEA_H_
#define MEA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MEA_F16 = 0, MEA_BF16 = 1 } mea_dtype_t;

/* The bias objects of the xFormers tutorial, as an enum: the masks are
 * generated inside the kernel, never stored ("Applicare Attenzione Causale con
 * Maschere Inferiori"; "Utilizzare Sequenze di Lunghezza Variabile"). */
typedef enum {
  MEA_BIAS_NONE = 0,             /* no mask                                  */
  MEA_BIAS_CAUSAL = 1,           /* LowerTriangularMask, bottom-right aligned */
  MEA_BIAS_BLOCKDIAG = 2,        /* BlockDiagonalMask over packed sequences   */
  MEA_BIAS_BLOCKDIAG_CAUSAL = 3  /* BlockDiagonalCausalMask                   */
} mea_bias_t;

typedef enum {
  MEA_OK = 0,
  MEA_ERR_INVALID_ARG = -1,   /* null pointer, bad size, inconsistent shapes     */
  MEA_ERR_UNSUPPORTED = -2,   /* valid but not implemented (K, alignment, dtype) */
  MEA_ERR_WORKSPACE = -3,     /* workspace missing or too small                  */
  MEA_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed               */
  MEA_ERR_DEVICE_TIMEOUT = -5 /* a bounded device wait ran out (device status)   */
} mea_status_t;

/*
 * mea_fwd -- prefill / training-forward attention.
 *
 * Layouts (element strides; the last dimension K is contiguous):
 *   q   [B, M, Hq,  K]  q_strides = {stride_b, stride_m, stride_h}
 *   k   [B, N, Hkv, K]  k_strides
 *   v   [B, N, Hkv, K]  v_strides
 *   out [B, M, Hq,  K]  o_strides  (written; same dtype as q)
 *   lse [B, Hq, M] fp32, contiguous, natural log; may be NULL.
 *
 * Heads: Hq % Hkv == 0; query head h reads key/value head h / (Hq / Hkv)
 * (grouped-query attention, tutorial section "Dimotrazione di Gruppo Query
 * Attention (GQA)"), without copying K/V.
 *
 * bias:
 *   NONE    every query sees every key.
 *   CAUSAL  query i sees key j iff j <= i + (N - M) (bottom-right alignment, the
 *           tril(diagonal=past_len) mask of "Transformer : comprendre
 *           l'entrainement et l'inference", section "Un cache KV simple").
 *   BLOCKDIAG / BLOCKDIAG_CAUSAL  packed variable-length batch: B must be 1 and
 *           seqstart_q / seqstart_k (DEVICE int32 arrays of num_seqs + 1
 *           non-decreasing offsets, first 0, last M resp. N) split the rows into
 *           sequences; a query sees only keys of its own sequence, and with
 *           _CAUSAL the bottom-right rule applies inside the sequence.
 *           seqstart_k may be NULL (then equal to seqstart_q, requires M == N).
 *           max_seqlen_q / max_seqlen_k are host-known upper bounds on the
 *           per-sequence lengths (they size the grid; no device sync is made).
 *           For NONE / CAUSAL pass NULL, NULL, 0, 0, 0.
 * alibi:  nonzero adds -slope_h * |pos_i - pos_j| after scaling, positions local
 *         to the sequence with pos_i = i + (N - M), slope_h = 2^(-8 (h+1) / Hq)
 *         computed in registers (tutorial section "Utilizzare SwiGLU e ALiBi").
 * scale:  multiplies q.k (pass 1/sqrt(K) for the usual attention); must be >= 0
 *         (a negative scale returns MEA_ERR_UNSUPPORTED: negate q instead).
 *
 * A query row that sees no key gets out = 0 and lse = -inf.
 * Launch: one CTA per (256 query rows, query head, batch or sequence); for
 * K = 64 fp16 without a mask or ALiBi one CTA per SM instead, each walking
 * several such units in turn (same results, bit for bit run to run).
 * Returns MEA_OK or an error status; never synchronises.
 */
int mea_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
            int B, int M, int N, int Hq, int Hkv, int K,
            const int64_t q_strides[3], const int64_t k_strides[3],
            const int64_t v_strides[3], const int64_t o_strides[3],
            mea_dtype_t dtype, mea_bias_t bias,
            const int32_t* seqstart_q, const int32_t* seqstart_k,
            int num_seqs, int max_seqlen_q, int max_seqlen_k,
            int alibi, float scale, cudaStream_t stream);

/*
 * mea_decode -- one decode step: a single new query per sequence against a
 * packed, ragged KV cache ("Transformer : comprendre l'entrainement et
 * l'inference", section "Pre-remplissage et decodage"; "Transformerを実装して
 * 少し理解した気になる会(その4)", section "KV Cache": only the last query row is
 * needed, against every cached key).
 *
 *   q        [B, Hq, K]       contiguous (a [B, 1, Hq, K] tensor)
 *   k_cache  [cache_rows, Hkv, K] contiguous; v_cache the same
 *   kv_seqstart  DEVICE int32 [B + 1]: sequence b owns cache rows
 *            kv_seqstart[b] .. kv_seqstart[b+1]-1 (its keys, oldest first,
 *            the new token's key/value already appended); kv_seqstart[B] <= cache_rows.
 *   out      [B, Hq, K]       written, same dtype as q
 *   lse      [B, Hq] fp32 natural log, may be NULL
 *   max_kv_len  host-known upper bound on every n_b (sizes the split grid).
 *
 * The query of sequence b sits at position n_b - 1 and sees all n_b keys
 * (with ALiBi: bias -slope_h * (n_b - 1 - j)).  An empty sequence gives out = 0,
 * lse = -inf.  The cache is split into fixed chunks processed in parallel; the
 * partial (max, sum, output) states are merged exactly by their log-sum-exp.
 *
 * Device-side errors: a sequence whose offsets are inconsistent (n_b < 0, a
 * negative start, rows past cache_rows, or n_b > max_kv_len rounded up to the
 * split size), or one whose bounded pipeline wait gave up, gets out = 0 and
 * lse = NaN for all its heads, and the device status word (mea_read_device_status)
 * records MEA_ERR_INVALID_ARG or MEA_ERR_DEVICE_TIMEOUT; the other sequences
 * are unaffected.  No result is ever assembled from another call's partials.
 *
 * workspace: DEVICE scratch of at least mea_decode_workspace_size(...) bytes,
 * 256-byte aligned, owned by the caller; its contents need no initialisation
 * and are garbage afterwards.  Calls that share a workspace must not overlap.
 */
size_t mea_decode_workspace_size(int B, int Hq, int Hkv, int K, int max_kv_len);

int mea_decode(const void* q, const void* k_cache, const void* v_cache,
               const int32_t* kv_seqstart, void* out, float* lse,
               int B, int Hq, int Hkv, int K, int cache_rows, int max_kv_len,
               mea_dtype_t dtype, int alibi, float scale,
               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * mea_decode_noalloc -- mea_decode without a caller-provided workspace.
 *
 * The pages have no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory at the point of the call.  Examples: a plugin
 * or plain C host program embedded in a runtime that owns all device memory
 * through its own pool and hands it no allocator, or a serving loop that must
 * not call cudaMalloc after start-up, because cudaMalloc can synchronise the
 * device and can fail once memory is exhausted.
 *
 * Arguments, layouts and results are those of mea_decode.  The split partials
 * go to a fixed 32 MiB device array inside this library instead of a workspace,
 * which bounds the problem size to
 *     mea_decode_workspace_size(B, Hq, Hkv, K, max_kv_len) <= 32 MiB
 * (e.g. B=64, Hq=32, K=128, max_kv_len=8192 needs 16.9 MB).  Larger problems
 * return MEA_ERR_WORKSPACE before anything is launched.  The call allocates
 * nothing: no cudaMalloc, no cudaFree and no allocating library routine.
 *
 * Notes for callers:
 *  - Every GPU that loads this library holds the 32 MiB array until the
 *    process exits.
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress, which allocates nothing); the first call on a
 *    device also loads the library's kernels there, so make it before any
 *    stream capture begins.
 *  - All calls on a device share the one array, which keeps the last call's
 *    contents.  Nothing in it has to start at zero: every partial a call reads,
 *    the same call has written first.  Calls whose executions overlap on the GPU
 *    (different streams, or different host threads) race on the array and give
 *    wrong results; serialise them.
 */
int mea_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* kv_seqstart, void* out, float* lse,
                       int B, int Hq, int Hkv, int K, int cache_rows, int max_kv_len,
                       mea_dtype_t dtype, int alibi, float scale, cudaStream_t stream);

/*
 * mea_fwd_block_sparse -- mea_fwd with whole blocks of the score matrix left
 * out ("FlashAttention (2022)", section "Cosa mostravano i numeri", which names
 * the block-sparse variant of the method): the scores of query rows
 * [128a, 128a + 128) against keys [128c, 128c + 128) of (batch b, query head h)
 * are dropped (bias -inf) when
 *     block_mask[b * mask_strides[0] + h * mask_strides[1] + a * ceil(N/128) + c] == 0,
 * on top of `bias` (MEA_BIAS_NONE or MEA_BIAS_CAUSAL; the block-diagonal kinds
 * return MEA_ERR_UNSUPPORTED).  Left-out blocks are neither loaded nor
 * multiplied.  The result is the dense definition with that mask, exact up to
 * the same rounding as mea_fwd; a row left with no visible key gets out = 0,
 * lse = -inf.
 *
 *   block_mask    DEVICE uint8, [B, Hq, ceil(M/128), ceil(N/128)] with the
 *                 last two dimensions contiguous; mask_strides (host, elements)
 *                 step b and h, 0 to share one mask across batches or heads.
 *   Other arguments as for mea_fwd.  Returns MEA_OK or an error status (a NULL
 *   mask or negative mask stride: MEA_ERR_INVALID_ARG); never synchronises.
 */
int mea_fwd_block_sparse(const void* q, const void* k, const void* v, void* out, float* lse,
                         int B, int M, int N, int Hq, int Hkv, int K,
                         const int64_t q_strides[3], const int64_t k_strides[3],
                         const int64_t v_strides[3], const int64_t o_strides[3],
                         mea_dtype_t dtype, mea_bias_t bias, const uint8_t* block_mask,
                         const int64_t mask_strides[2], int alibi, float scale,
                         cudaStream_t stream);

/* Rows and keys covered by one block-mask entry of mea_fwd_block_sparse (128). */
int mea_sparse_block_size(void);

/*
 * mea_prefill_chunk -- one chunk of prefill against a KV cache, with the cache
 * append fused into the attention launch ("Transformer : comprendre
 * l'entrainement et l'inference", sections "Pre-remplissage et decodage" and
 * "Un cache KV simple": the chunk's keys and values go after the cached ones,
 * and its queries attend to all of them under tril(diagonal=past_len)).
 * For sequence b with past = cache_seqlens[b] and n = q_seqlens[b] (M if
 * q_seqlens is NULL):
 *   1. k_cache[b, past + r] = k_new[b, r] and v_cache likewise, r < n;
 *   2. out[b, i], lse[b, :, i] for i < n: attention of q[b, i] (position
 *      past + i) over cache rows [0, past + n); causal: keys j <= past + i;
 *      ALiBi distance |past + i - j|; GQA as in mea_fwd.
 *
 *   q, out          [B, M, Hq, K]           element strides (b, m, h), K contiguous
 *   k_new, v_new    [B, M, Hkv, K]          the chunk's keys/values (rows >= n unused)
 *   k_cache, v_cache [B, cache_rows, Hkv, K] updated in place (rows [past, past+n))
 *   cache_seqlens   DEVICE int32 [B]        rows cached before the call (not updated:
 *                                           the caller adds n afterwards)
 *   q_seqlens       DEVICE int32 [B] or NULL real rows of each chunk (<= M)
 *   lse             [B, Hq, M] fp32 natural log, or NULL
 * Rows i >= n of out and lse are not written.  The launch reads cache rows
 * [0, past) only (the new rows come from k_new), so cache rows from past on may
 * hold anything; rows outside [past, past + n) are not written.  A sequence with past < 0, n
 * outside [0, M] or past + n > cache_rows is skipped and records
 * MEA_ERR_INVALID_ARG in the device status word.  cache_rows must be >= 1.
 * The caches must not overlap q, k_new, v_new or out.  Other conventions as
 * for mea_fwd (causal is 0 or 1).  Returns MEA_OK or an error status; never
 * synchronises.
 */
int mea_prefill_chunk(const void* q, const void* k_new, const void* v_new, void* k_cache,
                      void* v_cache, const int32_t* cache_seqlens, const int32_t* q_seqlens,
                      void* out, float* lse, int B, int M, int cache_rows, int Hq, int Hkv,
                      int K, const int64_t q_strides[3], const int64_t kn_strides[3],
                      const int64_t vn_strides[3], const int64_t kc_strides[3],
                      const int64_t vc_strides[3], const int64_t o_strides[3],
                      mea_dtype_t dtype, int causal, int alibi, float scale,
                      cudaStream_t stream);

/*
 * mea_bwd -- gradients of the attention of mea_fwd ("FlashAttention (2022)",
 * section "Il trucco della softmax che non ha bisogno di vedere tutto": the
 * backward pass recomputes the attention weights from q, k and the forward's
 * log-sum-exp instead of reading a stored score matrix).  With
 * p_ij = exp(scale q_i.k_j + b_ij - lse_i) and D_i = <dout_i, out_i>:
 *     dv_j = sum_i p_ij dout_i            dP_ij = <dout_i, v_j>
 *     dS_ij = p_ij (dP_ij - D_i)
 *     dq_i = scale sum_j dS_ij k_j        dk_j = scale sum_i dS_ij q_i
 * dk and dv of a key/value head sum over the Hq/Hkv query heads that read it.
 *
 *   q, out, dout, dq  [B, M, Hq, K]  contiguous, dtype `dtype`
 *   k, v, dk, dv      [B, N, Hkv, K] contiguous, dtype `dtype`
 *   lse               [B, Hq, M] fp32 natural log, as written by mea_fwd for the
 *                     same q, k, v, bias and scale (-inf for rows that see no key)
 *   bias, seqstart_q, seqstart_k, num_seqs, max_seqlen_k, alibi, scale: as for
 *   mea_fwd (max_seqlen_q is accepted for symmetry and unused).
 *
 * dq, dk, dv are written in full (rows that see no key, and keys no query sees,
 * get 0).  The outputs must not alias the inputs.
 *
 * workspace: DEVICE scratch of at least mea_bwd_workspace_size(B, M, Hq, K)
 * bytes, 256-byte aligned, owned by the caller, holding an fp32 dq accumulator
 * and D; it needs no initialisation and is garbage afterwards.  Calls that share
 * a workspace must not overlap.  Too small or misaligned: MEA_ERR_WORKSPACE.
 * Non-contiguous layouts are not accepted by this entry point (pass contiguous
 * copies); pointers not 16-byte aligned give MEA_ERR_UNSUPPORTED.
 * Returns MEA_OK or an error status; never synchronises.
 */
size_t mea_bwd_workspace_size(int B, int M, int Hq, int K);

int mea_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
            const float* lse, void* dq, void* dk, void* dv,
            int B, int M, int N, int Hq, int Hkv, int K,
            mea_dtype_t dtype, mea_bias_t bias,
            const int32_t* seqstart_q, const int32_t* seqstart_k,
            int num_seqs, int max_seqlen_q, int max_seqlen_k,
            int alibi, float scale, void* workspace, size_t workspace_bytes,
            cudaStream_t stream);

/*
 * mea_bwd_stages -- mea_bwd restricted to some of its three launches, in order:
 *   MEA_BWD_PREP (1)  D_i = <dout_i, out_i> and a zeroed fp32 dq accumulator,
 *                     both in the workspace;
 *   MEA_BWD_MAIN (2)  dk, dv and the dq accumulation (the score recomputation);
 *   MEA_BWD_DQ   (4)  the accumulator rounded into dq.
 * `stages` is a bitwise OR of these (nonzero, else MEA_ERR_INVALID_ARG); the
 * other arguments are those of mea_bwd.  Calling the three stages one by one on
 * one stream, with the same arguments and workspace, computes exactly what one
 * mea_bwd call computes; it lets a caller time or overlap the stages separately.
 * A stage reads the workspace its predecessor wrote, so a stage run alone is
 * meaningful only after its predecessors ran with the same workspace.
 */
enum { MEA_BWD_PREP = 1, MEA_BWD_MAIN = 2, MEA_BWD_DQ = 4 };

int mea_bwd_stages(const void* q, const void* k, const void* v, const void* out,
                   const void* dout, const float* lse, void* dq, void* dk, void* dv,
                   int B, int M, int N, int Hq, int Hkv, int K,
                   mea_dtype_t dtype, mea_bias_t bias,
                   const int32_t* seqstart_q, const int32_t* seqstart_k,
                   int num_seqs, int max_seqlen_q, int max_seqlen_k,
                   int alibi, float scale, void* workspace, size_t workspace_bytes,
                   int stages, cudaStream_t stream);

/* Number of key/value rows one decode split covers (the unit of parallelism). */
int mea_decode_chunk(void);

/* Text for a status code (static storage; never NULL). */
const char* mea_status_string(int status);

/*
 * Synchronises `stream`, then returns the first error a kernel recorded in the
 * current device's status word (MEA_OK if none) and, if `clear` is nonzero,
 * resets it to MEA_OK.  Returns MEA_ERR_CUDA if the synchronisation fails.
 */
int mea_read_device_status(cudaStream_t stream, int clear);

/*
 * mea_selftest_timeout -- exercises the failure path of the bounded waits.
 * Launches one CTA that waits, through the same bounded mbarrier wait the
 * kernels use, on a barrier nothing arrives on, and gives up after timeout_us
 * microseconds (1 .. 10^7, else MEA_ERR_INVALID_ARG).  Afterwards the device
 * status word holds MEA_ERR_DEVICE_TIMEOUT (see mea_read_device_status) and the
 * CUDA context stays usable: nothing faults, traps or hangs.
 */
int mea_selftest_timeout(int timeout_us, cudaStream_t stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int mea_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MEA_H_ */

/*
 * sala.h -- C ABI of the SALA hybrid-attention hot path (libsala, CUDA sm_100a).
 *
 * Four operations, after the MiniCPM-SALA pages:
 *   - Lightning linear attention, prefill and single-token decode
 *     (state recurrence S_t = S_{t-1} + k_t v_t^T of the summary page,
 *     "Prerequisites / Linear Attention"; QK-normalisation, GQA-to-MHA and the
 *     output gate of the tech-report mirror, section 02 (3); RoPE in the linear
 *     layers from section 02 (4), HyPE);
 *   - InfLLM-v2-style block selection and block-sparse softmax attention
 *     (tech-report mirror, section 02 (2): each query attends to a few selected
 *     key/value blocks, sparse at long length and dense at standard length,
 *     output gate; NoPE from section 02 (4); sliding window plus global anchors
 *     from the summary page, "Prerequisites / Sparse Attention").
 *
 * Conventions shared by every call
 * --------------------------------
 * Pointers.  Every tensor pointer is a DEVICE pointer on the current CUDA
 *   device, except where a comment says otherwise.  The caller owns all memory;
 *   the library never allocates, frees or synchronises (except
 *   sala_get_device_error), and every launch is asynchronous on `stream`
 *   (a cudaStream_t passed as void*; NULL = the legacy default stream).
 * Layout.  Activations are [B, T, H, D] with element strides {b, t, h} given
 *   in a sala_strides; the D stride is always 1.  Base pointers must be 16-byte
 *   aligned and every stride times the element size a multiple of 16 bytes.
 * Types.  SALA_BF16: bf16 activations, outputs written in bf16 (round to
 *   nearest even).  SALA_F32: fp32 activations and outputs.  Accumulation is
 *   fp32 everywhere; the Lightning state is always fp32.
 * Errors.  Argument checks run on the host before any launch and return
 *   SALA_ERR_INVALID_ARG / SALA_ERR_UNSUPPORTED without touching memory.  A
 *   failed launch returns SALA_ERR_CUDA.  Conditions only the device can see
 *   (a value outside the tensor-core operand range, a bounded wait that ran
 *   out) set a device error word that sala_get_device_error() reports.
 * Aliasing.  Outputs must not overlap inputs; `state` is read and written.
 */
#ifndef SALA_H
#define SALA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SALA_OK = 0,
    SALA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, stride or alignment */
    SALA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
    SALA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
    SALA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out */
    SALA_ERR_WORKSPACE = 5,    /* workspace missing or smaller than required */
    SALA_ERR_RANGE = 6,        /* a non-finite value reached a result on the device, or a
                                  decode position lies outside the cache */
    SALA_ERR_BOUNDS = 7        /* debug builds only (SALA_DEBUG): a device-side index
                                  check failed and its access was skipped */
} sala_status;

typedef enum { SALA_F32 = 0, SALA_BF16 = 1 } sala_dtype;

/* Element strides of a [B, T, H, D] activation (the D stride is 1). */
typedef struct {
    int64_t b, t, h;
} sala_strides;

/* Human-readable name of a status code (static string, never NULL). */
const char *sala_status_string(sala_status s);

/* Library version string, e.g. "sala-b200 0.1 (sm_100a)". */
const char *sala_version(void);

/*
 * Lightning attention prefill (chunked).
 *
 * For each (b, h) and t = 0..T-1, with p = pos0 + t:
 *   qh_t = RoPE_p(RMSNorm(q_t) * q_norm_w),  kh_t = RoPE_p(RMSNorm(k_t) * k_norm_w)
 *   S_t  = S_{t-1} + kh_t v_t^T                  (S_{-1} = initial state)
 *   o_t  = qh_t^T S_t                            (state inclusive of token t)
 *   y_t  = sigmoid(g_t) * o_t   (elementwise; y_t = o_t when g == NULL)
 * RMSNorm(x) = x / sqrt(mean(x^2) + eps) over D; RoPE is rotate-half: for
 * i < D/2 the pair (x_i, x_{i+D/2}) turns by p * rope_base^(-2i/D).
 * Chunked evaluation: O_c = (Q_c K_c^T masked s<=t) V_c + Q_c S_{c-1},
 * S_c = S_{c-1} + K_c^T V_c, on tensor cores for bf16 with D = 128.
 *
 *   q, k, v, g  [B,T,H,D] activations (g may be NULL: no gate)
 *   o           [B,T,H,D] output y
 *   state       [B,H,D,D] fp32, contiguous, S[b][h][i][j] (i key dim, j value
 *               dim).  In: the initial state (ignored when init_zero != 0).
 *               Out: the state after token T-1.
 *   q_norm_w, k_norm_w  [D] fp32 norm weights, or NULL for weight 1
 *   D           64 or 128;  T >= 0 (T = 0 only copies/zeroes the state)
 *   chunk       64 or 128 (tile length of the chunked evaluation)
 *   pos0        position of token 0 (RoPE), >= 0
 *   workspace   device scratch of at least sala_lightning_prefill_workspace()
 *               bytes (may be NULL when that returns 0); contents are scratch
 *               (per-segment states and each segment's largest |v|)
 *   dt          SALA_BF16 (D = 64 or 128) or SALA_F32 (D = 64 or 128)
 * Values: any finite bf16 v.  The tensor-core path multiplies v in fp16 after a
 *   power-of-two scale chosen per token segment from the segment's largest |v| (a
 *   segment whose values fp16 does not hold is recomputed with that scale), and
 *   undoes the scale in fp32.
 * Errors: INVALID_ARG (null q/k/v/o/state, bad sizes, strides or alignment),
 *         UNSUPPORTED (other D/chunk/dtype), WORKSPACE, CUDA.  Device: RANGE
 *         when an output or the state is not finite (a non-finite input).
 */
size_t sala_lightning_prefill_workspace(int B, int T, int H, int D, int chunk, sala_dtype dt);

sala_status sala_lightning_prefill(const void *q, const void *k, const void *v, const void *g,
                                   void *o, float *state, const float *q_norm_w,
                                   const float *k_norm_w, int B, int T, int H, int D,
                                   sala_strides sq, sala_strides sk, sala_strides sv,
                                   sala_strides sg, sala_strides so, int chunk, int64_t pos0,
                                   float rope_base, float eps, int init_zero, void *workspace,
                                   size_t workspace_bytes, sala_dtype dt, void *stream);

/*
 * Lightning attention decode: one new token per batch entry.
 *   qh = RoPE_p(RMSNorm(q) * q_norm_w), kh likewise, p = pos[b]
 *   S  <- S + kh v^T ;  o = qh^T S (updated state) ;  y = sigmoid(g) * o
 *
 *   q, k, v, g  [B,H,D] activations with strides {b, h} taken from the .b and
 *               .h fields of the sala_strides (.t unused); g may be NULL
 *   o           [B,H,D] output (strides `so`)
 *   state       [B,H,D,D] fp32 contiguous, updated in place
 *   pos         [B] int32 DEVICE array of positions (>= 0)
 *   dt          SALA_BF16 or SALA_F32;  D = 64 or 128
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
sala_status sala_lightning_decode(const void *q, const void *k, const void *v, const void *g,
                                  void *o, float *state, const float *q_norm_w,
                                  const float *k_norm_w, const int32_t *pos, int B, int H, int D,
                                  sala_strides sq, sala_strides sk, sala_strides sv,
                                  sala_strides sg, sala_strides so, float rope_base, float eps,
                                  sala_dtype dt, void *stream);

/*
 * Lightning state of a token segment, without outputs: the exchange step of a sequence
 * split across devices (each device holds a contiguous segment; the recurrence is a sum,
 * so a segment's start state is the initial state plus the contributions of the
 * segments before it).
 *   state = (init_zero ? 0 : state) + sum_t kh_t v_t^T over the T tokens,
 *   kh_t = RoPE_{pos0+t}(RMSNorm(k_t) * k_norm_w)  (as in sala_lightning_prefill)
 * Arguments, layouts, dtypes and limits as sala_lightning_prefill (k, v, state, k_norm_w,
 * the strides of k and v); the workspace is sala_lightning_prefill_workspace(B, T, H, D,
 * chunk) bytes.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
sala_status sala_lightning_state(const void *k, const void *v, float *state,
                                 const float *k_norm_w, int B, int T, int H, int D,
                                 sala_strides sk, sala_strides sv, int chunk, int64_t pos0,
                                 float rope_base, float eps, int init_zero, void *workspace,
                                 size_t workspace_bytes, sala_dtype dt, void *stream);

/*
 * Sum of `count` fp32 arrays: dst[e] = (accumulate ? dst[e] : 0) + sum_{i < count}
 * src[i * stride + e] for e < n (device pointers; stride >= n when count > 1).  Forms a
 * segment's start state from the gathered states of the segments before it.
 * Errors: INVALID_ARG, CUDA.
 */
sala_status sala_state_prefix_sum(const float *src, size_t n, int count, size_t stride,
                                  float *dst, int accumulate, void *stream);

/*
 * Block selection (InfLLM-v2 style, NoPE).
 * For each (b, kv head hk, query row t), c = floor(t / block):
 *   Kbar_j  = mean of the `block` keys of complete block j (fp32)
 *   score_j = (1/sqrt(D)) * sum_{h in group(hk)} q_{t,h} . Kbar_j,
 *             group(hk) = query heads hk*G .. hk*G+G-1, G = Hq / Hkv
 *   candidates: complete blocks n_init <= j <= c - n_local
 *   chosen: the top `topk` candidates (larger score first, ties -> smaller j),
 *   united with the init blocks {0..n_init-1} and the local window
 *   {c-n_local+1..c} (clipped to [0, c]); written sorted ascending and padded
 *   with -1 to n_sel = n_init + topk + n_local entries.
 * When every candidate fits the budget all causal blocks are chosen, which is
 * the dense fallback.  Scores are computed in fp32-equivalent precision (bf16
 * high/low operand splits on tensor cores, or fp32 for topk > 64); a decision
 * between two scores closer than about 1e-5 may differ from exact arithmetic.
 *
 *   q           [B,T,Hq,D], k [B,T,Hkv,D] (bf16)
 *   idx         [B,Hkv,T,n_sel] int32 output, contiguous
 *   ws          device scratch of >= sala_sparse_select_workspace(..., topk) bytes,
 *               caller-owned, free again when the call has run; block means only
 *               for topk <= 64 (T / 64 <= 65535), plus a score scratch of at most
 *               1 GiB otherwise
 *   block = 64, 1 <= topk <= 256, 0 <= n_init, 1 <= n_local, D = 64 or 128,
 *   Hq % Hkv == 0, Hq / Hkv <= 32.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
size_t sala_sparse_select_workspace(int B, int T, int Hq, int Hkv, int D, int block, int topk);

sala_status sala_sparse_select(const void *q, const void *k, int B, int T, int Hq, int Hkv,
                               int D, sala_strides sq, sala_strides sk, int block, int topk,
                               int n_init, int n_local, int32_t *idx, void *ws, size_t ws_bytes,
                               sala_dtype dt, void *stream);

/*
 * Block selection, per-head softmax-normalised variant.  The pages leave the
 * selection score open; this variant scores a candidate block by the attention
 * share each query head of the group would give its representative key:
 *   s_{h,j}  = (1/sqrt(D)) q_{t,h} . Kbar_j           (h in group(hk))
 *   p_{h,j}  = exp(s_{h,j}) / sum_{j'} exp(s_{h,j'})   (softmax over the row's
 *              candidates n_init <= j' <= c - n_local, complete blocks only)
 *   score_j  = sum_{h in group(hk)} p_{h,j}
 * Everything else (candidates, top `topk` with ties -> smaller j, init blocks,
 * local window, sorted, -1 padded) is as in sala_sparse_select.  Each head's p sums
 * to 1, so a row's scores sum to G; with G = 1 the choice equals sala_sparse_select's.
 * fp32-equivalent arithmetic (dot products on tensor cores from an exact three-part
 * bf16 split of the fp32 block means, fp32 exponentials of about 2^-22 relative error):
 * a decision between two scores closer than about 1e-5 of their size may differ from
 * exact arithmetic.
 *
 *   arguments, layouts and ownership as sala_sparse_select; ws of
 *   >= sala_sparse_select_head_softmax_workspace() bytes (block means with their three
 *   bf16 parts and a score scratch of at most 1 GiB); G = Hq / Hkv must be 1, 2, 4, 8,
 *   16 or 32.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
size_t sala_sparse_select_head_softmax_workspace(int B, int T, int Hq, int Hkv, int D,
                                                 int block);

sala_status sala_sparse_select_head_softmax(const void *q, const void *k, int B, int T, int Hq,
                                            int Hkv, int D, sala_strides sq, sala_strides sk,
                                            int block, int topk, int n_init, int n_local,
                                            int32_t *idx, void *ws, size_t ws_bytes,
                                            sala_dtype dt, void *stream);

/*
 * Block-sparse softmax attention (NoPE, causal).
 * For each (b, query head h, row t), hk = h / (Hq / Hkv):
 *   keys = union of blocks [j*block, (j+1)*block) over the entries j >= 0 of
 *          idx[b][hk][t][:], restricted to s <= t
 *   o    = sum_s softmax_s(scale * q_{t,h} . k_s) v_s ;  y = sigmoid(g) * o
 * An empty key set gives y = 0.  Entries of a row must be distinct; -1 entries
 * are skipped.  The GQA group of hk shares the row's selection.
 *
 *   q, g, o     [B,T,Hq,D] (g may be NULL), k, v [B,T,Hkv,D] (bf16)
 *   idx         [B,Hkv,T,n_sel] int32, contiguous, entries in [-1, ceil(T/block))
 *   scale       softmax scale; 0 selects 1/sqrt(D)
 *   ws          device scratch of >= sala_sparse_attn_workspace() bytes, 16-byte
 *               aligned, caller-owned; it receives an fp16 copy of v (the P.V
 *               tensor-core operand) times 2^-e, e a power-of-two exponent per
 *               (sequence, KV head) chosen from the largest |v| so that any finite
 *               bf16 v keeps its significant bits (the output is multiplied by
 *               2^e), and may be reused once the call has run
 *   block = 64, D = 64 or 128, 1 <= Hq / Hkv <= 16 (the GQA group fills one
 *   16-row tensor-core tile, padded with zero rows when smaller).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.  Device: RANGE when v holds
 *   an infinite or NaN value.
 */
size_t sala_sparse_attn_workspace(int B, int T, int Hkv, int D);

sala_status sala_sparse_attn(const void *q, const void *k, const void *v, const void *g,
                             const int32_t *idx, int n_sel, void *o, int B, int T, int Hq,
                             int Hkv, int D, sala_strides sq, sala_strides sk, sala_strides sv,
                             sala_strides sg, sala_strides so, int block, float scale,
                             void *ws, size_t ws_bytes, sala_dtype dt, void *stream);

/*
 * Block selection and block-sparse attention for a window of query rows: the
 * operations of sala_sparse_select / sala_sparse_select_head_softmax and
 * sala_sparse_attn (same definitions, MiniCPM-SALA tech-report mirror, section
 * 02 (2)) for the Tq query rows at positions qpos0 .. qpos0 + Tq - 1 of a sequence
 * whose keys and values cover positions 0 .. Tk - 1.  Row t of q, g, o and idx is
 * position qpos0 + t: its block c = floor((qpos0 + t) / block) sets its candidates,
 * local window and causal mask.  The result for each row equals that row of the
 * whole-sequence call (bit for bit when k and v are the whole sequence's, Tk = T:
 * the attention's per-(sequence, KV head) v scale is then the same), so a sequence
 * can be split over devices by query rows after gathering k and v on each.
 *
 *   q, g, o     [B,Tq,Hq,D] (g may be NULL), k, v [B,Tk,Hkv,D] (bf16), strided
 *   idx         [B,Hkv,Tq,n_sel] int32, contiguous (output of the selection, input
 *               of the attention)
 *   score       0: group-summed scores (sala_sparse_select), 1: per-head
 *               softmax-normalised scores (sala_sparse_select_head_softmax)
 *   ws          selection: >= sala_sparse_select_rows_workspace() bytes (block means
 *               of the Tk keys, plus the score scratch when score = 1 or topk > 64);
 *               attention: >= sala_sparse_attn_workspace(B, Tk, Hkv, D) bytes (the
 *               fp16 copy of the Tk values); caller-owned, reusable after the call
 *   0 <= qpos0, qpos0 + Tq <= Tk; every other limit as in the whole-sequence calls.
 * Errors: INVALID_ARG (also for a window outside [0, Tk)), UNSUPPORTED, WORKSPACE,
 *   CUDA.  Device (attention): RANGE when v holds an infinite or NaN value.
 */
size_t sala_sparse_select_rows_workspace(int B, int Tq, int Tk, int Hq, int Hkv, int D,
                                         int block, int topk, int score);

sala_status sala_sparse_select_rows(const void *q, const void *k, int B, int Tq, int qpos0,
                                    int Tk, int Hq, int Hkv, int D, sala_strides sq,
                                    sala_strides sk, int block, int topk, int n_init,
                                    int n_local, int score, int32_t *idx, void *ws,
                                    size_t ws_bytes, sala_dtype dt, void *stream);

sala_status sala_sparse_attn_rows(const void *q, const void *k, const void *v, const void *g,
                                  const int32_t *idx, int n_sel, void *o, int B, int Tq,
                                  int qpos0, int Tk, int Hq, int Hkv, int D, sala_strides sq,
                                  sala_strides sk, sala_strides sv, sala_strides sg,
                                  sala_strides so, int block, float scale, void *ws,
                                  size_t ws_bytes, sala_dtype dt, void *stream);

/*
 * Sparse-layer decode (InfLLM-v2 style, NoPE): one new query per sequence.
 * For sequence b at position p = pos[b], whose cache already holds the new token's key
 * and value at row p, the step computes row t = p of the prefill pair
 * sala_sparse_select + sala_sparse_attn over cache rows 0..p:
 *   c = p / block; candidates n_init <= j <= c - n_local scored against the block means
 *   kbar (score_j = sum_{h in group(hk)} q_h . kbar_j), the top `topk` (ties -> smaller
 *   j) plus the init blocks and the local window, sorted and -1 padded; then softmax
 *   attention of every query head of the group over those blocks' keys s <= p, gated.
 * Block means are a cache the caller keeps beside the KV cache: on entry kbar must hold
 * the means of the complete blocks 0..c-1 (sala_sparse_block_means fills them for a
 * prefilled cache); when p completes block c ((p + 1) % block == 0) the call writes
 * kbar[b][c] (summed in key order, bit-identical to sala_sparse_block_means).
 *
 *   q, g, o     [B,Hq,D] bf16 (strides .b, .h; .t unused), g may be NULL
 *   k_cache, v_cache  [B,Tmax,Hkv,D] bf16 (strides b, t, h); rows 0..pos[b] valid
 *   kbar        [B, Tmax/block, Hkv, D] fp32 contiguous, in/out as above
 *   pos         [B] int32 DEVICE array, 0 <= pos[b] < Tmax
 *   idx_out     [B,Hkv,n_init+topk+n_local] int32 (the selection), or NULL
 *   scale       softmax scale; 0 selects 1/sqrt(D)
 *   ws          device scratch of >= sala_sparse_decode_workspace() bytes, 16-byte
 *               aligned, caller-owned (scores, selection, split partials)
 *   block = 64, Tmax a multiple of 64, D = 64 or 128, 1 <= Hq / Hkv <= 16.
 * Values: any finite bf16 v (P.V runs as two bf16 products, P's high and low parts,
 *   on v as stored).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.  Device: RANGE when a pos[b] lies
 *   outside [0, Tmax) (that sequence is skipped) or an output is not finite (a
 *   non-finite input).
 */
size_t sala_sparse_decode_workspace(int B, int Tmax, int Hq, int Hkv, int D, int n_sel);

sala_status sala_sparse_decode(const void *q, const void *k_cache, const void *v_cache,
                               const void *g, float *kbar, const int32_t *pos, void *o,
                               int32_t *idx_out, int B, int Tmax, int Hq, int Hkv, int D,
                               sala_strides sq, sala_strides sk, sala_strides sv, sala_strides sg,
                               sala_strides so, int block, int topk, int n_init, int n_local,
                               float scale, void *ws, size_t ws_bytes, sala_dtype dt,
                               void *stream);

/*
 * Block means of the complete blocks of a filled cache, the kbar operand of
 * sala_sparse_decode: kbar[b][j][hk][:] = mean of keys j*64 .. j*64+63 for j < T / 64.
 *   k       [B,T,Hkv,D] bf16 (strides b, t, h)
 *   kbar    [B, kbar_blocks, Hkv, D] fp32 contiguous, kbar_blocks >= T / 64
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
sala_status sala_sparse_block_means(const void *k, int B, int T, int Hkv, int D, sala_strides sk,
                                    float *kbar, int kbar_blocks, sala_dtype dt, void *stream);

/*
 * Input projection of a Lightning layer with its operand preparation fused into the GEMM
 * epilogue (tech-report mirror, section 02 (3): QK-normalisation and an output gate in
 * the linear layers; section 02 (4): RoPE in the linear layers):
 *   [q | k | v | g] = x W^T;  qh = RoPE(RMSNorm(q) * q_norm_w), kh = RoPE(RMSNorm(k) *
 *   k_norm_w) at position pos0 + t;  v as projected;  gate = sigmoid(g) (fp16: a value
 *   in (0, 1)).
 * The weights are the caller's (the pages publish none; tests use seeded synthetic ones).
 *
 *   x        [B, T, hidden] bf16, rows packed: row r = b*T + t at x + r * x_row_stride
 *            (elements; x_row_stride >= hidden, rows 16-byte aligned)
 *   w        [4 H D, hidden] bf16 contiguous: rows h*D.. of section s (q, k, v, g) are
 *            head h's output features
 *   q_norm_w, k_norm_w  [D] fp32 or NULL (weight 1)
 *   qh, kh, gate  [B,T,H,D] fp16 outputs;  v  [B,T,H,D] bf16 output (strides sq..sg)
 *   D = 64 or 128, hidden a multiple of 64, H*D a multiple of 256; dt = SALA_BF16.
 * tcgen05 GEMM (128 x 256 tiles, fp32 accumulation in tensor memory); no workspace.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
sala_status sala_lightning_projection(const void *x, const void *w, const float *q_norm_w,
                                      const float *k_norm_w, void *qh, void *kh, void *v,
                                      void *gate, int B, int T, int hidden, int H, int D,
                                      int64_t x_row_stride, sala_strides sq, sala_strides sk,
                                      sala_strides sv, sala_strides sg, int64_t pos0,
                                      float rope_base, float eps, sala_dtype dt, void *stream);

/*
 * Lightning prefill on prepared operands, the outputs of sala_lightning_projection: the
 * recurrence of sala_lightning_prefill with q, k already normalised and rotated and the
 * gate already a multiplier,
 *   S_t = S_{t-1} + kh_t v_t^T,  y_t = gate_t * (qh_t^T S_t)   (gate NULL: no gate).
 *   qh, kh, gate  [B,T,H,D] fp16;  v, o  [B,T,H,D] bf16;  state as in
 *            sala_lightning_prefill (in/out, or zero-initialised with init_zero)
 *   D = 128, chunk = 128 (tensor-core path); workspace of
 *   sala_lightning_prefill_workspace(B, T, H, 128, 128, SALA_BF16) bytes.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.  Device: RANGE when an output or
 *   the state is not finite.
 */
sala_status sala_lightning_prefill_prepared(const void *qh, const void *kh, const void *v,
                                            const void *gate, void *o, float *state, int B, int T,
                                            int H, int D, sala_strides sq, sala_strides sk,
                                            sala_strides sv, sala_strides sg, sala_strides so,
                                            int chunk, int init_zero, void *workspace,
                                            size_t workspace_bytes, void *stream);

/*
 * Lightning prefill that allocates nothing (not part of the method: a library
 * convenience).  Some callers cannot hand the library a workspace:
 * code embedded in a host framework that owns all device memory and offers its
 * plugins no allocator, or a serving loop whose memory pool is frozen after
 * start-up and must not call cudaMalloc on the hot path.  This entry point takes
 * the same arguments as sala_lightning_prefill minus the workspace and keeps its
 * per-segment state scratch in a fixed array of 16 MiB + 64 KiB that lives in the
 * library's device image (every GPU that loads the library holds it until exit).
 *
 * Limits: the bf16 / head_dim 128 / chunk 128 path needs B*H <= 256 (one 64 KiB
 * state per segment, at least one segment per head); larger B*H returns
 * SALA_ERR_WORKSPACE before any launch.  With fewer segments than the regular
 * entry point it runs fewer CTAs, so it is slower for small B*H.  Other
 * dtype/head_dim/chunk combinations need no scratch and behave exactly like
 * sala_lightning_prefill.
 * Set-up: the first call on each device looks up the device address of the
 * scratch array.
 * Concurrency: every call on a device shares the one scratch array and leaves
 * its contents behind; calls that can overlap on the GPU (different streams,
 * or several threads) race on it and must be serialised by the caller.
 * Calls no cudaMalloc/cudaFree and no allocating library routine.
 */
sala_status sala_lightning_prefill_noalloc(const void *q, const void *k, const void *v,
                                           const void *g, void *o, float *state,
                                           const float *q_norm_w, const float *k_norm_w, int B,
                                           int T, int H, int D, sala_strides sq,
                                           sala_strides sk, sala_strides sv, sala_strides sg,
                                           sala_strides so, int chunk, int64_t pos0,
                                           float rope_base, float eps, int init_zero,
                                           sala_dtype dt, void *stream);

/*
 * Failure-path self-test (a library diagnostic, no counterpart on the pages): runs
 * the bounded mbarrier wait every kernel uses on a barrier that never completes,
 * with a budget of `cycles` SM clock cycles (1 .. 4e9), so the wait runs out, sets
 * SALA_ERR_TIMEOUT in the device error word and returns.  Nothing faults or hangs;
 * read the result with sala_get_device_error().
 * Errors: INVALID_ARG (cycles out of range), CUDA.
 */
sala_status sala_selftest_wait_timeout(long long cycles, void *stream);

/*
 * Synchronise `stream`, then read and clear the device error word of the
 * current device.  Returns SALA_OK, SALA_ERR_RANGE, SALA_ERR_TIMEOUT or (debug
 * builds) SALA_ERR_BOUNDS (the first condition raised since the last call), or
 * SALA_ERR_CUDA if the synchronisation itself failed.
 */
sala_status sala_get_device_error(void *stream);

/*
 * Device index checks.  The library built with SALA_DEBUG defined (libsala_debug.so;
 * the same kernels and arithmetic) checks, before the access, the indices that data
 * or arithmetic select: every block index an attention row reads (in [-1, key
 * blocks)), every per-row selection buffer slot and output position, every score
 * scratch slot and every decode block index.  A failed check skips its access and
 * raises SALA_ERR_BOUNDS in the device error word instead of faulting.
 * Returns the source line of the first failed check since the last call and clears it
 * (0: none) after synchronising the current device; -1 in the release library, which
 * compiles the checks out.  Errors: none (a failed synchronisation reads as 0).
 */
int sala_debug_bounds_line(void);

#ifdef __cplusplus
}
#endif

#endif /* SALA_H */

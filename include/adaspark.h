/*
 * adaspark.h -- C ABI of the AdaSpark layer hot path for NVIDIA B200 (sm_100a).
 *
 * The method (from "AdaSpark: Adaptive Sparsity for Efficient Long-Video
 * Understanding", papernotes.org note, sections 整体框架 and 关键设计 1-4, and the
 * paper's abstract / Figure 2 caption):
 *   - video tokens are split into 3D h x w x t cubes (key design 1);
 *   - AdaS-Attn: each query token scores the preceding cubes against their mean
 *     keys, P_i = softmax(q . kbar_j / sqrt(d_k)), keeps the Top-p set S_i and
 *     attends only to those cubes plus its own cube (key design 2);
 *   - AdaS-FFN: inside each cube the Top-p tokens by L2 norm go through the FFN;
 *     each skipped token is updated as y_k = x_k + mean_j FFN(x_j) over the
 *     cube's active tokens; text tokens always take the dense FFN (key design 3);
 *   - one threshold p drives both selections (key design 4).
 *
 * Conventions shared by every call:
 *   - Ownership: the caller allocates and frees every buffer, host and device.
 *     The library never allocates device memory; workspace sizes come from the
 *     *_workspace queries.
 *   - Execution: calls taking a `stream` (a cudaStream_t, NULL = legacy default
 *     stream) are asynchronous on it. Their return code covers host-side
 *     validation and launch errors only. Problems found on the device (a token
 *     layout that breaks the preconditions, a bounded wait that expired) set a
 *     status word in the workspace; the kernels
 *     then return early and adaspark_read_device_status() reports
 *     ADASPARK_EDEVICE.
 *   - Token layout: tokens are in cube-major order. The visual prefix holds
 *     cubes 0..C-1 contiguously (cube_ids nondecreasing 0..C-1, cube_offsets
 *     [C+1] with cube_offsets[0] = 0 and cube_offsets[C] = n_vis); the text
 *     suffix n_vis..n_tokens-1 has cube_id -1. Causality follows this order.
 *   - Calls are reentrant when they use distinct workspaces. No C++ exception
 *     crosses this interface.
 *   - Requires an sm_100 device; otherwise ADASPARK_EUNSUPPORTED.
 */
#ifndef ADASPARK_H
#define ADASPARK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
typedef enum {
  ADASPARK_OK = 0,
  ADASPARK_EINVAL = -1,        /* bad argument (host-side validation)          */
  ADASPARK_ECUDA = -2,         /* a CUDA runtime/driver call failed            */
  ADASPARK_EUNSUPPORTED = -3,  /* device is not sm_100, or a shape not handled */
  ADASPARK_EDEVICE = -4        /* a kernel flagged a problem (see status word) */
} adaspark_status;

/* Element types of the activations and weights. */
typedef enum { ADASPARK_BF16 = 0, ADASPARK_FP32 = 1 } adaspark_dtype;

/* Bits of the device status word (adaspark_read_device_status detail). */
#define ADASPARK_DEV_BAD_LAYOUT   0x1u  /* cube_ids / cube_offsets / text_mask inconsistent */
#define ADASPARK_DEV_TIMEOUT      0x2u  /* a bounded wait inside a kernel expired          */
#define ADASPARK_DEV_RANGE        0x4u  /* a value left the range the kernels represent   */
                                        /* exactly: AdaS-Attn: a row's largest cube score  */
                                        /* |q.kbar| * log2(e) / sqrt(d) reached 2^20 (the  */
                                        /* row then keeps only its own cube); AdaS-FFN: a  */
                                        /* SwiGLU activation or a W_down weight beyond the */
                                        /* fp16 range +-65504 (see adaspark_token_ffn)     */

/* Human-readable name of a return code. Never NULL. */
const char *adaspark_status_string(int status);

/* ------------------------------------------------------------------------ */
/* Key design 1: 3D spatio-temporal cube partition (host only).             */
/* ------------------------------------------------------------------------ */

/* Number of cubes of a T x H x W grid split into cube_h x cube_w x cube_t
 * windows (edge cubes truncated): ceil(T/cube_t)*ceil(H/cube_h)*ceil(W/cube_w).
 * Returns ADASPARK_EINVAL for a non-positive size or a NULL n_cubes. */
int adaspark_cube_count(int T, int H, int W, int cube_h, int cube_w, int cube_t,
                        int32_t *n_cubes);

/* Cube-major order of a video-token grid (key design 1).
 *   perm         [T*H*W]          out: perm[k] = raster index t*H*W + h*W + w of
 *                                      the k-th token in cube-major order
 *   cube_ids     [T*H*W + n_text] out: cube of each cube-major position; -1 for the
 *                                      n_text text tokens, which follow the video
 *   cube_offsets [n_cubes + 1]    out: first position of each cube, then T*H*W
 *   n_cubes                       out: number of cubes (size cube_offsets with
 *                                      adaspark_cube_count)
 * Cubes are enumerated time-major over the cube grid (t_b, h_b, w_b); tokens
 * inside a cube in (t, h, w) order; edge cubes are truncated. All arrays are
 * caller-allocated HOST memory. Runs on the host, once per video, outside the
 * per-layer path. Returns ADASPARK_EINVAL on a non-positive size, negative
 * n_text or NULL pointer. */
int adaspark_cube_partition(int T, int H, int W, int cube_h, int cube_w, int cube_t,
                            int n_text, int32_t *perm, int32_t *cube_ids,
                            int32_t *cube_offsets, int32_t *n_cubes);

/* ------------------------------------------------------------------------ */
/* Key design 2: AdaS-Attn.                                                 */
/* ------------------------------------------------------------------------ */

/* Counters written by adaspark_cube_attn (read with adaspark_attn_read_stats). */
typedef struct {
  uint64_t visual_rows;      /* (visual token, query head) rows that ran selection */
  uint64_t candidate_pairs;  /* sum over those rows of the preceding-cube count    */
  uint64_t selected_pairs;   /* sum over those rows of |S_i|                        */
  uint64_t overflow_rows;    /* rows whose Top-p cut needed extra score passes      */
  uint64_t tiles;            /* 128-row attention tiles executed (visual + text)    */
  uint64_t key_blocks;       /* executed (tile, key block) pairs                    */
  uint64_t key_block_keys;   /* keys covered by those blocks (for executed FLOPs)   */
  uint64_t near_margin_rows; /* Top-p rows whose cut lies within 1e-5 of flipping:  */
                             /* min(C_k* - p, p - C_k*-1, P_(k*) - P_(k*+1)) < 1e-5, */
                             /* from the fp32 masses (a row whose next score is     */
                             /* not known counts as near); 0 for Top-K             */
  uint64_t split_pairs;      /* (row, cube) pairs run in gathered tiles (split walk) */
  uint64_t gathered_blocks;  /* (gathered tile, key block) pairs they executed       */
  uint64_t reserved[6];
} adaspark_attn_stats;

/* Device workspace bytes needed by adaspark_cube_attn for these sizes
 * (0 when the sizes are invalid). For ADASPARK_BF16 this includes the region
 * of the split walk (adaspark_set_split_rows); the common layout alone, the
 * ADASPARK_FP32 figure for the same sizes, is also accepted and then runs the
 * single walk. The split walk's region holds up to 6 records per visual
 * (token, query head) row, each with a bf16 partial output of d elements:
 * about (12 d + 152) bytes per visual row, 3.1 GB for 65536 visual tokens, 28
 * query heads and d = 128. */
size_t adaspark_cube_attn_workspace(int n_tokens, int n_vis, int n_cubes, int hq, int hkv,
                                    int d, int dtype);

/* AdaS-Attn for one layer (key design 2 of the papernotes note; the abstract
 * scores relevance over the preceding cubes only).
 *
 * For a visual token t of cube i and query head h (KV head floor(h/(hq/hkv))):
 *   kbar_j = mean of K over cube j;  P = softmax_j<i(q . kbar_j / sqrt(d));
 *   S = Top-p(P, p): order by probability descending then cube index ascending,
 *       keep the smallest prefix whose cumulative mass reaches p (>= 1 cube;
 *       p = 1 keeps every preceding cube; the first cube has none);
 *   out[t,h] = softmax attention over the keys of the cubes in S and the keys of
 *       cube i at positions <= t, one softmax, scale 1/sqrt(d).
 * A text token attends densely and causally to every earlier token.
 *
 *   Q [n_tokens, hq, d], K/V [n_tokens, hkv, d]: device, row-major, element type
 *       `dtype` (BF16 or FP32), d = 64 or 128;
 *   cube_ids [n_tokens], cube_offsets [n_cubes + 1]: device int32 (layout above);
 *   n_vis = cube_offsets[n_cubes] (checked on the device);
 *   p in (0, 1]; hq % hkv == 0; every cube holds 1..256 tokens;
 *   out [n_tokens, hq, d]: device, element type `dtype`;
 *   workspace: device, >= adaspark_cube_attn_workspace(...) bytes, 256-byte aligned.
 * Errors: ADASPARK_EINVAL for NULL pointers, bad sizes, p outside (0, 1] or NaN,
 * hq % hkv != 0, unsupported d, a short or misaligned workspace; ADASPARK_ECUDA
 * for a failed launch. */
int adaspark_cube_attn(const void *Q, const void *K, const void *V, int dtype,
                       const int32_t *cube_ids, const int32_t *cube_offsets, int n_cubes,
                       int n_vis, int n_tokens, int hq, int hkv, int d, float p,
                       void *out, void *workspace, size_t workspace_bytes, void *stream);

/* AdaS-Attn with Top-K in place of Top-p: S = the k preceding cubes of largest
 * probability P (same order: probability descending, cube index ascending;
 * every preceding cube when there are at most k). This is the fixed-size
 * selection that the AdaSpark paper compares with Top-p in its ablation of
 * selection strategies (row "Top-K"); everything else, arguments, layout,
 * workspace and outputs, is as for adaspark_cube_attn, with k (>= 1) in place
 * of p. adaspark_attn_export_sets reads the sets of either call.
 * Errors: as adaspark_cube_attn, and ADASPARK_EINVAL for k < 1. */
int adaspark_cube_attn_topk(const void *Q, const void *K, const void *V, int dtype,
                            const int32_t *cube_ids, const int32_t *cube_offsets, int n_cubes,
                            int n_vis, int n_tokens, int hq, int hkv, int d, int k, void *out,
                            void *workspace, size_t workspace_bytes, void *stream);

/* AdaS-Attn with Uniform Sampling in place of Top-p: the other strategy of the
 * AdaSpark paper's selection-strategy ablation that does not look at the
 * content (row "Uniform Sampling"; the pages name it without defining it).
 * Read here as: a query of cube i takes k of its i preceding cubes at even
 * spacing from the first, cubes floor(m * i / k) for m = 0..k-1, and every
 * preceding cube when i <= k; every query head of every token of cube i has
 * the same set, and the own cube is attended causally as always. No cube mean
 * keys or scores are computed. Arguments, layout, workspace and outputs as for
 * adaspark_cube_attn with k (>= 1) in place of p; adaspark_attn_export_sets
 * reads its sets. Errors: as adaspark_cube_attn, and ADASPARK_EINVAL for
 * k < 1. */
int adaspark_cube_attn_uniform(const void *Q, const void *K, const void *V, int dtype,
                               const int32_t *cube_ids, const int32_t *cube_offsets, int n_cubes,
                               int n_vis, int n_tokens, int hq, int hkv, int d, int k, void *out,
                               void *workspace, size_t workspace_bytes, void *stream);

/* Device workspace bytes needed by adaspark_cube_attn_train (0 when the sizes
 * are invalid or dtype is not ADASPARK_BF16): adaspark_cube_attn_workspace
 * plus an fp32 copy of the output. */
size_t adaspark_cube_attn_train_workspace(int n_tokens, int n_vis, int n_cubes, int hq,
                                          int hkv, int d, int dtype);

/* adaspark_cube_attn for a step whose backward pass follows: the same sets and
 * output, and P goes to the PV product as a bf16 pair (hi + lo) so that the
 * workspace also keeps O in fp32 exact to about 2^-17 of each term; with it,
 * adaspark_cube_attn_backward takes D_r = dO_r . O_r directly instead of
 * summing it in an extra pass over the keys. Arguments as adaspark_cube_attn,
 * with workspace >= adaspark_cube_attn_train_workspace(...) bytes. Only
 * ADASPARK_BF16 (ADASPARK_FP32 returns ADASPARK_EUNSUPPORTED). */
int adaspark_cube_attn_train(const void *Q, const void *K, const void *V, int dtype,
                             const int32_t *cube_ids, const int32_t *cube_offsets, int n_cubes,
                             int n_vis, int n_tokens, int hq, int hkv, int d, float p, void *out,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Device workspace bytes needed by adaspark_cube_attn_backward (0 when the
 * sizes are invalid, dtype is not ADASPARK_BF16 or d is not 128). */
size_t adaspark_cube_attn_backward_workspace(int n_tokens, int n_vis, int n_cubes, int hq,
                                             int hkv, int d, int dtype);

/* Backward pass of AdaS-Attn for fine-tuning (the AdaSpark note adapts the
 * model with light fine-tuning), selection straight-through: the cube sets of
 * the forward call (adaspark_cube_attn or _topk) that filled `fwd_workspace`
 * are held fixed; the cube mean keys and the relevance softmax receive no
 * gradient. For row r (token, query head) with admitted keys A_r (selected
 * cubes, own cube causally; text rows: every earlier token), logits
 * z = q . k / sqrt(d), P = softmax over A_r, and the upstream dO:
 *   D_r = sum_j P_rj (dO_r . v_j)  (= dO_r . O_r),  dS_rj = P_rj (dO_r . v_j - D_r);
 *   dQ_r = sum_j dS_rj k_j / sqrt(d);
 *   dK_j = sum dS_rj q_r / sqrt(d), dV_j = sum P_rj dO_r over the rows of every
 *   query head of the KV group that admit key j.
 *
 *   Q, K, V, cube_ids, cube_offsets, sizes: exactly those of the forward call;
 *   dO [n_tokens, hq, d]: device bf16, the gradient of the forward's output;
 *   fwd_workspace: the forward call's workspace, untouched since (the backward
 *       reads its sets, mode and per-row log-sum-exp, and after
 *       adaspark_cube_attn_train its fp32 output; it does not modify it);
 *   dQ [n_tokens, hq, d], dK / dV [n_tokens, hkv, d]: device float32, written
 *       in full (not accumulated into);
 *   workspace: device, >= adaspark_cube_attn_backward_workspace(...) bytes,
 *       256-byte aligned (fwd_workspace too), 16-byte alignment for the arrays.
 * The products run in bf16 on the tensor cores with fp32 accumulation (P and
 * dS are rounded to bf16 as operands; the softmax is recomputed in fp32, and
 * D_r is summed from the same fp32 P and dP rather than taken from the bf16
 * output, so each row's dS sums to zero up to fp32 rounding).
 * Deterministic: no atomics. Only ADASPARK_BF16 with d = 128 (ADASPARK_FP32
 * and d = 64 return ADASPARK_EUNSUPPORTED); a forward call that reported a
 * device error makes this call report ADASPARK_EDEVICE. Other errors as for
 * adaspark_cube_attn. */
int adaspark_cube_attn_backward(const void *Q, const void *K, const void *V, const void *dO,
                                int dtype, const int32_t *cube_ids,
                                const int32_t *cube_offsets, int n_cubes, int n_vis,
                                int n_tokens, int hq, int hkv, int d,
                                const void *fwd_workspace, float *dQ, float *dK, float *dV,
                                void *workspace, size_t workspace_bytes, void *stream);

/* Expand the selection sets of the last adaspark_cube_attn call on `workspace`
 * into a dense bitmap: sel_bits [n_vis, hq, ceil(n_cubes/32)] uint32 in DEVICE
 * memory, bit j of row (t, h) set when cube j is in S for that row (the own cube
 * is not marked). Same sizes and cube_ids (device) as the call. Synchronizes
 * `stream` once to read the call's mode, then runs asynchronously. For parity
 * checks and analysis. */
int adaspark_attn_export_sets(const void *workspace, const int32_t *cube_ids, int n_cubes,
                              int n_vis, int n_tokens, int hq, int hkv, int d, int dtype,
                              uint32_t *sel_bits, void *stream);

/* Copy the counters of the last adaspark_cube_attn call to host memory.
 * Synchronizes `stream`. */
int adaspark_attn_read_stats(const void *workspace, adaspark_attn_stats *stats, void *stream);

/* Allocation-free AdaS-Attn. (The AdaSpark pages have no counterpart: this is
 * a calling convenience of this library.)
 *
 * For callers that cannot allocate device memory where they run the layer --
 * e.g. a plugin that its host framework gives only input and output buffers, a
 * serving loop that must not allocate (allocation may synchronize the device
 * or fragment a fixed budget), or a process whose device memory belongs to
 * another allocator. Same computation (as the single walk: the output of
 * adaspark_cube_attn with adaspark_set_split_rows(0), bit for bit), arguments
 * and errors as adaspark_cube_attn, without the workspace: the kernels use a
 * fixed array of
 * ADASPARK_NOALLOC_SCRATCH_BYTES that the library keeps in device memory on
 * every GPU where its device code is loaded, until the process exits.
 *   - Runs the single walk (no split walk). Returns ADASPARK_EINVAL when the
 *     sizes are invalid or when the single walk's workspace for them
 *     (adaspark_cube_attn_workspace with dtype ADASPARK_FP32, the common
 *     layout) exceeds ADASPARK_NOALLOC_SCRATCH_BYTES (check that first).
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture.
 *   - Calls no cudaMalloc / cudaFree and no allocating routine.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents: calls whose kernels may overlap on the GPU (different streams
 *     without ordering between them) race and give wrong results; serialize
 *     them. adaspark_attn_export_sets / adaspark_attn_read_stats cannot read
 *     this array (use adaspark_cube_attn for those).
 *   - The cached address belongs to the device context it was looked up in:
 *     after cudaDeviceReset() on a device, this entry point must not be called
 *     on that device again in the same process.
 *   - A device that is not sm_100 gives ADASPARK_EUNSUPPORTED before any
 *     lookup. */
#define ADASPARK_NOALLOC_SCRATCH_BYTES (32u << 20)
int adaspark_cube_attn_noalloc(const void *Q, const void *K, const void *V, int dtype,
                               const int32_t *cube_ids, const int32_t *cube_offsets,
                               int n_cubes, int n_vis, int n_tokens, int hq, int hkv, int d,
                               float p, void *out, void *stream);

/* ------------------------------------------------------------------------ */
/* Key design 3: AdaS-FFN with mean compensation.                           */
/* ------------------------------------------------------------------------ */

typedef struct {
  uint64_t active_visual;   /* visual tokens that went through the FFN      */
  uint64_t skipped_visual;  /* visual tokens updated by mean compensation   */
  uint64_t text_tokens;     /* text tokens (always dense)                   */
  uint64_t near_margin_cubes; /* cubes whose Top-p cut lies within 1e-5 of   */
                              /* flipping (the margin of adaspark_attn_stats, */
                              /* on the importance shares, fp32)              */
  uint64_t reserved[12];
} adaspark_ffn_stats;

/* Device workspace bytes needed by adaspark_token_ffn (0 when invalid). */
size_t adaspark_token_ffn_workspace(int n_tokens, int n_vis, int n_cubes, int D, int F,
                                    int dtype);

/* AdaS-FFN for one layer (key design 3 of the papernotes note; Figure 2 caption).
 *
 * Inside each cube c, importance w_u = ||x_u||_2 / sum_{v in c} ||x_v||_2; the
 * active set M_c = Top-p(w, p) (same rule as AdaS-Attn; a cube whose norms sum
 * to 0 keeps every token). With FFN(x) = W_down (silu(W_gate x) * (W_up x)):
 *   active visual or text token: y = x + FFN(x);
 *   skipped visual token k of cube c: y_k = x_k + (1/|M_c|) sum_{j in M_c} FFN(x_j).
 *
 *   x [n_tokens, D]: device, type `dtype`; W_gate, W_up [F, D]; W_down [D, F]:
 *       device, type `dtype`, row-major (nn.Linear [out, in] layout);
 *   cube_ids [n_tokens], cube_offsets [n_cubes + 1]: device int32;
 *   text_mask [n_tokens]: device uint8, must equal (cube_ids == -1);
 *   p in (0, 1]; D % 64 == 0 and F % 128 == 0 for BF16 (D, F multiples of 4 for FP32);
 *   y [n_tokens, D]: device float32 (the residual stream is kept in fp32);
 *   workspace: device, >= adaspark_token_ffn_workspace(...) bytes, 256-byte aligned.
 * Precision (BF16): the products accumulate in fp32; the SwiGLU activations
 * feed the down projection as fp16 (3 more mantissa bits than bf16) and W_down
 * is converted to fp16 for it (exact for |w| >= 2^-14, absolute error below
 * 2^-25 under that). An activation whose magnitude exceeds 65504 (stored
 * saturated) or a W_down weight beyond +-65504 sets ADASPARK_DEV_RANGE in the
 * status word (internal codes 0x65xx and 0x66xx of the detail): the output then
 * differs from the exact FFN and must not be used.
 * Errors as for adaspark_cube_attn. */
int adaspark_token_ffn(const void *x, const void *W_gate, const void *W_up, const void *W_down,
                       int dtype, const int32_t *cube_ids, const int32_t *cube_offsets,
                       const uint8_t *text_mask, int n_cubes, int n_vis, int n_tokens, int D,
                       int F, float p, float *y, void *workspace, size_t workspace_bytes,
                       void *stream);

/* Importance of a token inside its cube for AdaS-FFN (key design 3 only says
 * that importance comes from the L2 norm, followed by the Top-p rule). The linear share is the
 * reading adaspark_token_ffn takes; the other two are alternatives the text
 * does not exclude. All three rank a cube's tokens like their L2 norms. */
#define ADASPARK_IMPORTANCE_L2_SHARE   0  /* ||x_u|| / sum_v ||x_v||          */
#define ADASPARK_IMPORTANCE_L2SQ_SHARE 1  /* ||x_u||^2 / sum_v ||x_v||^2      */
#define ADASPARK_IMPORTANCE_SOFTMAX    2  /* softmax over the cube of ||x_u|| */

/* adaspark_token_ffn with the token importance chosen by `importance` (one of
 * ADASPARK_IMPORTANCE_*); everything else as for adaspark_token_ffn, whose
 * workspace query applies. A cube whose importance sums to 0 keeps every
 * token. Errors: as adaspark_token_ffn, and ADASPARK_EINVAL for an unknown
 * importance code. */
int adaspark_token_ffn_ex(const void *x, const void *W_gate, const void *W_up,
                          const void *W_down, int dtype, const int32_t *cube_ids,
                          const int32_t *cube_offsets, const uint8_t *text_mask, int n_cubes,
                          int n_vis, int n_tokens, int D, int F, float p, int importance,
                          float *y, void *workspace, size_t workspace_bytes, void *stream);

/* Device workspace bytes needed by adaspark_token_ffn_backward (0 when the
 * sizes are invalid or dtype is not ADASPARK_BF16). */
size_t adaspark_token_ffn_backward_workspace(int n_tokens, int n_vis, int n_cubes, int D, int F,
                                             int dtype);

/* Backward pass of AdaS-FFN for fine-tuning (the AdaSpark note adapts the model
 * with light fine-tuning), selection straight-through: the active sets of the
 * forward call that filled `fwd_workspace` are held fixed, the token norms get
 * no gradient. For the forward of key design 3 and the upstream dy:
 *   skipped visual token k of cube c:  dx_k = dy_k;
 *   active token a of cube c:          df_a = dy_a + (sum of dy_k over the
 *                                      cube's skipped tokens) / |M_c|;
 *   text token:                        df = dy;
 *   computed rows (active and text), with g = W_gate x, u = W_up x:
 *     dh = W_down^T df, du = dh * silu(g), dg = dh * u * silu'(g),
 *     dx = dy + W_gate^T dg + W_up^T du;
 *   dW_gate = sum dg x^T, dW_up = sum du x^T, dW_down = sum df h^T over the
 *   computed rows, h = silu(g) * u.
 *
 *   W_gate, W_up [F, D], W_down [D, F]: device bf16, the forward's weights;
 *   cube_offsets [n_cubes + 1]: device int32, the forward's;
 *   dy [n_tokens, D]: device float32 (the gradient of the forward's y);
 *   fwd_workspace: the workspace of an adaspark_token_ffn / _ex call with the
 *       same sizes, weights and x, left untouched since (the backward reads its
 *       active set, compaction and gathered rows; it does not modify it);
 *   dx [n_tokens, D], dW_gate / dW_up [F, D], dW_down [D, F]: device float32,
 *       written in full (not accumulated into);
 *   workspace: device, >= adaspark_token_ffn_backward_workspace(...) bytes,
 *       256-byte aligned; also 256-byte alignment for fwd_workspace, 16 bytes
 *       for every array.
 * Contractions run in bf16 on the tensor cores with fp32 accumulation (df, dg,
 * du and h are rounded to bf16 as operands). Only ADASPARK_BF16:
 * ADASPARK_FP32 returns ADASPARK_EUNSUPPORTED. A forward call that reported a
 * device error makes this call report ADASPARK_EDEVICE (read with
 * adaspark_read_device_status on `workspace`). Other errors as for
 * adaspark_token_ffn. */
int adaspark_token_ffn_backward(const void *W_gate, const void *W_up, const void *W_down,
                                int dtype, const int32_t *cube_offsets, int n_cubes, int n_vis,
                                int n_tokens, int D, int F, const float *dy,
                                const void *fwd_workspace, float *dx, float *dW_gate,
                                float *dW_up, float *dW_down, void *workspace,
                                size_t workspace_bytes, void *stream);

/* Copy the active flags of the last adaspark_token_ffn call on `workspace` into
 * active [n_tokens] uint8 DEVICE memory (1 = through the FFN). Asynchronous. */
int adaspark_ffn_export_active(const void *workspace, int n_tokens, int n_vis, int n_cubes,
                               int D, int F, int dtype, uint8_t *active, void *stream);

/* Copy the counters of the last adaspark_token_ffn call to host memory.
 * Synchronizes `stream`. */
int adaspark_ffn_read_stats(const void *workspace, adaspark_ffn_stats *stats, void *stream);

/* ------------------------------------------------------------------------ */
/* Status, timing and launch accounting.                                    */
/* ------------------------------------------------------------------------ */

/* ------------------------------------------------------------------------ */
/* A whole layer around the two calls (beyond the pages' problem statement:  */
/* the pages describe where AdaS-Attn and AdaS-FFN sit in a decoder layer,   */
/* not its projections), and RMSNorm.                                        */
/* ------------------------------------------------------------------------ */

/* Device workspace bytes for adaspark_layer (0 when the sizes are invalid or
 * dtype is not ADASPARK_BF16). */
size_t adaspark_layer_workspace(int n_tokens, int n_vis, int n_cubes, int hq, int hkv, int d,
                                int D, int F, int dtype);

/* One AdaSpark layer, wired as the stacked configuration uses it:
 *   Q = x W_q^T, K = x W_k^T, V = x W_v^T   (bf16, fp32 accumulation)
 *   a = AdaS-Attn(Q, K, V) with p_attn      (as adaspark_cube_attn)
 *   h = x + a W_o^T                         (bf16, fp32 accumulation)
 *   y = AdaS-FFN(h) with p_ffn              (as adaspark_token_ffn; y fp32)
 * The projections run on the library's tensor-core GEMM.
 *   x [n_tokens, D] bf16; W_q [hq*d, D], W_k/W_v [hkv*d, D], W_o [D, hq*d],
 *   W_gate/W_up [F, D], W_down [D, F]: bf16, row-major (output rows first);
 *   layout arguments and p as for the two calls; y [n_tokens, D] fp32;
 *   workspace: device, >= adaspark_layer_workspace(...) bytes, 256-byte aligned;
 *   it also holds Q, K, V, a and h (see adaspark_layer_buffers).
 * Requires d = 64 or 128 and D a multiple of 64. ADASPARK_EUNSUPPORTED for FP32,
 * ADASPARK_EINVAL for bad arguments; device-detected problems of any stage are
 * reported by adaspark_read_device_status on the layer workspace. */
int adaspark_layer(const void *x, const void *W_q, const void *W_k, const void *W_v,
                   const void *W_o, const void *W_gate, const void *W_up, const void *W_down,
                   int dtype, const int32_t *cube_ids, const int32_t *cube_offsets,
                   const uint8_t *text_mask, int n_cubes, int n_vis, int n_tokens, int hq,
                   int hkv, int d, int D, int F, float p_attn, float p_ffn, float *y,
                   void *workspace, size_t workspace_bytes, void *stream);

/* Byte offsets inside an adaspark_layer workspace of the layer's intermediate
 * tensors after a call: offsets[0..6] = Q, K, V, a (attention output), h, the
 * AdaS-Attn workspace and the AdaS-FFN workspace (for their export and stats
 * calls). `offsets` is host memory of 7 entries. */
int adaspark_layer_buffers(int n_tokens, int n_vis, int n_cubes, int hq, int hkv, int d, int D,
                           int F, int dtype, size_t *offsets);

/* RMSNorm: out[r] = x[r] / sqrt(mean_j x[r, j]^2 + eps) * weight (weight may be
 * NULL: no scaling), for the normalization between stacked layers.
 *   x [n_rows, D] device, element type x_dtype (BF16 or FP32); weight [D] bf16
 *   device or NULL; out [n_rows, D] bf16 device. Asynchronous on `stream`.
 * Errors: ADASPARK_EINVAL for NULL x/out, negative sizes, eps < 0 or NaN, an
 * unknown dtype. */
int adaspark_rmsnorm(const void *x, int x_dtype, const void *weight, void *out, int n_rows, int D,
                     float eps, void *stream);

/* Synchronize `stream` and read the status word of a workspace of either call.
 * Returns ADASPARK_OK, or ADASPARK_EDEVICE with *detail (if not NULL) holding the
 * ADASPARK_DEV_* bits in bits 0-7 and an internal code of the first failing
 * check in bits 8-23. The word is cleared by the next call on the workspace. */
int adaspark_read_device_status(const void *workspace, uint32_t *detail, void *stream);

/* Test hook for the bounded waits inside the kernels (not for production use;
 * the AdaSpark pages have no counterpart). Every wait on another warp or on the
 * tensor core is bounded; when a bound runs out the kernel records
 * ADASPARK_DEV_TIMEOUT, lets its issued copies and products finish, frees its
 * tensor memory and returns, and the device stays usable. With on != 0, every
 * later bf16 adaspark_cube_attn / _topk / _train launch of this process runs
 * its attention kernel with waits bounded by wait_cycles SM cycles (1e5 ..
 * 2e9) and withholds the announcement of each tile's first key block, so those
 * waits run out: the call then reports ADASPARK_EDEVICE with
 * ADASPARK_DEV_TIMEOUT. on == 0 restores the normal bound (about 2e9 cycles)
 * and behaviour. Process-wide, not thread-safe; ADASPARK_EINVAL for a bound
 * outside the range. */
int adaspark_debug_wait_expiry(int on, long long wait_cycles);

/* Split walk of the bf16 forward (adaspark_cube_attn and adaspark_cube_attn_topk;
 * not the training-mode call, Uniform Sampling, p = 1, or the allocation-free
 * entry point). A visual attention tile (128 consecutive visual tokens of one
 * query head) walks the key blocks of every cube any of its rows selected. A
 * selected cube that at most `rows` of the tile's rows chose, and that is no
 * row's own cube, leaves the tile's walk: its (row, cube) pairs are regrouped
 * by (KV head, cube) into gathered 128-row tiles, run over that cube's keys
 * alone, and each row merges their normalised partial outputs (bf16) by their
 * log2-sum-exps at the end of its own walk. The sets and the softmax are
 * those of the single walk; only the rounding of the merged parts differs.
 * Needs the workspace adaspark_cube_attn_workspace returns for BF16 (a smaller
 * workspace that still holds the common layout runs the single walk); a tile
 * whose records would pass the workspace's record capacity (6 per visual row)
 * keeps its whole walk. rows = 0 turns it off; default 8. Process-wide, not
 * thread-safe; ADASPARK_EINVAL for rows outside [0, 128]. */
int adaspark_set_split_rows(int rows);

/* Per-kernel timing with CUDA events recorded on the launching stream around
 * each launch of this library. Off by default; process-wide; not thread-safe. */
typedef struct {
  char name[48];     /* kernel name                      */
  uint64_t launches; /* timed launches since the last read */
  double total_ms;   /* summed event-to-event time        */
} adaspark_kernel_time;

int adaspark_timer_enable(int on);
/* Synchronize the recorded events, fill up to `max` entries and reset. */
int adaspark_timer_read(adaspark_kernel_time *out, int max, int *n_out);

/* Number of kernels this library has launched since it was loaded. */
uint64_t adaspark_launch_count(void);

/* ADASPARK_OK when `device` is an sm_100 GPU, else ADASPARK_EUNSUPPORTED
 * (ADASPARK_ECUDA if the query fails). */
int adaspark_device_check(int device);

#ifdef __cplusplus
}
#endif

#endif /* ADASPARK_H */

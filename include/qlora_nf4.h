/*
 * qlora_nf4.h -- C ABI of libqlora_nf4.so: a LoRA-adapted linear layer over a frozen NF4
 * (4-bit NormalFloat) base weight, forward and hand-derived backward, for sm_100a (B200).
 *
 * The operation ("Unsloth vs QLoRA vs Liger-Kernel", section 1, LoRA forward formula; FAQ
 * "What is the difference between LoRA and QLoRA?", NF4 base weights):
 *
 *     XA = X A^T                                   [M, r]
 *     h  = X deq(W0)^T + s XA B^T,   s = alpha / r [M, N]
 *
 * and its exact gradients for dY = dL/dh with W0 frozen ("Unsloth vs QLoRA vs
 * Liger-Kernel", section 2, hand-derived backward; "FTDD-03" teaching script, [SLIDE 3]):
 *
 *     dYB = dY B,  dX = dY deq(W0) + s dYB A,  dB = s dY^T XA,  dA = s dYB^T X.
 *
 * Shapes and layouts (all row-major, C order):
 *   X  [M, K] bf16   tokens x in-features          W0 [N, K] (nn.Linear weight [out, in])
 *   A  [r, K] bf16   LoRA down-projection          B  [N, r] bf16  LoRA up-projection
 *   h, dY [M, N] bf16                              dX [M, K] bf16
 *   dA [r, K] fp32, dB [N, r] fp32 (overwritten, not accumulated)
 *
 * NF4 storage (the readings the pages leave open are fixed here):
 *   q       [N, K/2] uint8  two 4-bit codes per byte, element 2j of a row in the HIGH nibble
 *   absmax  [N, K/64] fp32  per 64-element block of a row (block index n*K/64 + kb)
 *   double-quantised variant: absmax_q8 [N*K/64] uint8 and absmax_scale [ceil(N*K/64/256)]
 *   fp32, effective absmax = fp32(q8 * scale[block/256]).
 *   Codebook: the 16 NormalFloat levels (asymmetric N(0,1) quantiles with an exact zero,
 *   normalised to [-1, 1]) in fp32; code c dequantises to bf16(fp32(level[c] * absmax)).
 *
 * Beyond the single layer: several adapters sharing X packed into one layer
 * (qlora_grouped_*), the layer without a saved X A^T (XA_saved = NULL: recomputed), the
 * SwiGLU glue (flat or on a packed gate/up output) and the LM head + cross-entropy over a
 * frozen NF4 head, chunked over tokens (qlora_lm_head_ce).
 *
 * Conventions for every entry point:
 *   - Pointers named as device memory are caller-owned device allocations on the current
 *     device; the library allocates nothing and keeps no state between calls.
 *   - Device pointers must be 16-byte aligned (QLORA_ERR_ALIGN otherwise).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and the call
 *     returns without synchronising.  Launch failures are returned as QLORA_ERR_CUDA; a fault
 *     during execution surfaces at the caller's next synchronisation.
 *   - Shape errors are reported before any work is enqueued (QLORA_ERR_SHAPE).
 *   - Kernels bound every wait on another warp's progress; a wait that runs out sets the
 *     device error word read by qlora_device_error() and the kernel returns early.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_NULL = 1,      /* a required pointer is NULL */
  QLORA_ERR_SHAPE = 2,     /* M < 1, N or K not a multiple of 64, r out of range: [1, 128] for
                              qlora_linear_*, multiples of 8 in [8, 128] for the other calls */
  QLORA_ERR_ALIGN = 3,     /* a device pointer is not 16-byte aligned */
  QLORA_ERR_ARCH = 4,      /* current device is not compute capability 10.0 (sm_100a) */
  QLORA_ERR_WORKSPACE = 5, /* workspace NULL or smaller than qlora_workspace_bytes() */
  QLORA_ERR_CUDA = 6,      /* a CUDA runtime/driver call or kernel launch failed */
  QLORA_ERR_TIMEOUT = 7    /* a kernel's bounded wait ran out (see qlora_device_error) */
} qlora_status;

typedef void* qlora_stream_t; /* a cudaStream_t */

/* A packed NF4 weight: caller-owned device memory.  With double_quant == 0, `absmax` is
 * used and absmax_q8 / absmax_scale are ignored; with double_quant != 0 the reverse. */
typedef struct {
  const uint8_t* q;            /* [N, K/2] */
  const float* absmax;         /* [N*K/64] or NULL when double_quant */
  const uint8_t* absmax_q8;    /* [N*K/64] when double_quant */
  const float* absmax_scale;   /* [ceil(N*K/64/256)] when double_quant */
  int N;
  int K;
  int double_quant;
} qlora_nf4_weight;

/* Human-readable name of a status code (static string, never NULL). */
QLORA_API const char* qlora_status_str(qlora_status s);

/* Host-only: the fp32 NF4 codebook (16 ascending levels, out[0] = -1, out[7] = 0,
 * out[15] = +1), derived at library load from the NormalFloat construction.  Needs no GPU. */
QLORA_API qlora_status qlora_nf4_codebook(float out[16]);

/* NF4 quantise + pack ("Unsloth vs QLoRA vs Liger-Kernel", FAQ on LoRA vs QLoRA: base
 * weights in 4-bit NormalFloat; "Speed up fine-tuning 2x", internals item 1).
 *   W       [N, K] bf16 device, read only.
 *   q       [N, K/2] uint8 device, written.
 *   absmax  [N*K/64] fp32 device, written: first-level absmax (also when double_quant).
 *   absmax_q8 [N*K/64] uint8 and absmax_scale [ceil(N*K/64/256)] fp32 device, written only
 *           when double_quant != 0 (may be NULL otherwise).
 * Codes are chosen with the effective absmax (the double-quantised one when requested):
 * x = fp32(w / absmax), code = number of codebook midpoints strictly below x; a block
 * whose effective absmax is 0 gets code 7 (the exact zero) everywhere. */
QLORA_API qlora_status qlora_nf4_pack(const void* W, int N, int K, int double_quant, uint8_t* q,
                            float* absmax, uint8_t* absmax_q8, float* absmax_scale,
                            qlora_stream_t stream);

/* Dequantise a packed weight to bf16 Wd [N, K] device (diagnostic/test export; the linear
 * entry points never materialise it).  Uses the same device routine as the GEMM mainloop. */
QLORA_API qlora_status qlora_nf4_dequant(const qlora_nf4_weight* W, void* Wd, qlora_stream_t stream);

/* Scratch bytes the linear entry points need for (M, N, K, r), 1 <= r <= 128: the scaled rank-r
 * activations, the fused down-projection's counters, the few-token split partials of the rank-r
 * reductions and the stream-K partial sums of the dequant GEMM (sized for any device of up to
 * 160 SMs), for M <= 32 a region where the down-projection leaves its split partials for the
 * few-token kernels' last launch to add (so each direction is three launches), plus, for r not
 * a multiple of 8, the zero-padded copies described below.  Needs no GPU; 0 for an invalid
 * shape. */
QLORA_API size_t qlora_workspace_bytes(int M, int N, int K, int r);

/* Forward.  X [M, K], A [r, K], B [N, r] bf16 device (read); H [M, N] bf16 device (written);
 * XA_saved [M, r] bf16 device (written: X A^T rounded to bf16, kept for the backward), or
 * NULL to keep nothing and let the backward recompute it ("What is Unsloth? Faster LLM
 * Fine-Tuning Explained", "How does Unsloth make fine-tuning faster?": recompute instead of
 * store).
 * ws: device scratch of at least qlora_workspace_bytes(M, N, K, r) bytes.
 * alpha: LoRA alpha; s = alpha / r.  1 <= r <= 128.  A rank that is not a multiple of 8 runs
 * at r rounded up to 8 on zero-padded copies of A, B (and, backward, XA_saved) in ws, the
 * padded rows and columns contributing exact zeros; the results are those of rank r, at the
 * cost of a few device copies per call (the tensor-memory operands need rows of a multiple of
 * 16 bytes).
 * For M <= 32 the base product applies each block's absmax to the block's 64-deep partial sum
 * (the weight enters as bf16(code value) * absmax rather than bf16(code value * absmax)); the
 * two agree within one bf16 rounding of the weight.  Larger M and dX use the dequantised
 * bf16 weight exactly as qlora_nf4_dequant returns it. */
QLORA_API qlora_status qlora_linear_fwd(const void* X, const qlora_nf4_weight* W, const void* A,
                              const void* B, int M, int r, float alpha, void* H, void* XA_saved,
                              void* ws, size_t ws_bytes, qlora_stream_t stream);

/* Backward.  dY [M, N], X [M, K], A, B, XA_saved [M, r] bf16 device (read).  XA_saved may be
 * NULL: X A^T is then recomputed from X (one more pass over X), bit-identical to the value the
 * forward would have saved, so the results do not change.
 * dX [M, K] bf16 device (written; may be NULL to skip the dX GEMM).
 * dA [r, K] and dB [N, r] fp32 device (overwritten).  ws and r as for the forward.
 * With XA_saved and dX given, dA and dB may be computed on a library-owned stream beside the dX
 * GEMM (qlora_set_side_overlap); the call joins it back to `stream` before returning, so the
 * outputs are ordered on `stream` as usual.  For M <= 32, dA and dB are computed in the
 * few-token dX kernel's last launch, summed over the tokens in order in fp32. */
QLORA_API qlora_status qlora_linear_bwd(const void* dY, const void* X, const qlora_nf4_weight* W,
                              const void* A, const void* B, const void* XA_saved, int M, int r,
                              float alpha, void* dX, float* dA, float* dB, void* ws,
                              size_t ws_bytes, qlora_stream_t stream);

/* ---- Several adapters packed into one launch sequence. ----
 * n adapters share the input X and own consecutive row ranges of one stacked base weight:
 * q/k/v projections, or gate/up ("Speed Up Fine-Tuning 2x with Unsloth on Llama and Mistral",
 * "How it works internally", item 3: several LoRA adapters packed into a single tensor;
 * "Unsloth vs QLoRA vs Liger-Kernel", section 5, step 2: adapters on q/k/v/o/gate/up/down).
 * Adapter g has N_g = group_rows[g] output rows (host array of n_groups ints) and rank r; all
 * share alpha, so s = alpha / r.  Layouts (bf16 unless noted, all device):
 *   W        NF4 [N, K], N = sum N_g: the adapters' base weights stacked by rows (pack the
 *            stacked bf16 weight with qlora_nf4_pack);
 *   A        [n r, K]: A_0, A_1, ... stacked by rows;      B  [N, r]: B_0, B_1, ... by rows;
 *   H, dY    [M, N]: adapter g's outputs in columns [sum_{i<g} N_i, sum_{i<=g} N_i);
 *   XA_saved [M, n r]: X A_g^T in columns [g r, (g + 1) r) (NULL: recomputed, as for one);
 *   dA       [n r, K] fp32 (rows of A_g at g r);          dB [N, r] fp32 (rows of B_g).
 * The results equal n separate qlora_linear_fwd / qlora_linear_bwd calls on the slices, with
 * dX their sum; X is read once for all adapters' down-projections, and each large product is
 * one launch over all adapters' rows.  Requirements: 1 <= n_groups <= 8; r and n r multiples
 * of 8 in [8, 128]; every N_g a multiple of 128 (of 64 when n_groups = 1); sum N_g = W->N.
 * Violations return QLORA_ERR_SHAPE (QLORA_ERR_NULL for a NULL group_rows). */
QLORA_API size_t qlora_grouped_workspace_bytes(int M, int N, int K, int r, int n_groups);

QLORA_API qlora_status qlora_grouped_fwd(const void* X, const qlora_nf4_weight* W, const void* A,
                               const void* B, const int* group_rows, int n_groups, int M, int r,
                               float alpha, void* H, void* XA_saved, void* ws, size_t ws_bytes,
                               qlora_stream_t stream);

/* The packed gate/up forward with its SwiGLU ("Unsloth vs QLoRA vs Liger-Kernel", section 2:
 * the SwiGLU MLP among the hand-derived fused ops): qlora_grouped_fwd with group_rows {I, I}
 * (gate rows [0, I) of W, up rows [I, 2I); I = W->N / 2), writing GU [M, 2I] (g, u) as that
 * call writes H, and also act [M, I] = silu(g) * u (bf16 g and u, fp32 math, bf16 result: the
 * bits qlora_swiglu_packed_fwd gives on GU).  Where the dequant GEMM runs whole tiles (M > 32,
 * enough tiles for every SM, I % 128 == 0, rank fusion not used) each CTA takes a gate tile and
 * then the up tile of the same rows and tokens, and the up tile's epilogue computes act from
 * the g it has just written: no separate launch and no second read of GU.  Otherwise the call
 * is qlora_grouped_fwd followed by qlora_swiglu_packed_fwd.  The workspace is
 * qlora_grouped_workspace_bytes(M, W->N, K, r, 2).  Requirements as for qlora_grouped_fwd with
 * n_groups = 2 (I a multiple of 128); act must be 16-byte aligned. */
QLORA_API qlora_status qlora_grouped_fwd_swiglu(const void* X, const qlora_nf4_weight* W,
                                                const void* A, const void* B, int M, int r,
                                                float alpha, void* GU, void* XA_saved, void* act,
                                                void* ws, size_t ws_bytes, qlora_stream_t stream);

QLORA_API qlora_status qlora_grouped_bwd(const void* dY, const void* X, const qlora_nf4_weight* W,
                               const void* A, const void* B, const void* XA_saved,
                               const int* group_rows, int n_groups, int M, int r, float alpha,
                               void* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                               qlora_stream_t stream);

/* SwiGLU glue for the MLP workload: a = g * sigmoid(g) * u (elementwise, n elements, bf16
 * device), and its exact backward dg = da*u*sig(g)*(1 + g*(1 - sig(g))), du = da*g*sig(g).
 * Computed in fp32, rounded to bf16.  ("Unsloth vs QLoRA vs Liger-Kernel", section 2: the
 * SwiGLU MLP is among the hand-differentiated ops.) */
QLORA_API qlora_status qlora_swiglu_fwd(const void* g, const void* u, void* a, int64_t n,
                              qlora_stream_t stream);
QLORA_API qlora_status qlora_swiglu_bwd(const void* g, const void* u, const void* da, void* dg, void* du,
                              int64_t n, qlora_stream_t stream);

/* The same glue on the output of a packed gate/up layer (gate and up adapters sharing X, see
 * qlora_grouped_fwd with group_rows {I, I}): gu [M, 2I] bf16 holds g in columns [0, I) and u
 * in [I, 2I) of each row; a and da are [M, I]; dgu [M, 2I] receives dg and du in the same
 * places, i.e. the upstream gradient of the packed layer.  I must be a multiple of 8.  M = 0
 * does nothing. */
QLORA_API qlora_status qlora_swiglu_packed_fwd(const void* gu, void* a, int64_t M, int I,
                                               qlora_stream_t stream);
QLORA_API qlora_status qlora_swiglu_packed_bwd(const void* gu, const void* da, void* dgu,
                                               int64_t M, int I, qlora_stream_t stream);

/* ---- LM head + cross-entropy over a frozen NF4 head, chunked over tokens. ----
 * "Unsloth vs QLoRA vs Liger-Kernel", section 3 (fused cross-entropy): the projection to the
 * vocabulary and the loss are computed in chunks of tokens so the [tokens x vocab] logits are
 * never held at once.  For each chunk of `chunk` tokens (<= 0: all M at once):
 *   z = X_c deq(W)^T                    [chunk, V] bf16 in the workspace (the dequant GEMM)
 *   token_loss_m = logsumexp(z_m) - z_m[label_m]          (fp32, online max / sum of exp)
 *   dz = (softmax(z) - onehot(label)) / count, in place   (only when dX is requested)
 *   dX_c = dz deq(W)                    [chunk, K] bf16 (the dequant GEMM, transposed access)
 * and loss = sum(token_loss) / count, count = number of labels in [0, V).  A label outside
 * [0, V) (e.g. -100) ignores its token: loss 0, gradient 0, not counted; with no counted token
 * loss and dX are 0.  W is the NF4 head [V, K] (V % 64 == 0, K % 64 == 0, V >= 128, K >= 128;
 * QLORA_ERR_SHAPE otherwise); it gets no gradient.
 *   X [M, K] bf16, labels [M] int32 (device, read); loss [1] fp32 (device, written);
 *   token_loss [M] fp32 (device, written; may be NULL); dX [M, K] bf16 (written; NULL: loss
 *   only).  ws: device scratch of qlora_lm_head_ce_workspace_bytes(M, V, K, chunk) bytes,
 *   about chunk x V x 2 plus the GEMM's partial sums. */
QLORA_API size_t qlora_lm_head_ce_workspace_bytes(int M, int V, int K, int chunk);
QLORA_API qlora_status qlora_lm_head_ce(const void* X, const qlora_nf4_weight* W, const int* labels,
                                        int M, int chunk, float* loss, float* token_loss, void* dX,
                                        void* ws, size_t ws_bytes, qlora_stream_t stream);

/* Its cross-entropy stages, for custom compositions (the GEMMs are qlora_nf4_gemm with r = 0):
 * count_out[0] = number of labels in [0, V); z [rows, V] bf16 (V % 8 == 0) -> token_loss
 * [rows] and, with write_grad, z := (softmax(z) - onehot) / count_in[0] in place;
 * loss[0] = sum(token_loss[0..M)) / count_in[0] (0 when the count is 0). */
QLORA_API qlora_status qlora_cross_entropy_count(const int* labels, int M, int V, int* count_out,
                                                 qlora_stream_t stream);
QLORA_API qlora_status qlora_cross_entropy_rows(void* z, int rows, int V, const int* labels,
                                                const int* count_in, float* token_loss,
                                                int write_grad, qlora_stream_t stream);
QLORA_API qlora_status qlora_cross_entropy_mean(const float* token_loss, int M, const int* count_in,
                                                float* loss, qlora_stream_t stream);

/* ---- The stages the two linear entry points are composed of (same validation rules). ---- */

/* The stage calls take an optional adapter split, `group_rows` (host array of n_groups row
 * counts, with the rules of the packed-adapter entry points) or NULL for a single adapter.
 *
 * Rank-r down-projection: out = in . Wl^T with in [M, C] bf16 and Wl given either as
 * w [r, C] (w_is_r_by_c = 1, the LoRA A) or as w [C, r] (w_is_r_by_c = 0, the LoRA B).
 * Writes bf16(out) to `saved` [M, r] (may be NULL) and bf16(scale * out) to `scaled` [M, r].
 * With group_rows (w_is_r_by_c = 0 only): r = n r_g output columns, w = B [C, r_g] stacked by
 * adapter, and Wl is block-diagonal: rows of adapter g feed columns g r_g .. g r_g + r_g - 1.
 * The reduction over C is split across the CTAs of a thread-block cluster and summed in a fixed
 * order in distributed shared memory.  ws / ws_bytes (may be NULL / 0; 16-byte aligned): with
 * few tokens the reduction is split further over several clusters whose fp32 partials (up to
 * 128 r 4 bytes per 128 tokens for each cluster) go to ws and a second launch adds them in
 * cluster order; without room in ws it stays on one cluster per 128 tokens.  Either way the
 * results do not depend on timing. */
QLORA_API qlora_status qlora_lora_down(const void* in, int M, int C, const void* w,
                                       int w_is_r_by_c, int r, const int* group_rows,
                                       int n_groups, float scale, void* saved, void* scaled,
                                       void* ws, size_t ws_bytes, qlora_stream_t stream);

/* The dequant GEMM with the fused rank-r extension (r = 0: none, ext_w / ext_act may be NULL,
 * and the reduction, K or N, must be at least 128):
 *   transpose_w = 0: out[M, N] = act[M, K] . deq(W0)^T + ext_act[M, r] . ext_w^T, ext_w = B [N, r]
 *   transpose_w = 1: out[M, K] = act[M, N] . deq(W0)   + ext_act[M, r] . ext_w,   ext_w = A [r, K]
 * act, ext_w, ext_act bf16 device (read); out bf16 device (written).  The scale s is expected
 * to be folded into ext_act already (qlora_lora_down's `scaled` output).
 * With group_rows (transpose_w = 0 only): ext_act is [M, n r] and output row n of adapter g
 * takes ext_act's columns g r .. g r + r - 1; ext_w = B [N, r] stacked by adapter.
 * ws: device scratch for the partial sums of problems with fewer output tiles (128 output
 * features x up to 512 tokens) than SMs, which are cut along the reduction so every SM works;
 * at least qlora_workspace_bytes(M, N, K, r) bytes (may be NULL when that shape needs none). */
QLORA_API qlora_status qlora_nf4_gemm(const void* act, const qlora_nf4_weight* W, int transpose_w,
                                      const void* ext_w, const void* ext_act, int M, int r,
                                      const int* group_rows, int n_groups, void* out, void* ws,
                                      size_t ws_bytes, qlora_stream_t stream);

/* Rank-r weight gradient: G[c, j] = scale * sum_m big[m, c] small[m, j] with big [M, C] and
 * small [M, r] bf16 device; written fp32 as out [C, r] (out_r_by_c = 0, e.g. dB) or
 * out [r, C] (out_r_by_c = 1, e.g. dA).  With group_rows (adapters along big's columns):
 * small is [M, n r] and column c of adapter g uses small[m, g r + j].
 * Reduced over M inside thread-block clusters: ws / ws_bytes are ignored (may be NULL / 0). */
QLORA_API qlora_status qlora_lora_grad(const void* big, int M, int C, const void* small, int r,
                                       const int* group_rows, int n_groups, float scale,
                                       float* out, int out_r_by_c, void* ws, size_t ws_bytes,
                                       qlora_stream_t stream);

/* Host-only (no GPU needed): the dequant GEMM's launch plan for a problem of M tokens, rows_w
 * output rows (N for the forward, K for dX) and steps_per_tile 64-deep reduction steps (K/64
 * or N/64, plus the extension's) on a device with sm_count SMs.  Writes the token tile (bt
 * tokens per MMA, nh halves per tile), the schedule (0: whole tiles, one CTA per SM; 1:
 * stream-K), the grid and the stream-K partial-sum bytes the workspace must hold. */
QLORA_API qlora_status qlora_gemm_plan(int M, int rows_w, int steps_per_tile, int sm_count,
                                       int* bt, int* nh, int* streamk, int* grid,
                                       size_t* partial_bytes);

/* Host-only: 1 if the dequant GEMM launch for this problem computes the rank-r down-projection
 * itself (X A^T in the forward, transpose_w = 0; dY B in dX, transpose_w = 1) for n adapters of
 * rank r packed into rank_cols = n r columns, else 0 (the layer then launches it separately
 * first).  *bt (nullable) receives the fused launch's tokens per half tile, else 0.  The
 * tensor cores add the rank product on 128-token windows of a token tile's first tiles, so it
 * fuses when: whole tiles of two halves of 144..240 tokens model at most 4 % slower than the
 * GEMM's own choice of tile; rank_cols is a multiple of 8 up to 32 (dX: r = 16 or 32); the rank
 * operand's tiles fit in shared memory; and every token tile's windows (up to 4) fall on its
 * tiles in the first wave that reaches it.  No counterpart on the pages: it reports a scheduling
 * decision of this implementation ("Unsloth vs QLoRA vs Liger-Kernel", section 2: the rank-r
 * products fused into the layer's kernels). */
QLORA_API int qlora_gemm_rank_fusable(int M, int rows_w, int steps_per_tile, int sm_count,
                                      int rank_cols, int r, int transpose_w, int* bt);

/* Host-only, process-wide: 1 makes qlora_linear_* / qlora_grouped_* compute the rank-r
 * down-projection inside the dequant GEMM launch whenever qlora_gemm_rank_fusable says that
 * launch can (saving one launch and one read of X or dY); 0 (the default) always launches it
 * separately.  Results agree within the parity tolerance either way (the fp32 sums run in a
 * different order).  Off by default because on a B200 the fused q_proj step (4096 tokens,
 * 4096 x 4096, r = 16) measured 0.388 ms against 0.359 ms separate: the other tiles of a token
 * tile wait at their extension step for the window tiles.  Returns the previous setting.  No
 * counterpart on the pages (a scheduling choice of this implementation). */
QLORA_API int qlora_set_rank_fusion(int enable);

/* Host-only, process-wide: where dB and dA of qlora_linear_bwd / qlora_grouped_bwd run when
 * XA_saved and dX are given and the dX GEMM runs whole tiles.  They can run on a few SMs taken
 * from the GEMM (qlora_backward_side_sms) while the GEMM runs on the rest, on a stream the library
 * owns, forked from the caller's stream after dY B and joined back before the call returns
 * (two events; inside a stream capture they become graph edges, so the captured graph has the
 * same fork and join).  0: never (dB and dA after the GEMM); 1 (the default): when the
 * launcher's schedule model expects that to be faster and the shape is one where it measured
 * faster (qlora_backward_side_sms); 2: always, with the model's best split.
 * Every output has the same bits in all three modes: the side kernel sums each reduction in the
 * same step ranges and order as the cluster kernels that run otherwise.  If the side stream
 * cannot be created the work runs after the GEMM.  Concurrent calls on one device take turns at
 * the fork/join (a mutex).  Returns the previous mode.  No counterpart on the pages (a
 * scheduling choice of this implementation). */
QLORA_API int qlora_set_side_overlap(int mode);

/* Host-only, no GPU needed: the number of SMs (even, 2..32) qlora_linear_bwd /
 * qlora_grouped_bwd give to dB and dA beside the dX GEMM, for M tokens, W0 [N, K] and
 * R = n r packed rank columns on a device of sm_count SMs, under side-overlap mode `mode`
 * (0, 1, 2 as in qlora_set_side_overlap; -1: the current setting); 0 when they run after the
 * GEMM.  The split minimises the launcher's schedule model of max(GEMM on the other SMs, dY
 * and X streamed at ~26 GB/s per SM); mode 1 takes it only when that model beats running them
 * after the GEMM, R <= 32 and dY (2 M N bytes) is at most 48 MiB (larger ranks or operands
 * measured slower beside the GEMM on a B200); modes 1 and 2 give 0 for stream-K shapes,
 * M <= 256 and fewer than 64 SMs. */
QLORA_API int qlora_backward_side_sms(int M, int N, int K, int R, int sm_count, int mode);

/* Number of kernels this library has launched in this process so far (all devices). */
QLORA_API uint64_t qlora_launch_counter(void);

/* ---- Allocation-free forward (no counterpart on the pages: an engineering addition). ----
 *
 * For callers that cannot allocate device memory at all -- for example code running inside
 * a host framework that owns every device allocation and hands out no workspace, or a host
 * that links this C ABI without any device allocator of its own -- and so cannot provide the
 * `ws` buffer qlora_linear_fwd needs.  Same computation and arguments as qlora_linear_fwd
 * minus the workspace: the scratch (the scaled rank-r activation s*XA and the down-projection
 * partials) lives in a fixed array inside this library, qlora_noalloc_scratch_bytes() bytes
 * per GPU (8 MiB), which every GPU that loads the library keeps until the process exits.
 * Returns QLORA_ERR_WORKSPACE, before enqueuing anything, when (M, K, r) would need more
 * scratch than that (roughly 2*M*r bytes plus M*r*4 bytes per split of the down-projection).
 * The first call on a device looks up the array's device address (with that device current),
 * so make that first call before any stream capture.  The entry point calls no cudaMalloc or
 * cudaFree.  All calls on a device share the one array and each call overwrites it in full
 * (it keeps the last call's contents; nothing in it must start at zero): calls whose kernels
 * overlap on the GPU -- on different streams without ordering between them -- race. */
QLORA_API qlora_status qlora_linear_fwd_noalloc(const void* X, const qlora_nf4_weight* W,
                                                const void* A, const void* B, int M, int r,
                                                float alpha, void* H, void* XA_saved,
                                                qlora_stream_t stream);

/* Size in bytes of the fixed scratch array used by qlora_linear_fwd_noalloc. */
QLORA_API size_t qlora_noalloc_scratch_bytes(void);

/* Self-test of the failure detection: enqueues one thread that waits, through the kernels'
 * own bounded wait, on a barrier nothing completes.  The wait runs out after its 2 s limit and
 * the kernel returns; a following qlora_device_error() then reports QLORA_ERR_TIMEOUT with
 * code 6 (the self-test's site, CTA 0, tag 0), provided the word was clear before.  The
 * context stays usable. */
QLORA_API qlora_status qlora_selftest_bounded_wait(qlora_stream_t stream);

/* Synchronising: returns the device error word of the current device (0 = none; otherwise
 * a code naming the wait that ran out) and clears it. */
QLORA_API qlora_status qlora_device_error(int* code);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */

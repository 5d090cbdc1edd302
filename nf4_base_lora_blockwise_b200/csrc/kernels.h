// kernels.h -- internal launchers behind the C ABI (not exported).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "nf4_dequant.cuh"

namespace qlora {

// Launch `kernel`, as a programmatic dependent of the previous kernel on the stream when `pdl`
// (its CTAs call pdl_wait() before touching global memory), optionally as clusters of
// `cluster` CTAs.
template <typename... Params, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, bool pdl, int cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(n);
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, int cluster, Args... args) {
  return launch_kernel(kernel, grid, block, smem, stream, true, cluster, args...);
}

// ------------------------------ adapters packed along the output rows -----------------------
// A stacked base weight [sum N_g, K] whose rows are split into n adapters (q/k/v, gate/up):
// adapter g owns rows [end[g-1], end[g]) and columns [g r, (g + 1) r) of the packed rank-r
// activations ([M, n r]: X A_cat^T, dY B_bd).  Every end is a multiple of 128, so no 128-row
// tile of any kernel straddles two adapters.  n = 1 is the plain single-adapter layer.
constexpr int kMaxGroups = 8;
struct RowGroups {
  int n;
  int end[kMaxGroups];
};
// Adapter owning `row` (static indices only, so a kernel parameter stays in the constant bank).
__host__ __device__ __forceinline__ int row_group(const RowGroups& g, int row) {
  int i = 0;
#pragma unroll
  for (int j = 0; j < kMaxGroups - 1; ++j) i += (j + 1 < g.n && row >= g.end[j]) ? 1 : 0;
  return i;
}
inline RowGroups single_group(int rows) {
  RowGroups g = {};
  g.n = 1;
  g.end[0] = rows;
  return g;
}

// ------------------------------ NF4 pack / dequant -----------------------------------------
cudaError_t launch_nf4_pack(const __nv_bfloat16* W, int N, int K, int dq, uint8_t* q,
                            float* absmax, uint8_t* absmax_q8, float* absmax_scale,
                            const Codebook& cb, cudaStream_t stream);
cudaError_t launch_nf4_dequant(const uint8_t* q, const float* absmax, const uint8_t* q8,
                               const float* scale, int dq, int N, int K, __nv_bfloat16* out,
                               const Codebook& cb, cudaStream_t stream);

// ------------------------------ dequant GEMM (tcgen05) -------------------------------------
// out[M, rows_w] = act[M, red] . deq(W)^T-or-not + s_small[M, r] . ext^T, where the weight
// operand is dequantised in the mainloop.  kTransW = false: forward (rows_w = N, red = K);
// kTransW = true: dX (rows_w = K, red = N).
struct GemmArgs {
  int M;
  int rows_w;
  int kt;          // reduction steps of 64
  int n_ext;       // LoRA extension chunks (64 wide along r)
  int r_pad16;     // r rounded up to a multiple of 16
  int bt;          // tokens per half tile = MMA N
  int nh;          // token halves per tile (1 or 2)
  int kblocks;     // K / 64 = absmax blocks per row of W0
  int N;           // rows of W0
  int dq;
  const float* absmax;
  const uint8_t* absmax_q8;
  const float* absmax_scale;
  __nv_bfloat16* out;
  int* err;        // device error word
  float* partial;  // stream-K partial sums [grid][2][tile tokens][128] fp32 (workspace)
  int streamk;     // set by the launcher
  RowGroups groups;  // forward: the adapter of each row tile selects its slice of ext_act
  Codebook cb;
  // Rank-r down-projection fused into the launch (whole-tile schedules only; rank_cols <= 32):
  // the tensor cores compute rank = act . Wr -- Wr = A^T [K, n r] for the forward (X A^T), the
  // block-diagonal B [N, n r] for dX (dY B) -- in 128-token windows from the activation tiles
  // already in shared memory, the epilogue warps write rank (bf16, nullable) and
  // rank_scale * rank (bf16, the extension operand ext_act maps) and count the published windows
  // per token tile in rank_flags, which every tile's extension step waits on.
  int fuse;                     // 0: ext_act was written by an earlier launch
  int rank_cols;                // n r
  int rank_r;                   // r of one adapter
  RowGroups rank_groups;        // dX: the adapters' row ranges of B (= column ranges of dY)
  const __nv_bfloat16* rank_w;  // forward: A [n r, K]; dX: B [N, r]
  __nv_bfloat16* rank_saved;    // [M, n r] or null
  __nv_bfloat16* rank_scaled;   // [M, n r]
  float rank_scale;
  unsigned* rank_flags;         // [token tiles], zero before the launch
  unsigned rank_slot;           // bytes of one rank-operand tile (gemm_rank_slot_bytes)
  // SMs the launch may use (0: all of them); the rest are left to a kernel running beside it.
  // The tile (bt, nh) must be the one gemm_pick_tile gives for that many SMs.
  int sm_limit;
  // SwiGLU on a packed gate/up layer (whole tiles, forward, unfused rank; 0 / null: off):
  // rows [0, glu_I) of W0 are the gate rows and [glu_I, 2 glu_I) the up rows (glu_I % 128 == 0).
  // CTA b takes (gate row tile j, token tile) pairs b, b + G, ..., each as the gate tile followed
  // by the matching up tile, and the up tile's epilogue adds glu_out[M, glu_I] =
  // silu(g) * u from the g it wrote one tile earlier (bf16 g and u, fp32 math).
  __nv_bfloat16* glu_out;
  int glu_I;
};

struct GemmMaps {
  CUtensorMap act;      // [M, red] bf16, box {64, bt}, 128B swizzle
  CUtensorMap q;        // [N, K/2] u8
  CUtensorMap ext_w;    // B_lora [N, r] (fwd) or A_lora [r, K] (dX), bf16
  CUtensorMap ext_act;  // scaled rank-r activation [M, n, r] bf16 (n adapters), box {64, 1, bt}
  CUtensorMap rank;     // fused down-projection: A [n r, K] box {64, n r} (fwd) or
                        // B [N, r] box {r, 64} (dX); unused otherwise
};

// Work schedule of one launch: whole tiles (one CTA per tile, at most one per SM) or, with
// fewer tiles than SMs, stream-K over one CTA per SM (up to kGemmMaxCtas) plus a finalize
// kernel that adds the partial sums of cut tiles.
constexpr int kGemmMaxCtas = 160;
struct GemmSchedule {
  int n_tiles;
  int streamk;
  int grid;
  size_t partial_floats;  // workspace the stream-K partials need
};
// fused: the tile a launch with the fused down-projection uses (two halves of 144..240 tokens).
GemmSchedule gemm_schedule(int M, int rows_w, int steps_per_tile, int sm_count,
                           bool fused = false);
// Whether a launch of this shape can fuse a rank-`rank_cols` down-projection (whole tiles, every
// token tile's 16-token blocks spread over its first wave of tiles at most 2 per tile).
bool gemm_rank_fusable(int M, int rows_w, int steps_per_tile, int sm_count, int rank_cols,
                       unsigned rank_slot);
// Bytes of one rank-operand tile of the fused down-projection (0: that form is not fused):
// forward A [n r rounded up to 16 rows, 64 k] (128 B rows); dX B [64 n rows, r] for r = 16, 32.
inline unsigned gemm_rank_slot_bytes(bool trans_w, int rank_cols, int r) {
  if (trans_w) return (r == 16 || r == 32) ? 128u * static_cast<unsigned>(r) : 0u;
  return 128u * static_cast<unsigned>((rank_cols + 15) / 16 * 16);
}
// SMs to hand to `side_bytes` of streaming work (dB and dA) that runs beside a whole-tile
// launch of this shape: the count s (even, 2..32) minimising the schedule model's
// max(launch on sm_count - s SMs with its tile re-picked, side_bytes at ~26 GB/s per SM),
// or 0 when running the work after the launch is modelled no slower (always 0 for stream-K
// shapes and M <= 256).  force: the best s even then.  *us: the modelled duration of both.
int gemm_side_sms(int M, int rows_w, int steps_per_tile, int sm_count, double side_bytes,
                  bool force, double* us);
// Counters the fused down-projection needs in the workspace (zeroed before each launch).
size_t gemm_rank_flag_bytes(int M);
// Partial-sum bytes any device (at most kGemmMaxCtas SMs) may need for this shape.
size_t gemm_partial_bytes_bound(int M, int rows_w, int steps_per_tile);

// Token tile: bt tokens per MMA (N) and nh halves per tile.  Up to 256 tokens: one half of
// M rounded up to 16.  More: two halves of 256, or, when whole tiles fill the GPU, the
// narrower bt (multiple of 16, >= 128) that a cost model of the busiest CTA favours.
struct GemmTile {
  int bt;
  int nh;
};
GemmTile gemm_pick_tile(int M, int rows_w, int steps_per_tile, int sm_count, bool fused = false);
cudaError_t gemm_device_sms(int* sms);  // SMs of the current device (cached)
size_t gemm_smem_bytes(int bt, int nh);
// Whether a forward launch of the packed gate/up layer [2 I, K] on M tokens can add the SwiGLU
// output in its epilogue (GemmArgs::glu_out): whole tiles on sm_count SMs, I % 128 == 0.
bool gemm_glu_ok(int M, int I, int steps_per_tile, int sm_count);
// Falls back to whole tiles when stream-K is chosen but `partial` is null or smaller than the
// schedule needs (partial_floats_avail).  *launched = kernels enqueued (1, or 2 with stream-K).
cudaError_t launch_qlora_gemm(bool trans_w, const GemmMaps& maps, GemmArgs args,
                              size_t partial_floats_avail, cudaStream_t stream, int* launched);

// The same GEMM on CTA pairs (tcgen05.mma.cta_group::2, M = 256 over two SMs; qlora_gemm2.cu)
// for the whole-tile regime: pair tiles of 256 weight rows x (nh x bt) tokens, each CTA of a
// pair holding 128 rows and bt / 2 tokens of every MMA's activation block (TMA boxes of bt / 2
// rows).  No partial sums.  gemm2_applies: enough pair tiles for every pair, and no adapter
// boundary inside a 256-row pair tile.
GemmTile gemm2_pick_tile(int M, int rows_w, int steps_per_tile, int sm_count);
bool gemm2_applies(int M, int rows_w, int steps_per_tile, int sm_count, const RowGroups& groups);
size_t gemm2_smem_bytes(int bt, int nh);
cudaError_t launch_qlora_gemm2(bool trans_w, const GemmMaps& maps, const GemmArgs& args,
                               cudaStream_t stream, int* launched);

// ------------------------------ few-token forward (mma.sync, register-direct) ---------------
// h[M, N] = X[M, K] . deq(W0)^T + ext_act[M, g(n), r] . ext_w[N, r]^T for M <= 32 (g(n) the
// adapter of row n): stream-K over (128-row tile, 64-block) units with fp32 partial slots and
// a fixed-order finalize.
// The rank-r down-projection of a few-token layer left as fp32 partials for its consumer to
// add (rank_down_plan's second-level split, gsplit > 1, one row tile: M <= 128): the consumer
// sums part[g][m][j] over g in order -- rank_down_finalize's arithmetic, so the same bits --
// and uses bf16(scale * sum) as the LoRA term's rank-r activation.
struct RankFold {
  const float* part;     // [gsplit][128][R] fp32
  int gsplit;
  int R;                 // n r columns
  float scale;           // alpha / r
  __nv_bfloat16* saved;  // [M, R]: bf16(sum), written by the consumer (nullable)
};
constexpr int kFoldMaxR = 128;

struct GemvPlan {
  int tt;                 // token tiles of 8
  long long units;
  int grid;
  int max_seg;            // row tiles a CTA's range can touch
  size_t partial_floats;
  size_t smem;
};
// dX for few tokens (nf4_dx_fewtok.cu): CTAs of 256 output columns x a range of weight rows,
// fp32 partials per row split in the workspace, a finalize adding them in order with the LoRA
// term.  Tile maps: codes [N, K/2] u8 box {128, 64} and dY [M, N] bf16 box {64, 16 mb}, both
// 128B-swizzled.
constexpr int kFewTokDxMaxTokens = 32;
struct FewTokDxPlan {
  int gk, splits, grid;
  int mb;             // 16-token blocks (1 or 2)
  size_t part_bytes;  // workspace the partials need
};
FewTokDxPlan fewtok_dx_plan(int M, int N, int K, int sm_count);
// tm_am (nullable): fp32 absmax [N, K/64] in boxes {4, 64}, taken when the absmax is not
// double-quantised and K % 256 == 0 (the stage's block scales then arrive with its codes).
cudaError_t launch_nf4_fewtok_dx(const CUtensorMap& tm_q, const CUtensorMap& tm_dy,
                                 const CUtensorMap* tm_am, const FewTokDxPlan& p, int M, int N,
                                 int K, const float* absmax,
                                 const uint8_t* absmax_q8, const float* absmax_scale, int dq,
                                 const __nv_bfloat16* sdyb, const __nv_bfloat16* A, int R,
                                 __nv_bfloat16* dx, float* part, size_t part_bytes,
                                 const Codebook& cb, int* err, cudaStream_t stream,
                                 bool finalize = true);
// The few-token layer backward's last launch, after the main dX kernel ran without its
// finalize (or alone, with dx null): dY B summed from the down-projection's partials (fold),
// dX from the main kernel's split partials (xpart, splits) plus (s dYB) A, dA = s dYB^T X and
// dB_g = s dY_g^T XA_g, each summed over the M <= 32 tokens in order in fp32.
struct FewTokTail {
  RankFold fold;             // dY B partials (fold.R = n r; fold.saved unused)
  const __nv_bfloat16* X;    // [M, K]
  const __nv_bfloat16* dY;   // [M, N]
  const __nv_bfloat16* XA;   // [M, n r]
  const __nv_bfloat16* A;    // [n r, K]
  RowGroups groups;          // adapters along W0's rows; r columns of XA each
  int r;
  float* dA;                 // [n r, K]
  float* dB;                 // [N, r]
};
cudaError_t launch_fewtok_bwd_tail(const FewTokTail& tail, const float* xpart, int splits, int M,
                                   int N, int K, __nv_bfloat16* dx, cudaStream_t stream);
constexpr int kGemvMaxTokens = 32;
GemvPlan gemv_plan(int M, int N, int K, int sm_count);
cudaError_t launch_nf4_gemv_fwd(const __nv_bfloat16* X, const uint8_t* q, const float* absmax,
                                const uint8_t* absmax_q8, const float* absmax_scale, int dq, int M,
                                int N, int K, const __nv_bfloat16* ext_act,
                                const __nv_bfloat16* ext_w, int r, const RowGroups& groups,
                                __nv_bfloat16* out, float* partial, size_t partial_floats,
                                const Codebook& cb, cudaStream_t stream,
                                const RankFold* fold = nullptr);

// ------------------------------ rank-r products (TMA ring, mma.sync, cluster reduction) ------
// down: out[m, j] = sum_c in[m, c] Wl(j, c), Wl = A [R, C] (w_rc) or B [C, rg] (block-diagonal
//       over n adapters along C when groups.n > 1: R = n rg); writes bf16(out) to `saved`
//       (nullable) and bf16(scale * out) to `scaled`, both [M, R].
// grad: G[c, j] = scale * sum_m big[m, c] small[m, g(c) R + j], small [M, ld_small], g(c) the
//       adapter of column c; written as out[c R + j] (out_cr) or out[j C + c].
// The reduction is split over the CTAs of a cluster and summed in rank order through
// distributed shared memory: one launch, no scratch, deterministic.
struct SmallTile {   // a [64 rows, w columns] bf16 tile as TMA writes it
  int blocks;        // 1, or 2 for w = 128 (two 64-column blocks)
  int box_w;         // columns per TMA box
  uint32_t pitch;    // bytes per row of a block
  uint32_t mask;     // swizzle mask (pitch / 16 - 1 when swizzled, else 0)
  int swizzle;       // TMA swizzle span in bytes (0 = none, 32, 64, 128)
  uint32_t bytes;    // bytes per stage
};
SmallTile small_tile(int w);
struct RankPlan {
  int rows;         // down only: 1 = whole token rows per warp (no cross-CTA reduction)
  int split;        // CTAs per cluster
  int grid;
  int stages;
  size_t smem;
  SmallTile small;  // the Wl / small tile of one stage
  int box_rows_in;  // TMA box height of `in` / `big`
  int box_rows_w;   // TMA box height of Wl (A: R; B: 64 or 256) / small (64)
  int gsplit;       // down, few tokens: clusters per row tile along the reduction (1: one),
                    // their fp32 partials summed in order by a finalize kernel
  size_t part_bytes;  // scratch those partials take
};
struct RankMaps {
  CUtensorMap big;    // in / big [M, C] bf16: box {64, 128} (down) or {64, 64} (grad), SW128
  CUtensorMap small;  // down: A [R, C] box {64, R} SW128, or B [C, rg] per small_tile(rg);
                      // grad: small [M, ld_small] per small_tile(R)
};
// scratch_bytes: workspace the plan may use for a second-level split of the reduction.
RankPlan rank_down_plan(int M, int C, int R, int rg, bool w_rc, int sm_count,
                        size_t scratch_bytes = 0);
RankPlan rank_grad_plan(int M, int C, int R, int sm_count);
// scratch: p.part_bytes of workspace when p.gsplit > 1 (then a finalize kernel follows, unless
// !finalize: the partials' consumer adds them itself, see RankFold).
cudaError_t launch_rank_down(const RankMaps& maps, const RankPlan& p, int M, int C, int R, int rg,
                             bool w_rc, const RowGroups& groups, float scale,
                             __nv_bfloat16* saved, __nv_bfloat16* scaled, int* err,
                             cudaStream_t stream, float* scratch = nullptr,
                             bool finalize = true);
cudaError_t launch_rank_grad(const RankMaps& maps, const RankPlan& p, int M, int C, int R,
                             int ld_small, const RowGroups& groups, float scale, float* out,
                             bool out_cr, int* err, cudaStream_t stream);
// Two gradients of one backward (dB and dA) in one launch, when they share the rank, the
// cluster size and the small-tile layout (rank_grad_pair_ok); same results as two launches.
bool rank_grad_pair_ok(const RankPlan& p1, int R1, const RankPlan& p2, int R2);
cudaError_t launch_rank_grad_pair(const RankMaps& m1, const RankPlan& p1, int M, int C1, int R,
                                  int ld1, const RowGroups& g1, float* out1, bool cr1,
                                  const RankMaps& m2, const RankPlan& p2, int C2, int ld2,
                                  const RowGroups& g2, float* out2, bool cr2, float scale,
                                  int* err, cudaStream_t stream);

// dB and dA of one backward (the second problem may be absent: m2 == nullptr) on `ctas` CTAs,
// one per SM, beside another kernel: each CTA walks whole tiles, summing a tile's reduction in
// the step ranges of the cluster plan p1 / p2, so the results are bit for bit those of
// launch_rank_grad with the same plans.  Launched as a plain (not programmatic) dependent.
cudaError_t launch_rank_grad_side(const RankMaps& m1, const RankPlan& p1, int M, int C1, int R1,
                                  int ld1, const RowGroups& g1, float* out1, bool cr1,
                                  const RankMaps* m2, const RankPlan* p2, int C2, int R2,
                                  int ld2, const RowGroups& g2, float* out2, bool cr2,
                                  float scale, int* err, int ctas, cudaStream_t stream);

// ------------------------------ LM-head cross-entropy ---------------------------------------
// count = number of labels in [0, V); z [rows, V] bf16 (V % 8 == 0) -> loss [rows] and, with
// write_grad, z := (softmax(z) - onehot(label)) / count in place; out = sum(token_loss) / count.
cudaError_t launch_ce_count(const int* labels, int M, int V, int* count, cudaStream_t stream);
cudaError_t launch_ce_rows(__nv_bfloat16* z, int rows, int V, const int* labels, const int* count,
                           float* loss, bool write_grad, cudaStream_t stream);
cudaError_t launch_ce_mean(const float* token_loss, int M, const int* count, float* out,
                           cudaStream_t stream);

// ------------------------------ failure-detection self-test ---------------------------------
// One thread waits on an mbarrier nothing completes; the bounded wait runs out and sets *err.
cudaError_t launch_bounded_wait_selftest(int* err, cudaStream_t stream);

// ------------------------------ SwiGLU ------------------------------------------------------
cudaError_t launch_swiglu_fwd(const __nv_bfloat16* g, const __nv_bfloat16* u, __nv_bfloat16* a,
                              int64_t n, cudaStream_t stream);
cudaError_t launch_swiglu_bwd(const __nv_bfloat16* g, const __nv_bfloat16* u,
                              const __nv_bfloat16* da, __nv_bfloat16* dg, __nv_bfloat16* du,
                              int64_t n, cudaStream_t stream);
// Packed gate/up [M, 2I] (g in columns [0, I), u in [I, 2I)); a, da [M, I]; dgu [M, 2I].
cudaError_t launch_swiglu_packed_fwd(const __nv_bfloat16* gu, __nv_bfloat16* a, int64_t M, int I,
                                     cudaStream_t stream);
cudaError_t launch_swiglu_packed_bwd(const __nv_bfloat16* gu, const __nv_bfloat16* da,
                                     __nv_bfloat16* dgu, int64_t M, int I, cudaStream_t stream);

}  // namespace qlora

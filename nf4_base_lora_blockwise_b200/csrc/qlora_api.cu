// qlora_api.cu -- the C ABI of libqlora_nf4.so (declared in include/qlora_nf4.h): argument
// validation, the NF4 codebook, TMA descriptor encoding, workspace carving and the launch
// sequence of the forward and backward passes.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/qlora_nf4.h"
#include "kernels.h"

namespace qlora {

__device__ int g_qlora_error_word = 0;

namespace {

// ---------------------------------------------------------------------------------------------
// NF4 codebook, derived here independently of any table: quantiles of N(0, 1) at evenly spaced
// probabilities between 1/2 and an offset p* close to 1 -- 8 positive levels, 7 negative ones
// and an exact zero -- divided by the largest one so the set spans [-1, 1].
// p* = 1 - (1/32 + 1/30) / 2.  The inverse normal CDF is found by bisection on erfc.
// ("Unsloth vs QLoRA vs Liger-Kernel", FAQ "What is the difference between LoRA and QLoRA?":
// base weights in 4-bit NormalFloat.)
// ---------------------------------------------------------------------------------------------
double normal_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double normal_quantile(double p) {
  double lo = -12.0, hi = 12.0;
  for (int i = 0; i < 2000; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (mid <= lo || mid >= hi) break;
    if (normal_cdf(mid) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

Codebook make_codebook() {
  const double pstar = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
  double lv[16];
  int n = 0;
  for (int j = 0; j < 7; ++j) lv[n++] = -normal_quantile(pstar + (0.5 - pstar) * j / 7.0);
  lv[n++] = 0.0;
  for (int j = 0; j < 8; ++j) lv[n++] = normal_quantile(pstar + (0.5 - pstar) * j / 8.0);
  std::sort(lv, lv + 16);
  double mx = 0.0;
  for (double v : lv) mx = std::max(mx, std::fabs(v));
  Codebook cb;
  for (int i = 0; i < 16; ++i) cb.level[i] = static_cast<float>(lv[i] / mx);
  for (int i = 0; i < 15; ++i) cb.mid[i] = (cb.level[i] + cb.level[i + 1]) * 0.5f;
  return cb;
}

const Codebook& codebook() {
  static const Codebook cb = make_codebook();
  return cb;
}

// ---------------------------------------------------------------------------------------------
// Device checks and the per-device error word.
// ---------------------------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_arch_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 wrong arch
int* g_err_ptr[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

qlora_status current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_arch_ok[*dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess)
      return QLORA_ERR_CUDA;
    g_arch_ok[*dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_arch_ok[*dev] == 1 ? QLORA_OK : QLORA_ERR_ARCH;
}

qlora_status error_word_ptr(int dev, int** p) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_qlora_error_word) != cudaSuccess) return QLORA_ERR_CUDA;
    g_err_ptr[dev] = static_cast<int*>(a);
  }
  *p = g_err_ptr[dev];
  return QLORA_OK;
}

qlora_status encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !f)
      return QLORA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  *fn = g_encode;
  return QLORA_OK;
}

// 2-D row-major tensor [outer, inner] of `dtype`, row pitch `pitch_bytes`, box {bi, bo}.
qlora_status encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                       uint64_t inner, uint64_t outer, uint64_t pitch_bytes, uint32_t bi,
                       uint32_t bo, CUtensorMapSwizzle swz) {
  PFN_cuTensorMapEncodeTiled_v12000 fn;
  qlora_status st = encoder(&fn);
  if (st != QLORA_OK) return st;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {bi, bo};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

// 3-D row-major bf16 tensor [d2, d1, d0] (d0 contiguous), pitches p1 = d0 * 2 and p2 = d1 * p1
// bytes, box {b0, 1, b2}, 128-byte swizzle.
qlora_status encode_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                            uint64_t d2, uint32_t b0, uint32_t b2) {
  PFN_cuTensorMapEncodeTiled_v12000 fn;
  qlora_status st = encoder(&fn);
  if (st != QLORA_OK) return st;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, 1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qlora_status check_weight(const qlora_nf4_weight* W) {
  if (!W || !W->q) return QLORA_ERR_NULL;
  if (W->double_quant) {
    if (!W->absmax_q8 || !W->absmax_scale) return QLORA_ERR_NULL;
  } else if (!W->absmax) {
    return QLORA_ERR_NULL;
  }
  if (W->N < 64 || W->K < 64 || (W->N % 64) || (W->K % 64)) return QLORA_ERR_SHAPE;
  if (!aligned16(W->q) || (W->absmax && !aligned16(W->absmax)) ||
      (W->absmax_q8 && !aligned16(W->absmax_q8)) ||
      (W->absmax_scale && !aligned16(W->absmax_scale)))
    return QLORA_ERR_ALIGN;
  return QLORA_OK;
}

bool rank_ok(int r) { return r >= 8 && r <= 128 && (r % 8) == 0; }

// Adapters packed along W0's rows: n in [1, kMaxGroups], n r a valid rank, every adapter's row
// count a positive multiple of 128 (any multiple of 64 for n = 1), summing to N.
qlora_status make_groups(const int* rows, int n, int N, int r, RowGroups* g) {
  if (!rows) return QLORA_ERR_NULL;
  if (n < 1 || n > kMaxGroups || !rank_ok(r) || !rank_ok(n * r)) return QLORA_ERR_SHAPE;
  *g = RowGroups{};
  g->n = n;
  long long end = 0;
  for (int i = 0; i < n; ++i) {
    if (rows[i] < 64 || rows[i] % (n == 1 ? 64 : 128)) return QLORA_ERR_SHAPE;
    end += rows[i];
    if (end > N) return QLORA_ERR_SHAPE;
    g->end[i] = static_cast<int>(end);
  }
  return end == N ? QLORA_OK : QLORA_ERR_SHAPE;
}

int ext_steps(int r) { return ((r + 15) / 16 * 16 + 63) / 64; }

// Stream-K partial-sum bytes of the forward (rows N, K/64 steps) or dX (rows K, N/64 steps).
size_t gemm_ws_bytes(int M, int N, int K, int r, bool trans) {
  if (!trans && M <= kGemvMaxTokens) return 4 * gemv_plan(M, N, K, kGemmMaxCtas).partial_floats;
  if (trans) {
    const size_t sk = gemm_partial_bytes_bound(M, K, N / 64 + ext_steps(r));
    if (M > kFewTokDxMaxTokens) return sk;
    const size_t ft = fewtok_dx_plan(M, N, K, kGemmMaxCtas).part_bytes;  // few-token dX partials
    return ft > sk ? ft : sk;
  }
  return gemm_partial_bytes_bound(M, N, K / 64 + ext_steps(r));
}

// ---------------------------------------------------------------------------------------------
// Workspace layout (each region 256-byte aligned):
//   [0]  small0   bf16 [M, r]   s*XA (forward) / dYB (backward)
//   [1]  small1   bf16 [M, r]   s*dYB (backward)
//   [2]  flags    u32 per token tile: the fused down-projection's published blocks, zeroed by
//                 the call before the launch that counts them
//   [3]  scratch  fp32 partial sums of the dequant GEMM (stream-K slots, or the few-token
//                 kernel's segment slots), written and read within one launch pair
//   [4]  rpart    (M <= 32) fp32 partials of the rank-r down-projection, added by the
//                 few-token kernels' last launch (RankFold, FewTokTail)
// The rank-r products reduce inside their clusters and need no scratch.
// ---------------------------------------------------------------------------------------------
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WsLayout {
  size_t small0, small1, flags, flags_bytes, scratch, scratch_bytes, rpart, rpart_bytes, total;
};

WsLayout ws_layout(int M, int N, int K, int r) {
  WsLayout L;
  const size_t small = align256(static_cast<size_t>(M) * r * 2);
  const size_t gemm = std::max(gemm_ws_bytes(M, N, K, r, false), gemm_ws_bytes(M, N, K, r, true));
  L.small0 = 0;
  L.small1 = small;
  L.flags = 2 * small;
  L.flags_bytes = align256(gemm_rank_flag_bytes(M));
  L.scratch = L.flags + L.flags_bytes;
  L.scratch_bytes = align256(gemm);
  // Few tokens: the down-projection's second-level partials, left for the few-token kernels'
  // last launch to add (one row tile; at most one cluster per SM, up to kGemmMaxCtas).
  L.rpart = L.scratch + L.scratch_bytes;
  L.rpart_bytes =
      M <= kGemvMaxTokens ? align256(static_cast<size_t>(kGemmMaxCtas) * 128 * r * 4) : 0;
  L.total = L.rpart + L.rpart_bytes;
  return L;
}

// A single-adapter layer of rank r that is not a multiple of 8 runs at rp = r rounded up to 8
// (the TMA operands need rows of a multiple of 16 bytes) on zero-padded copies kept after the
// layer's own workspace: A [rp, K], B [N, rp], XA [M, rp], and the gradients dA [rp, K] and
// dB [N, rp] in fp32, copied back into the caller's [r, K] / [N, r].
int pad8(int r) { return (r + 7) / 8 * 8; }

struct PadLayout {
  size_t inner, a, b, xa, da, db, total;
};

PadLayout pad_layout(int M, int N, int K, int r) {
  PadLayout P;
  const size_t rp = static_cast<size_t>(pad8(r));
  P.inner = ws_layout(M, N, K, static_cast<int>(rp)).total;
  P.a = P.inner;
  P.b = P.a + align256(rp * K * 2);
  P.xa = P.b + align256(static_cast<size_t>(N) * rp * 2);
  P.da = P.xa + align256(static_cast<size_t>(M) * rp * 2);
  P.db = P.da + align256(rp * K * 4);
  P.total = P.db + align256(static_cast<size_t>(N) * rp * 4);
  return P;
}

// A [r, K] -> ap [rp, K] and B [N, r] -> bp [N, rp], zero elsewhere.
qlora_status pad_factors(const void* A, const void* B, int r, int rp, int N, int K, void* ap,
                         void* bp, cudaStream_t s) {
  if (cudaMemsetAsync(ap, 0, static_cast<size_t>(rp) * K * 2, s) != cudaSuccess ||
      cudaMemcpyAsync(ap, A, static_cast<size_t>(r) * K * 2, cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess ||
      cudaMemsetAsync(bp, 0, static_cast<size_t>(N) * rp * 2, s) != cudaSuccess ||
      cudaMemcpy2DAsync(bp, rp * 2ull, B, r * 2ull, r * 2ull, N, cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

// The rank-r down-projection a dequant GEMM launch computes itself (see GemmArgs::fuse).
struct RankFusion {
  const void* w;      // forward: A [n r, K]; dX: B [N, r]
  int cols, r;        // n r, r
  RowGroups groups;   // dX: the adapters along N
  void* saved;        // [M, n r] bf16 or null
  void* scaled;       // [M, n r] bf16: the GEMM's extension operand
  float scale;
  unsigned* flags;    // workspace counters, zeroed here before the launch
  size_t flag_bytes;
};

GemmArgs gemm_args(const qlora_nf4_weight* W, int M, int r, const RowGroups& groups, bool trans,
                   void* out, int* err, int sms, bool fused = false) {
  GemmArgs a;
  a.M = M;
  a.rows_w = trans ? W->K : W->N;
  a.kt = (trans ? W->N : W->K) / 64;
  a.r_pad16 = (r + 15) / 16 * 16;
  a.n_ext = (a.r_pad16 + 63) / 64;
  const GemmTile tl = gemm_pick_tile(M, a.rows_w, a.kt + a.n_ext, sms, fused);
  a.bt = tl.bt;
  a.nh = tl.nh;
  a.kblocks = W->K / 64;
  a.N = W->N;
  a.dq = W->double_quant ? 1 : 0;
  a.absmax = W->absmax;
  a.absmax_q8 = W->absmax_q8;
  a.absmax_scale = W->absmax_scale;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.err = err;
  a.partial = nullptr;
  a.streamk = 0;
  a.groups = groups;
  a.cb = codebook();
  a.fuse = 0;
  a.rank_cols = 0;
  a.rank_r = 0;
  a.rank_groups = single_group(64);
  a.rank_w = nullptr;
  a.rank_saved = nullptr;
  a.rank_scaled = nullptr;
  a.rank_scale = 0.f;
  a.rank_flags = nullptr;
  a.rank_slot = 0;
  a.sm_limit = 0;
  a.glu_out = nullptr;
  a.glu_I = 0;
  return a;
}

// Maps for the dequant GEMM.  act: [M, red] bf16; ext_act: [M, n, r] bf16 (scaled rank-r
// term of n adapters; n = 1 for dX, whose extension runs over all n r columns at once).
qlora_status gemm_maps(GemmMaps* m, const qlora_nf4_weight* W, bool trans, const void* act,
                       const void* ext_w, const void* ext_act, int M, int r, int n_groups,
                       int bt) {
  const uint64_t red = trans ? W->N : W->K;
  qlora_status st;
  st = encode_2d(&m->act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, red, M, red * 2, 64, bt,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QLORA_OK) return st;
  if (!trans)
    st = encode_2d(&m->q, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->q, W->K / 2, W->N, W->K / 2, 32, 128,
                   CU_TENSOR_MAP_SWIZZLE_32B);
  else
    st = encode_2d(&m->q, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->q, W->K / 2, W->N, W->K / 2, 64, 64,
                   CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != QLORA_OK) return st;
  if (r == 0) {  // no extension steps: the kernel never loads through these, only prefetches
    m->ext_w = m->act;
    m->ext_act = m->act;
    return QLORA_OK;
  }
  if (!trans)  // B_lora [N, r]
    st = encode_2d(&m->ext_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ext_w, r, W->N, r * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  else  // A_lora [r, K]
    st = encode_2d(&m->ext_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ext_w, W->K, r, W->K * 2, 64, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QLORA_OK) return st;
  return encode_3d_bf16(&m->ext_act, ext_act, r, trans ? 1 : n_groups, M, 64, bt);
}

qlora_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

std::atomic<uint64_t> g_launches{0};
// Whether the layer fuses its rank-r down-projections into the dequant GEMM launches when the
// schedule allows (qlora_set_rank_fusion; off by default: on the 4096-token q_proj step it
// measured slower than the separate launches).
std::atomic<int> g_rank_fusion{0};
void count(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

// ---------------------------------------------------------------------------------------------
// Work beside the dX GEMM.  When the GEMM runs whole tiles, dB and dA can run on a few SMs
// taken from it (gemm_side_sms) while it runs on the rest, on a stream this library
// owns, forked from and joined back to the caller's stream with events (inside a stream
// capture the fork and the join become graph edges).  qlora_set_side_overlap: 0 never,
// 1 (default) when the schedule model expects it to be faster than running them after the
// GEMM, 2 always (with the model's best split) when the GEMM runs whole tiles.
// ---------------------------------------------------------------------------------------------
struct SideExec {
  std::mutex mu;  // one fork/join sequence at a time per device (the events are shared)
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool ready = false, broken = false;
};
SideExec g_side[64];
constexpr double kSideMaxActBytes = 48.0 * 1024 * 1024;  // dY bytes the GEMM keeps in L2
std::mutex g_side_init_mu;
std::atomic<int> g_side_overlap{1};
SideExec* side_exec(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_side_init_mu);
  SideExec& se = g_side[dev];
  if (!se.ready && !se.broken) {
    if (cudaStreamCreateWithFlags(&se.stream, cudaStreamNonBlocking) == cudaSuccess &&
        cudaEventCreateWithFlags(&se.fork, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&se.join, cudaEventDisableTiming) == cudaSuccess)
      se.ready = true;
    else {
      se.broken = true;
      (void)cudaGetLastError();
    }
  }
  return se.ready ? &se : nullptr;
}

// ---------------------------------------------------------------------------------------------
// Stage bodies (validated by their callers).
// ---------------------------------------------------------------------------------------------
// Swizzle enum of a TMA span in bytes (0 = none).
CUtensorMapSwizzle swizzle_of(int span) {
  switch (span) {
    case 32: return CU_TENSOR_MAP_SWIZZLE_32B;
    case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
    case 128: return CU_TENSOR_MAP_SWIZZLE_128B;
    default: return CU_TENSOR_MAP_SWIZZLE_NONE;
  }
}

// groups: the adapters packed along the rows of B (w_rc = false); r is then n r_g.
// scratch / scratch_bytes (nullable / 0): workspace for the few-token split of the reduction.
qlora_status do_lora_down(const void* in, int M, int C, const void* w, bool w_rc, int r,
                          const RowGroups& groups, float scale, void* saved, void* scaled,
                          int* err, cudaStream_t s, void* scratch = nullptr,
                          size_t scratch_bytes = 0, void* fold_part = nullptr,
                          size_t fold_bytes = 0) {
  int sms = 0;
  if (gemm_device_sms(&sms) != cudaSuccess) return QLORA_ERR_CUDA;
  const int rg = w_rc ? r : r / groups.n;
  const RankPlan p = rank_down_plan(M, C, r, rg, w_rc, sms, scratch ? scratch_bytes : 0);
  // fold_part: the same plan, its second-level partials left in fold_part for the consumer to
  // add (no finalize launch); the caller has checked down_foldable.
  if (fold_part && (p.gsplit < 2 || p.part_bytes > fold_bytes)) return QLORA_ERR_WORKSPACE;
  RankMaps maps;
  qlora_status st = encode_2d(&maps.big, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, in, C, M, C * 2ull,
                              64, p.box_rows_in, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QLORA_OK) return st;
  if (w_rc)  // A [r, C]: box {64 columns, r rows}
    st = encode_2d(&maps.small, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, C, r, C * 2ull, 64, r,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  else  // B [C, rg]: box {box_w, 64 or 256 rows}
    st = encode_2d(&maps.small, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, rg, C, rg * 2ull,
                   p.small.box_w, p.box_rows_w, swizzle_of(p.small.swizzle));
  if (st != QLORA_OK) return st;
  const cudaError_t e = launch_rank_down(
      maps, p, M, C, r, rg, w_rc, groups, scale, static_cast<__nv_bfloat16*>(saved),
      static_cast<__nv_bfloat16*>(scaled), err, s,
      static_cast<float*>(fold_part ? fold_part : scratch), fold_part == nullptr);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  count(p.gsplit > 1 && !fold_part ? 2 : 1);
  return QLORA_OK;
}

// Whether do_lora_down of this shape can leave its partials for the consumer (fold_part): the
// plan do_lora_down takes with scratch_bytes splits the reduction over clusters (gsplit > 1)
// into a single row tile, and the partials fit fold_bytes.
bool down_foldable(int M, int C, int r, int rg, bool w_rc, int sms, size_t scratch_bytes,
                   size_t fold_bytes, int* gsplit) {
  const RankPlan p = rank_down_plan(M, C, r, rg, w_rc, sms, scratch_bytes);
  *gsplit = p.gsplit;
  return M <= 128 && r <= kFoldMaxR && !p.rows && p.gsplit > 1 && p.part_bytes <= fold_bytes;
}

// `partial` / `partial_bytes`: scratch for the stream-K partial sums (whole tiles if too small).
// groups (forward only): adapters packed along W0's rows, each with r columns of ext_act.
// SwiGLU output of a packed gate/up forward (GemmArgs::glu_out): a [M, I] bf16.
struct GluOut {
  void* a;
  int I;
};

qlora_status do_gemm(const void* act, const qlora_nf4_weight* W, bool trans, const void* ext_w,
                     const void* ext_act, int M, int r, const RowGroups& groups, void* out,
                     int* err, void* partial, size_t partial_bytes, cudaStream_t s,
                     const RankFusion* fuse = nullptr, int sm_limit = 0,
                     const RankFold* fold = nullptr, const FewTokTail* tail = nullptr,
                     const GluOut* glu = nullptr) {
  // fold (few-token forward) / tail (few-token dX): the few-token kernels' last launch adds the
  // down-projection's partials itself (the caller has checked that those kernels apply).
  if (!trans && M <= kGemvMaxTokens && partial) {
    // Few tokens: the register-direct kernel streams the weight without the tcgen05 rings.
    const cudaError_t e = launch_nf4_gemv_fwd(
        static_cast<const __nv_bfloat16*>(act), W->q, W->absmax, W->absmax_q8, W->absmax_scale,
        W->double_quant ? 1 : 0, M, W->N, W->K, static_cast<const __nv_bfloat16*>(ext_act),
        static_cast<const __nv_bfloat16*>(ext_w), r, groups, static_cast<__nv_bfloat16*>(out),
        static_cast<float*>(partial), partial_bytes / 4, codebook(), s, fold);
    if (e == cudaSuccess) {
      count(2);
      return QLORA_OK;
    }
    // cudaErrorInvalidValue: the scratch is too small for its partials (nothing was launched,
    // so no error is pending); use the tcgen05 kernel instead.
    if (e != cudaErrorInvalidValue || fold) return QLORA_ERR_CUDA;
  }
  int sms = 0;
  if (gemm_device_sms(&sms) != cudaSuccess) return QLORA_ERR_CUDA;
  if (trans && M <= kFewTokDxMaxTokens && partial && !fuse) {
    // Few tokens: dX streams the weight panel by panel without the tcgen05 rings' hand-offs.
    const FewTokDxPlan fp = fewtok_dx_plan(M, W->N, W->K, sms);
    if (fp.part_bytes <= partial_bytes) {
      CUtensorMap mq, md;
      qlora_status st = encode_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->q, W->K / 2, W->N,
                                  W->K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B);
      if (st != QLORA_OK) return st;
      st = encode_2d(&md, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, W->N, M, W->N * 2ull, 64,
                     16 * fp.mb, CU_TENSOR_MAP_SWIZZLE_128B);
      if (st != QLORA_OK) return st;
      // fp32 block scales [N, K/64] in boxes of 4 blocks x 64 rows (rows of K/64 * 4 bytes:
      // a multiple of 16 when K % 256 == 0).
      CUtensorMap ma;
      const bool am_tma = !W->double_quant && W->K % 256 == 0 && aligned16(W->absmax);
      if (am_tma && (st = encode_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, W->absmax, W->K / 64,
                                    W->N, (W->K / 64) * 4ull, 4, 64,
                                    CU_TENSOR_MAP_SWIZZLE_NONE)) != QLORA_OK)
        return st;
      const cudaError_t e = launch_nf4_fewtok_dx(
          mq, md, am_tma ? &ma : nullptr, fp, M, W->N, W->K, W->absmax, W->absmax_q8, W->absmax_scale,
          W->double_quant ? 1 : 0, static_cast<const __nv_bfloat16*>(ext_act),
          static_cast<const __nv_bfloat16*>(ext_w), r, static_cast<__nv_bfloat16*>(out),
          static_cast<float*>(partial), partial_bytes, codebook(), err, s, tail == nullptr);
      if (e != cudaSuccess) return QLORA_ERR_CUDA;
      if (tail &&
          launch_fewtok_bwd_tail(*tail, static_cast<float*>(partial), fp.splits, M, W->N, W->K,
                                 static_cast<__nv_bfloat16*>(out), s) != cudaSuccess)
        return QLORA_ERR_CUDA;
      count(2);
      return QLORA_OK;
    }
  }
  if (tail) return QLORA_ERR_WORKSPACE;  // the caller checked the few-token plan fits
  if (sm_limit > 0 && sm_limit < sms && !fuse) sms = sm_limit;
  else sm_limit = 0;
  GemmArgs a = gemm_args(W, M, r, groups, trans, out, err, sms, fuse != nullptr);
  a.partial = static_cast<float*>(partial);
  a.sm_limit = sm_limit;
  if (glu) {  // the caller checked gemm_glu_ok
    a.glu_out = static_cast<__nv_bfloat16*>(glu->a);
    a.glu_I = glu->I;
  }
  GemmMaps maps;
#ifdef QLORA_CTA_PAIRS
  if (!fuse && !sm_limit && gemm2_applies(M, a.rows_w, a.kt + a.n_ext, sms, groups)) {
    // Enough whole tiles for every SM pair: M = 256 MMAs over CTA pairs (each CTA loads half of
    // every activation block, so the tensor maps' boxes are bt / 2 tokens high).
    const GemmTile t2 = gemm2_pick_tile(M, a.rows_w, a.kt + a.n_ext, sms);
    a.bt = t2.bt;
    a.nh = t2.nh;
    qlora_status st = gemm_maps(&maps, W, trans, act, ext_w, ext_act, M, r, groups.n, a.bt / 2);
    if (st != QLORA_OK) return st;
    int launched = 0;
    const cudaError_t e = launch_qlora_gemm2(trans, maps, a, s, &launched);
    count(launched);
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  }
#endif
  qlora_status st = gemm_maps(&maps, W, trans, act, ext_w, ext_act, M, r, groups.n, a.bt);
  if (st != QLORA_OK) return st;
  maps.rank = maps.act;  // never read unless fused
  if (fuse) {
    a.rank_slot = gemm_rank_slot_bytes(trans, fuse->cols, fuse->r);
    if (!trans)  // A [n r, K]: box {64 columns, n r rounded up to 16 rows (zero fill)}
      st = encode_2d(&maps.rank, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, fuse->w, W->K, fuse->cols,
                     W->K * 2ull, 64, (fuse->cols + 15) / 16 * 16, CU_TENSOR_MAP_SWIZZLE_128B);
    else  // B [N, r]: box {r columns, 64 rows}
      st = encode_2d(&maps.rank, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, fuse->w, fuse->r, W->N,
                     fuse->r * 2ull, fuse->r, 64, swizzle_of(fuse->r * 2));
    if (st != QLORA_OK) return st;
    a.fuse = 1;
    a.rank_cols = fuse->cols;
    a.rank_r = fuse->r;
    a.rank_groups = fuse->groups;
    a.rank_w = static_cast<const __nv_bfloat16*>(fuse->w);
    a.rank_saved = static_cast<__nv_bfloat16*>(fuse->saved);
    a.rank_scaled = static_cast<__nv_bfloat16*>(fuse->scaled);
    a.rank_scale = fuse->scale;
    a.rank_flags = fuse->flags;
    if (cudaMemsetAsync(fuse->flags, 0, fuse->flag_bytes, s) != cudaSuccess) return QLORA_ERR_CUDA;
  }
  int launched = 0;
  const cudaError_t e = launch_qlora_gemm(trans, maps, a, partial ? partial_bytes / 4 : 0, s,
                                          &launched);
  count(launched);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// Tensor maps of one rank-r gradient: big [M, C] in boxes of {64, 64}; small [M, ld] in boxes
// of the plan's small tile.
qlora_status grad_maps(RankMaps* maps, const RankPlan& p, const void* big, int M, int C,
                       const void* small, int ld_small) {
  qlora_status st = encode_2d(&maps->big, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, big, C, M, C * 2ull,
                              64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QLORA_OK) return st;
  return encode_2d(&maps->small, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, small, ld_small, M,
                   ld_small * 2ull, p.small.box_w, 64, swizzle_of(p.small.swizzle));
}

// groups: the adapters packed along the columns of `big`; small is then [M, n r].
qlora_status do_lora_grad(const void* big, int M, int C, const void* small, int r,
                          const RowGroups& groups, float scale, float* out, bool out_cr, int* err,
                          cudaStream_t s) {
  int sms = 0;
  if (gemm_device_sms(&sms) != cudaSuccess) return QLORA_ERR_CUDA;
  const RankPlan p = rank_grad_plan(M, C, r, sms);
  const int ld_small = groups.n * r;
  RankMaps maps;
  qlora_status st = grad_maps(&maps, p, big, M, C, small, ld_small);
  if (st != QLORA_OK) return st;
  const cudaError_t e =
      launch_rank_grad(maps, p, M, C, r, ld_small, groups, scale, out, out_cr, err, s);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  count(1);
  return QLORA_OK;
}

// SMs the dX GEMM of a backward gives to dB and dA (0: they run after it), for W [N, K] with
// n r = R rank columns, under side-overlap mode `mode`.
int side_sms(int M, int N, int K, int R, int sms, int mode) {
  if (mode == 0 || M < 1 || N < 64 || K < 64 || R < 1) return 0;
  // Measured on a B200, where the model alone is too hopeful: with n r > 32 the side kernel is
  // bound by its mma.sync work, not its stream (proj_70b_dq, r = 64: 5.25 -> 8.34 ms per
  // step), and when dY (which the GEMM re-reads once per row tile) is too big to stay in L2 the
  // side stream's DRAM traffic costs the GEMM more than the side saves (mlp_8b +1.5 %, 16384
  // tokens +2.4 %; q_proj, dY 32 MiB: 0.349 -> 0.327 ms).
  if (mode == 1 && (R > 32 || 2.0 * M * N > kSideMaxActBytes)) return 0;
  double us = 0.0;
  // dB streams dY [M, N], dA streams X [M, K].
  const double bytes = 2.0 * M * (static_cast<double>(N) + K);
  return gemm_side_sms(M, K, N / 64 + ext_steps(R), sms, bytes, mode == 2, &us);
}

// dX = dY deq(W0) + (s dYB) A on all but `spare` SMs, with dB_g = s dY_g^T XA_g and
// dA = s dYB^T X on those `spare` SMs at the same time (a side stream forked after dYB).  The
// side kernels sum in the cluster kernels' order, so every output has the bits of the serial
// path.  *done = false when the side stream is unavailable (nothing enqueued).
qlora_status gemm_with_side_grads(const void* dY, const void* X, const void* XA, const void* dYB,
                                  const void* sdYB, const qlora_nf4_weight* W, const void* A,
                                  const RowGroups& g, int M, int r, float scale, void* dX,
                                  float* dA, float* dB, int* err, void* scratch,
                                  size_t scratch_bytes, cudaStream_t s, int dev, int sms,
                                  int spare, bool* done) {
  *done = false;
  SideExec* se = side_exec(dev);
  if (!se) return QLORA_OK;
  const int R = g.n * r, N = W->N, K = W->K;
  const RankPlan pB = rank_grad_plan(M, N, r, sms);
  const RankPlan pA = rank_grad_plan(M, K, R, sms);
  RankMaps mB, mA;
  qlora_status st = grad_maps(&mB, pB, dY, M, N, XA, R);
  if (st != QLORA_OK) return st;
  if ((st = grad_maps(&mA, pA, X, M, K, dYB, R)) != QLORA_OK) return st;
  std::lock_guard<std::mutex> lk(se->mu);
  if (cudaEventRecord(se->fork, s) != cudaSuccess ||
      cudaStreamWaitEvent(se->stream, se->fork, 0) != cudaSuccess)
    return QLORA_ERR_CUDA;
  *done = true;
  cudaError_t e;
  if (r == R) {  // one launch: both problems share the kernel instance
    e = launch_rank_grad_side(mB, pB, M, N, r, R, g, dB, true, &mA, &pA, K, R, R,
                              single_group(K), dA, false, scale, err, spare, se->stream);
    if (e == cudaSuccess) count(1);
  } else {
    e = launch_rank_grad_side(mB, pB, M, N, r, R, g, dB, true, nullptr, nullptr, 0, 0, 0, g,
                              nullptr, false, scale, err, spare, se->stream);
    if (e == cudaSuccess) {
      count(1);
      e = launch_rank_grad_side(mA, pA, M, K, R, R, single_group(K), dA, false, nullptr, nullptr,
                                0, 0, 0, g, nullptr, false, scale, err, spare, se->stream);
      if (e == cudaSuccess) count(1);
    }
  }
  st = e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  if (st == QLORA_OK)
    st = do_gemm(dY, W, true, A, sdYB, M, R, single_group(K), dX, err, scratch, scratch_bytes, s,
                 nullptr, sms - spare);
  // Join whatever was enqueued, so the caller's stream (or capture) waits for the side work.
  if (cudaEventRecord(se->join, se->stream) != cudaSuccess ||
      cudaStreamWaitEvent(s, se->join, 0) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return st;
}

// dB = s dY^T XA (per adapter) and dA = s dYB^T X of one backward, in one launch when their
// plans match (single adapter), else one after the other.
qlora_status do_weight_grads(const void* dY, const void* X, const void* XA, const void* dYB,
                             int M, int N, int K, int r, const RowGroups& g, float scale,
                             float* dA, float* dB, int* err, cudaStream_t s) {
  const int R = g.n * r;
  int sms = 0;
  if (gemm_device_sms(&sms) != cudaSuccess) return QLORA_ERR_CUDA;
  const RankPlan pB = rank_grad_plan(M, N, r, sms);
  const RankPlan pA = rank_grad_plan(M, K, R, sms);
  if (!rank_grad_pair_ok(pB, r, pA, R)) {
    qlora_status st = do_lora_grad(dY, M, N, XA, r, g, scale, dB, true, err, s);
    if (st != QLORA_OK) return st;
    return do_lora_grad(X, M, K, dYB, R, single_group(K), scale, dA, false, err, s);
  }
  RankMaps mB, mA;
  qlora_status st = grad_maps(&mB, pB, dY, M, N, XA, R);
  if (st != QLORA_OK) return st;
  if ((st = grad_maps(&mA, pA, X, M, K, dYB, R)) != QLORA_OK) return st;
  const cudaError_t e = launch_rank_grad_pair(mB, pB, M, N, r, R, g, dB, true, mA, pA, K, R,
                                              single_group(K), dA, false, scale, err, s);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  count(1);
  return QLORA_OK;
}

// ---------------------------------------------------------------------------------------------
// The layer over n adapters packed along W0's rows (n = 1: a single adapter).  W is
// [N = sum N_g, K]; A [n r, K] stacks A_g; B [N, r] stacks B_g; XA_saved, dA and the packed
// rank-r operands are [M, n r] / [n r, K]; dB is [N, r]; s = alpha / r for every adapter.
// The caller has checked W and built `g`.
// ---------------------------------------------------------------------------------------------
// `scale` is alpha / r of the caller's rank (the padded-rank path passes r rounded up).
qlora_status linear_fwd(const void* X, const qlora_nf4_weight* W, const void* A, const void* B,
                        const RowGroups& g, int M, int r, float scale, void* H, void* XA_saved,
                        void* ws, size_t ws_bytes, cudaStream_t s,
                        const GluOut* glu = nullptr) {
  if (!X || !A || !B || !H) return QLORA_ERR_NULL;
  const int R = g.n * r;
  if (M < 1 || !rank_ok(r) || !rank_ok(R)) return QLORA_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(H) ||
      (XA_saved && !aligned16(XA_saved)))
    return QLORA_ERR_ALIGN;
  const WsLayout L = ws_layout(M, W->N, W->K, R);
  if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  int dev;
  qlora_status st;
  if ((st = current_device(&dev)) != QLORA_OK) return st;
  int* err;
  if ((st = error_word_ptr(dev, &err)) != QLORA_OK) return st;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  auto* sxa = reinterpret_cast<__nv_bfloat16*>(w8 + L.small0);

  // XA = X A^T [M, n r] (saved in bf16 unless XA_saved is NULL) and s * XA: every adapter's
  // down-projection in one pass over X -- inside the GEMM launch below when its schedule allows
  // (whole tiles: the GEMM streams every X tile anyway), else as a launch of its own.
  int sms = 0;
  if (gemm_device_sms(&sms) != cudaSuccess) return QLORA_ERR_CUDA;
  if (!glu && g_rank_fusion.load(std::memory_order_relaxed) && M > kGemvMaxTokens &&
      gemm_rank_fusable(M, W->N, W->K / 64 + ext_steps(r), sms, R,
                                              gemm_rank_slot_bytes(false, R, r))) {
    const RankFusion f{A, R, r, single_group(W->K), XA_saved, sxa, scale,
                       reinterpret_cast<unsigned*>(w8 + L.flags), L.flags_bytes};
    return do_gemm(X, W, false, B, sxa, M, r, g, H, err, w8 + L.scratch, L.scratch_bytes, s, &f);
  }
  // Few tokens: the few-token kernel's finalize adds X A^T's partials itself and writes the
  // saved XA (one launch fewer; the same bits).
  int gsplit = 0;
  if (M <= kGemvMaxTokens &&
      gemv_plan(M, W->N, W->K, std::min(sms, kGemmMaxCtas)).partial_floats * 4 <=
          L.scratch_bytes &&
      down_foldable(M, W->K, R, R, true, sms, L.scratch_bytes, L.rpart_bytes, &gsplit)) {
    st = do_lora_down(X, M, W->K, A, true, R, single_group(W->K), scale, nullptr, nullptr, err, s,
                      w8 + L.scratch, L.scratch_bytes, w8 + L.rpart, L.rpart_bytes);
    if (st != QLORA_OK) return st;
    const RankFold f{reinterpret_cast<const float*>(w8 + L.rpart), gsplit, R, scale,
                     static_cast<__nv_bfloat16*>(XA_saved)};
    return do_gemm(X, W, false, B, sxa, M, r, g, H, err, w8 + L.scratch, L.scratch_bytes, s,
                   nullptr, 0, &f);
  }
  // (The GEMM's scratch is free until the GEMM runs: the few-token split uses it first.)
  st = do_lora_down(X, M, W->K, A, true, R, single_group(W->K), scale, XA_saved, sxa, err, s,
                    w8 + L.scratch, L.scratch_bytes);
  if (st != QLORA_OK) return st;
  // h = X deq(W0)^T + (s XA_g) B_g^T for the rows of each adapter g, in one launch.
  return do_gemm(X, W, false, B, sxa, M, r, g, H, err, w8 + L.scratch, L.scratch_bytes, s,
                 nullptr, 0, nullptr, nullptr, glu);
}

qlora_status linear_bwd(const void* dY, const void* X, const qlora_nf4_weight* W, const void* A,
                        const void* B, const void* XA_saved, const RowGroups& g, int M, int r,
                        float scale, void* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                        cudaStream_t s) {
  if (!dY || !X || !A || !B || !dA || !dB) return QLORA_ERR_NULL;
  const int R = g.n * r;
  if (M < 1 || !rank_ok(r) || !rank_ok(R)) return QLORA_ERR_SHAPE;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(A) || !aligned16(B) ||
      (XA_saved && !aligned16(XA_saved)) || !aligned16(dA) || !aligned16(dB) ||
      (dX && !aligned16(dX)))
    return QLORA_ERR_ALIGN;
  const WsLayout L = ws_layout(M, W->N, W->K, R);
  if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  int dev;
  qlora_status st;
  if ((st = current_device(&dev)) != QLORA_OK) return st;
  int* err;
  if ((st = error_word_ptr(dev, &err)) != QLORA_OK) return st;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  auto* dyb = reinterpret_cast<__nv_bfloat16*>(w8 + L.small0);
  auto* sdyb = reinterpret_cast<__nv_bfloat16*>(w8 + L.small1);
  float* scratch = reinterpret_cast<float*>(w8 + L.scratch);

  // Few tokens: dY B left as partials, the few-token dX kernel, and one last launch that adds
  // the partials and computes dX, dA and dB (XA recomputed first when it was not saved, with
  // the forward's own plan, so the same bits).
  {
    int fsms = 0, gsplit = 0;
    if (gemm_device_sms(&fsms) != cudaSuccess) return QLORA_ERR_CUDA;
    if (M <= kFewTokDxMaxTokens &&
        (!dX || fewtok_dx_plan(M, W->N, W->K, fsms).part_bytes <= L.scratch_bytes) &&
        down_foldable(M, W->N, R, r, false, fsms, L.scratch_bytes, L.rpart_bytes, &gsplit)) {
      const void* xa = XA_saved;
      if (!xa) {
        st = do_lora_down(X, M, W->K, A, true, R, single_group(W->K), scale, dyb, sdyb, err, s,
                          scratch, L.scratch_bytes);
        if (st != QLORA_OK) return st;
        xa = dyb;
      }
      st = do_lora_down(dY, M, W->N, B, false, R, g, scale, nullptr, nullptr, err, s, scratch,
                        L.scratch_bytes, w8 + L.rpart, L.rpart_bytes);
      if (st != QLORA_OK) return st;
      FewTokTail t;
      t.fold = RankFold{reinterpret_cast<const float*>(w8 + L.rpart), gsplit, R, scale, nullptr};
      t.X = static_cast<const __nv_bfloat16*>(X);
      t.dY = static_cast<const __nv_bfloat16*>(dY);
      t.XA = static_cast<const __nv_bfloat16*>(xa);
      t.A = static_cast<const __nv_bfloat16*>(A);
      t.groups = g;
      t.r = r;
      t.dA = dA;
      t.dB = dB;
      if (dX)
        return do_gemm(dY, W, true, A, sdyb, M, R, single_group(W->K), dX, err, scratch,
                       L.scratch_bytes, s, nullptr, 0, nullptr, &t);
      if (launch_fewtok_bwd_tail(t, nullptr, 0, M, W->N, W->K, nullptr, s) != cudaSuccess)
        return QLORA_ERR_CUDA;
      count(1);
      return QLORA_OK;
    }
  }
  // Without a saved XA, recompute it from X (the forward's own kernel on the same inputs, so
  // bit for bit the value it would have saved) and take dB first, while small0 holds it.
  if (!XA_saved) {
    st = do_lora_down(X, M, W->K, A, true, R, single_group(W->K), scale, dyb, sdyb, err, s,
                      scratch, L.scratch_bytes);
    if (st != QLORA_OK) return st;
    st = do_lora_grad(dY, M, W->N, dyb, r, g, scale, dB, true, err, s);
    if (st != QLORA_OK) return st;
  }
  // dYB = dY B_bd [M, n r] (bf16, for dA) and s * dYB, B_bd the block-diagonal of the B_g --
  // inside the dX launch when its schedule allows, else as a launch of its own.
  // dX = dY deq(W0) + (s dYB) A: one extension over all n r columns sums the adapters' terms.
  int sms = 0;
  if (gemm_device_sms(&sms) != cudaSuccess) return QLORA_ERR_CUDA;
  if (dX && g_rank_fusion.load(std::memory_order_relaxed) &&
      gemm_rank_fusable(M, W->K, W->N / 64 + ext_steps(R), sms, R,
                              gemm_rank_slot_bytes(true, R, r))) {
    const RankFusion f{B, R, r, g, dyb, sdyb, scale, reinterpret_cast<unsigned*>(w8 + L.flags),
                       L.flags_bytes};
    st = do_gemm(dY, W, true, A, sdyb, M, R, single_group(W->K), dX, err, scratch,
                 L.scratch_bytes, s, &f);
    if (st != QLORA_OK) return st;
  } else {
    st = do_lora_down(dY, M, W->N, B, false, R, g, scale, dyb, sdyb, err, s, scratch,
                      L.scratch_bytes);
    if (st != QLORA_OK) return st;
    const int spare = (dX && XA_saved)
                          ? side_sms(M, W->N, W->K, R, sms,
                                     g_side_overlap.load(std::memory_order_relaxed))
                          : 0;
    if (spare > 0) {
      bool done = false;
      st = gemm_with_side_grads(dY, X, XA_saved, dyb, sdyb, W, A, g, M, r, scale, dX, dA, dB, err,
                                scratch, L.scratch_bytes, s, dev, sms, spare, &done);
      if (st != QLORA_OK || done) return st;
    }
    if (dX && (st = do_gemm(dY, W, true, A, sdyb, M, R, single_group(W->K), dX, err, scratch,
                            L.scratch_bytes, s)) != QLORA_OK)
      return st;
  }
  // dB_g = s dY_g^T XA_g  [N, r];  dA = s dYB^T X  [n r, K] (one launch when they match).
  if (XA_saved)
    return do_weight_grads(dY, X, XA_saved, dyb, M, W->N, W->K, r, g, scale, dA, dB, err, s);
  return do_lora_grad(X, M, W->K, dyb, R, single_group(W->K), scale, dA, false, err, s);
}

}  // namespace
}  // namespace qlora

// ---------------------------------------------------------------------------------------------
// Fixed scratch for qlora_linear_fwd_noalloc: a file-scope device array, so that entry point
// needs no caller-provided workspace and allocates nothing.  Every GPU that loads this library
// holds the array until the process exits.  In host code the name is only a host-side stand-in
// for the device symbol; kernels get its device address, looked up once per device with that
// device current (cudaGetSymbolAddress).
// ---------------------------------------------------------------------------------------------
namespace qlora {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices];

qlora_status noalloc_scratch(int dev, void** p) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_noalloc_scratch) != cudaSuccess || !a) return QLORA_ERR_CUDA;
    g_noalloc_ptr[dev] = a;
  }
  *p = g_noalloc_ptr[dev];
  return QLORA_OK;
}
}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" {

const char* qlora_status_str(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_NULL: return "null pointer";
    case QLORA_ERR_SHAPE: return "bad shape";
    case QLORA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QLORA_ERR_ARCH: return "device is not sm_100 (B200)";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "a bounded device wait ran out";
  }
  return "unknown status";
}

qlora_status qlora_nf4_codebook(float out[16]) {
  if (!out) return QLORA_ERR_NULL;
  const Codebook& cb = codebook();
  for (int i = 0; i < 16; ++i) out[i] = cb.level[i];
  return QLORA_OK;
}

qlora_status qlora_nf4_pack(const void* W, int N, int K, int double_quant, uint8_t* q,
                            float* absmax, uint8_t* absmax_q8, float* absmax_scale,
                            qlora_stream_t stream) {
  if (!W || !q || !absmax) return QLORA_ERR_NULL;
  if (double_quant && (!absmax_q8 || !absmax_scale)) return QLORA_ERR_NULL;
  if (N < 1 || K < 64 || (K % 64)) return QLORA_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(q) || !aligned16(absmax) ||
      (double_quant && (!aligned16(absmax_q8) || !aligned16(absmax_scale))))
    return QLORA_ERR_ALIGN;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_nf4_pack(static_cast<const __nv_bfloat16*>(W), N, K,
                                   double_quant ? 1 : 0, q, absmax, absmax_q8, absmax_scale,
                                   codebook(), static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(double_quant ? 3 : 1);
  return st;
}

qlora_status qlora_nf4_dequant(const qlora_nf4_weight* W, void* Wd, qlora_stream_t stream) {
  if (!W || !W->q || !Wd) return QLORA_ERR_NULL;
  if (W->double_quant ? (!W->absmax_q8 || !W->absmax_scale) : !W->absmax) return QLORA_ERR_NULL;
  if (W->N < 1 || W->K < 64 || (W->K % 64)) return QLORA_ERR_SHAPE;
  if (!aligned16(W->q) || !aligned16(Wd)) return QLORA_ERR_ALIGN;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_nf4_dequant(W->q, W->absmax, W->absmax_q8, W->absmax_scale,
                                      W->double_quant ? 1 : 0, W->N, W->K,
                                      static_cast<__nv_bfloat16*>(Wd), codebook(),
                                      static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

size_t qlora_workspace_bytes(int M, int N, int K, int r) {
  if (M < 1 || N < 64 || K < 64 || r < 1 || r > 128) return 0;
  if (rank_ok(r)) return ws_layout(M, N, K, r).total;
  return pad_layout(M, N, K, r).total;
}

qlora_status qlora_linear_fwd(const void* X, const qlora_nf4_weight* W, const void* A,
                              const void* B, int M, int r, float alpha, void* H, void* XA_saved,
                              void* ws, size_t ws_bytes, qlora_stream_t stream) {
  qlora_status st = check_weight(W);
  if (st != QLORA_OK) return st;
  const float scale = alpha / static_cast<float>(r);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (r < 1 || r > 128 || rank_ok(r))
    return linear_fwd(X, W, A, B, single_group(W->N), M, r, scale, H, XA_saved, ws, ws_bytes, s);
  // r not a multiple of 8: the layer runs at r rounded up to 8 on zero-padded copies.  (Every
  // check the inner call makes on the caller's buffers is made here first, so nothing is
  // enqueued before an error.)
  if (!X || !A || !B || !H) return QLORA_ERR_NULL;
  if (M < 1) return QLORA_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(H)) return QLORA_ERR_ALIGN;
  const PadLayout P = pad_layout(M, W->N, W->K, r);
  if (!ws || ws_bytes < P.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int rp = pad8(r);
  if ((st = pad_factors(A, B, r, rp, W->N, W->K, w8 + P.a, w8 + P.b, s)) != QLORA_OK) return st;
  void* xap = XA_saved ? w8 + P.xa : nullptr;
  st = linear_fwd(X, W, w8 + P.a, w8 + P.b, single_group(W->N), M, rp, scale, H, xap, ws, P.inner,
                  s);
  if (st != QLORA_OK || !XA_saved) return st;
  return cuda_status(cudaMemcpy2DAsync(XA_saved, r * 2ull, xap, rp * 2ull, r * 2ull, M,
                                       cudaMemcpyDeviceToDevice, s));
}

qlora_status qlora_linear_bwd(const void* dY, const void* X, const qlora_nf4_weight* W,
                              const void* A, const void* B, const void* XA_saved, int M, int r,
                              float alpha, void* dX, float* dA, float* dB, void* ws,
                              size_t ws_bytes, qlora_stream_t stream) {
  qlora_status st = check_weight(W);
  if (st != QLORA_OK) return st;
  const float scale = alpha / static_cast<float>(r);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (r < 1 || r > 128 || rank_ok(r))
    return linear_bwd(dY, X, W, A, B, XA_saved, single_group(W->N), M, r, scale, dX, dA, dB, ws,
                      ws_bytes, s);
  // r not a multiple of 8: zero-padded copies of A, B and XA at r rounded up to 8; dA and dB
  // come back from padded buffers (their extra rows / columns are zero).
  if (!dY || !X || !A || !B || !dA || !dB) return QLORA_ERR_NULL;
  if (M < 1) return QLORA_ERR_SHAPE;
  if (!aligned16(dY) || !aligned16(X) || (dX && !aligned16(dX))) return QLORA_ERR_ALIGN;
  const PadLayout P = pad_layout(M, W->N, W->K, r);
  if (!ws || ws_bytes < P.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int rp = pad8(r);
  if ((st = pad_factors(A, B, r, rp, W->N, W->K, w8 + P.a, w8 + P.b, s)) != QLORA_OK) return st;
  void* xap = nullptr;
  if (XA_saved) {
    xap = w8 + P.xa;
    if (cudaMemsetAsync(xap, 0, static_cast<size_t>(M) * rp * 2, s) != cudaSuccess ||
        cudaMemcpy2DAsync(xap, rp * 2ull, XA_saved, r * 2ull, r * 2ull, M,
                          cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return QLORA_ERR_CUDA;
  }
  auto* dap = reinterpret_cast<float*>(w8 + P.da);
  auto* dbp = reinterpret_cast<float*>(w8 + P.db);
  st = linear_bwd(dY, X, W, w8 + P.a, w8 + P.b, xap, single_group(W->N), M, rp, scale, dX, dap,
                  dbp, ws, P.inner, s);
  if (st != QLORA_OK) return st;
  if (cudaMemcpyAsync(dA, dap, static_cast<size_t>(r) * W->K * 4, cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess ||
      cudaMemcpy2DAsync(dB, r * 4ull, dbp, rp * 4ull, r * 4ull, W->N, cudaMemcpyDeviceToDevice,
                        s) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

size_t qlora_grouped_workspace_bytes(int M, int N, int K, int r, int n_groups) {
  if (M < 1 || N < 64 || K < 64 || n_groups < 1 || n_groups > kMaxGroups || !rank_ok(r) ||
      !rank_ok(n_groups * r))
    return 0;
  return ws_layout(M, N, K, n_groups * r).total;
}

qlora_status qlora_grouped_fwd(const void* X, const qlora_nf4_weight* W, const void* A,
                               const void* B, const int* group_rows, int n_groups, int M, int r,
                               float alpha, void* H, void* XA_saved, void* ws, size_t ws_bytes,
                               qlora_stream_t stream) {
  qlora_status st = check_weight(W);
  if (st != QLORA_OK) return st;
  RowGroups g;
  if ((st = make_groups(group_rows, n_groups, W->N, r, &g)) != QLORA_OK) return st;
  return linear_fwd(X, W, A, B, g, M, r, alpha / static_cast<float>(r), H, XA_saved, ws,
                    ws_bytes,
                    static_cast<cudaStream_t>(stream));
}

qlora_status qlora_grouped_fwd_swiglu(const void* X, const qlora_nf4_weight* W, const void* A,
                                      const void* B, int M, int r, float alpha, void* GU,
                                      void* XA_saved, void* act, void* ws, size_t ws_bytes,
                                      qlora_stream_t stream) {
  qlora_status st = check_weight(W);
  if (st != QLORA_OK) return st;
  if (!act) return QLORA_ERR_NULL;
  if (!aligned16(act)) return QLORA_ERR_ALIGN;
  if (W->N < 16 || W->N % 16) return QLORA_ERR_SHAPE;
  const int I = W->N / 2;
  const int rows[2] = {I, I};
  RowGroups g;
  if ((st = make_groups(rows, 2, W->N, r, &g)) != QLORA_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int sms = 0;
  if (gemm_device_sms(&sms) != cudaSuccess) return QLORA_ERR_CUDA;
  const float scale = alpha / static_cast<float>(r);
  if (M > kGemvMaxTokens && rank_ok(r) && gemm_glu_ok(M, I, W->K / 64 + ext_steps(r), sms)) {
    const GluOut glu{act, I};
    return linear_fwd(X, W, A, B, g, M, r, scale, GU, XA_saved, ws, ws_bytes, s, &glu);
  }
  // Otherwise the packed SwiGLU kernel after the layer: the same bits.
  if ((st = linear_fwd(X, W, A, B, g, M, r, scale, GU, XA_saved, ws, ws_bytes, s)) != QLORA_OK)
    return st;
  return qlora_swiglu_packed_fwd(GU, act, M, I, stream);
}

qlora_status qlora_grouped_bwd(const void* dY, const void* X, const qlora_nf4_weight* W,
                               const void* A, const void* B, const void* XA_saved,
                               const int* group_rows, int n_groups, int M, int r, float alpha,
                               void* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                               qlora_stream_t stream) {
  qlora_status st = check_weight(W);
  if (st != QLORA_OK) return st;
  RowGroups g;
  if ((st = make_groups(group_rows, n_groups, W->N, r, &g)) != QLORA_OK) return st;
  return linear_bwd(dY, X, W, A, B, XA_saved, g, M, r, alpha / static_cast<float>(r), dX, dA, dB,
                    ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_lora_down(const void* in, int M, int C, const void* w, int w_is_r_by_c, int r,
                             const int* group_rows, int n_groups, float scale, void* saved,
                             void* scaled, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!in || !w || !scaled) return QLORA_ERR_NULL;
  if (M < 1 || C < 64 || (C % 64) || !rank_ok(r)) return QLORA_ERR_SHAPE;
  RowGroups g = single_group(C);
  if (group_rows) {  // B of n adapters [C, r / n], block-diagonal over the output columns
    if (w_is_r_by_c || n_groups < 1 || r % n_groups) return QLORA_ERR_SHAPE;
    const qlora_status gs = make_groups(group_rows, n_groups, C, r / n_groups, &g);
    if (gs != QLORA_OK) return gs;
  }
  if (!aligned16(in) || !aligned16(w) || !aligned16(scaled) || (saved && !aligned16(saved)))
    return QLORA_ERR_ALIGN;
  if (ws && !aligned16(ws)) return QLORA_ERR_ALIGN;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  int* err;
  if ((st = error_word_ptr(dev, &err)) != QLORA_OK) return st;
  return do_lora_down(in, M, C, w, w_is_r_by_c != 0, r, g, scale, saved, scaled, err,
                      static_cast<cudaStream_t>(stream), ws, ws ? ws_bytes : 0);
}

qlora_status qlora_nf4_gemm(const void* act, const qlora_nf4_weight* W, int transpose_w,
                            const void* ext_w, const void* ext_act, int M, int r,
                            const int* group_rows, int n_groups, void* out, void* ws,
                            size_t ws_bytes, qlora_stream_t stream) {
  if (!act || !out || (r != 0 && (!ext_w || !ext_act))) return QLORA_ERR_NULL;
  qlora_status st = check_weight(W);
  if (st != QLORA_OK) return st;
  if (M < 1 || (r != 0 && !rank_ok(r))) return QLORA_ERR_SHAPE;
  // Without an extension a tile is its reduction steps alone; the dequant groups take two
  // steps at a time, so there must be at least two of them.
  if (r == 0 && (transpose_w ? W->N : W->K) < 128) return QLORA_ERR_SHAPE;
  if (r == 0 && group_rows) return QLORA_ERR_SHAPE;
  RowGroups g = single_group(transpose_w ? W->K : W->N);
  if (group_rows) {  // forward only: adapters along W0's rows, ext_act [M, n, r]
    if (transpose_w) return QLORA_ERR_SHAPE;
    if ((st = make_groups(group_rows, n_groups, W->N, r, &g)) != QLORA_OK) return st;
  }
  if (!aligned16(act) || (ext_w && !aligned16(ext_w)) || (ext_act && !aligned16(ext_act)) ||
      !aligned16(out))
    return QLORA_ERR_ALIGN;
  const size_t need = gemm_ws_bytes(M, W->N, W->K, g.n * r, transpose_w != 0);
  if (need && (!ws || ws_bytes < need)) return QLORA_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return QLORA_ERR_ALIGN;
  int dev;
  if ((st = current_device(&dev)) != QLORA_OK) return st;
  int* err;
  if ((st = error_word_ptr(dev, &err)) != QLORA_OK) return st;
  return do_gemm(act, W, transpose_w != 0, ext_w, ext_act, M, r, g, out, err, ws, ws_bytes,
                 static_cast<cudaStream_t>(stream));
}

qlora_status qlora_lora_grad(const void* big, int M, int C, const void* small, int r,
                             const int* group_rows, int n_groups, float scale, float* out,
                             int out_r_by_c, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!big || !small || !out) return QLORA_ERR_NULL;
  if (M < 1 || C < 64 || (C % 64) || !rank_ok(r)) return QLORA_ERR_SHAPE;
  RowGroups g = single_group(C);
  if (group_rows) {  // adapters along big's columns, small [M, n r]
    const qlora_status gs = make_groups(group_rows, n_groups, C, r, &g);
    if (gs != QLORA_OK) return gs;
  }
  if (!aligned16(big) || !aligned16(small) || !aligned16(out)) return QLORA_ERR_ALIGN;
  (void)ws;  // the cluster reduction needs no scratch
  (void)ws_bytes;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  int* err;
  if ((st = error_word_ptr(dev, &err)) != QLORA_OK) return st;
  return do_lora_grad(big, M, C, small, r, g, scale, out, out_r_by_c == 0, err,
                      static_cast<cudaStream_t>(stream));
}

qlora_status qlora_gemm_plan(int M, int rows_w, int steps_per_tile, int sm_count, int* bt,
                             int* nh, int* streamk, int* grid, size_t* partial_bytes) {
  if (!bt || !nh || !streamk || !grid || !partial_bytes) return QLORA_ERR_NULL;
  if (M < 1 || rows_w < 1 || steps_per_tile < 2 || sm_count < 1) return QLORA_ERR_SHAPE;
  const GemmTile t = gemm_pick_tile(M, rows_w, steps_per_tile, sm_count);
  const GemmSchedule sc = gemm_schedule(M, rows_w, steps_per_tile, sm_count);
  *bt = t.bt;
  *nh = t.nh;
  *streamk = sc.streamk;
  *grid = sc.grid;
  *partial_bytes = 4 * sc.partial_floats;
  return QLORA_OK;
}

int qlora_set_rank_fusion(int enable) {
  return g_rank_fusion.exchange(enable ? 1 : 0, std::memory_order_relaxed);
}

int qlora_set_side_overlap(int mode) {
  return g_side_overlap.exchange(mode < 0 ? 0 : (mode > 2 ? 2 : mode), std::memory_order_relaxed);
}

int qlora_backward_side_sms(int M, int N, int K, int R, int sm_count, int mode) {
  if (sm_count < 1) return 0;
  if (mode < 0) mode = qlora::g_side_overlap.load(std::memory_order_relaxed);
  return qlora::side_sms(M, N, K, R, sm_count, mode > 2 ? 2 : mode);
}

int qlora_gemm_rank_fusable(int M, int rows_w, int steps_per_tile, int sm_count, int rank_cols,
                            int r, int transpose_w, int* bt) {
  if (bt) *bt = 0;
  if (M < 1 || rows_w < 1 || steps_per_tile < 2 || sm_count < 1 || r < 8 || r > rank_cols)
    return 0;
  if (!gemm_rank_fusable(M, rows_w, steps_per_tile, sm_count, rank_cols,
                         gemm_rank_slot_bytes(transpose_w != 0, rank_cols, r)))
    return 0;
  if (bt) *bt = gemm_pick_tile(M, rows_w, steps_per_tile, sm_count, true).bt;
  return 1;
}

qlora_status qlora_selftest_bounded_wait(qlora_stream_t stream) {
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  int* err;
  if ((st = error_word_ptr(dev, &err)) != QLORA_OK) return st;
  st = cuda_status(launch_bounded_wait_selftest(err, static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

uint64_t qlora_launch_counter(void) { return g_launches.load(std::memory_order_relaxed); }

qlora_status qlora_swiglu_fwd(const void* g, const void* u, void* a, int64_t n,
                              qlora_stream_t stream) {
  if (!g || !u || !a) return QLORA_ERR_NULL;
  if (n < 0) return QLORA_ERR_SHAPE;
  if (!aligned16(g) || !aligned16(u) || !aligned16(a)) return QLORA_ERR_ALIGN;
  if (n == 0) return QLORA_OK;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_swiglu_fwd(static_cast<const __nv_bfloat16*>(g),
                                     static_cast<const __nv_bfloat16*>(u),
                                     static_cast<__nv_bfloat16*>(a), n,
                                     static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

qlora_status qlora_swiglu_bwd(const void* g, const void* u, const void* da, void* dg, void* du,
                              int64_t n, qlora_stream_t stream) {
  if (!g || !u || !da || !dg || !du) return QLORA_ERR_NULL;
  if (n < 0) return QLORA_ERR_SHAPE;
  if (!aligned16(g) || !aligned16(u) || !aligned16(da) || !aligned16(dg) || !aligned16(du))
    return QLORA_ERR_ALIGN;
  if (n == 0) return QLORA_OK;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_swiglu_bwd(
      static_cast<const __nv_bfloat16*>(g), static_cast<const __nv_bfloat16*>(u),
      static_cast<const __nv_bfloat16*>(da), static_cast<__nv_bfloat16*>(dg),
      static_cast<__nv_bfloat16*>(du), n, static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

qlora_status qlora_swiglu_packed_fwd(const void* gu, void* a, int64_t M, int I,
                                     qlora_stream_t stream) {
  if (!gu || !a) return QLORA_ERR_NULL;
  if (M < 0 || I < 8 || I % 8) return QLORA_ERR_SHAPE;
  if (!aligned16(gu) || !aligned16(a)) return QLORA_ERR_ALIGN;
  if (M == 0) return QLORA_OK;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_swiglu_packed_fwd(static_cast<const __nv_bfloat16*>(gu),
                                            static_cast<__nv_bfloat16*>(a), M, I,
                                            static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

qlora_status qlora_swiglu_packed_bwd(const void* gu, const void* da, void* dgu, int64_t M, int I,
                                     qlora_stream_t stream) {
  if (!gu || !da || !dgu) return QLORA_ERR_NULL;
  if (M < 0 || I < 8 || I % 8) return QLORA_ERR_SHAPE;
  if (!aligned16(gu) || !aligned16(da) || !aligned16(dgu)) return QLORA_ERR_ALIGN;
  if (M == 0) return QLORA_OK;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_swiglu_packed_bwd(
      static_cast<const __nv_bfloat16*>(gu), static_cast<const __nv_bfloat16*>(da),
      static_cast<__nv_bfloat16*>(dgu), M, I, static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

size_t qlora_lm_head_ce_workspace_bytes(int M, int V, int K, int chunk) {
  if (M < 1 || V < 128 || V % 64 || K < 128 || K % 64) return 0;
  const int c = chunk < 1 || chunk > M ? M : chunk;
  const size_t scratch = std::max(gemm_ws_bytes(c, V, K, 0, false), gemm_ws_bytes(c, V, K, 0, true));
  return align256(static_cast<size_t>(c) * V * 2) + align256(static_cast<size_t>(M) * 4) + 256 +
         align256(scratch);
}

qlora_status qlora_lm_head_ce(const void* X, const qlora_nf4_weight* W, const int* labels, int M,
                              int chunk, float* loss, float* token_loss, void* dX, void* ws,
                              size_t ws_bytes, qlora_stream_t stream) {
  if (!X || !labels || !loss) return QLORA_ERR_NULL;
  qlora_status st = check_weight(W);
  if (st != QLORA_OK) return st;
  const int V = W->N, K = W->K;
  // Both GEMMs run without an extension, so each reduction (K forward, V for dX) must give
  // every tile at least the two steps the dequant groups take at a time.
  if (M < 1 || K < 128 || V < 128) return QLORA_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(labels) || !aligned16(loss) ||
      (token_loss && !aligned16(token_loss)) || (dX && !aligned16(dX)))
    return QLORA_ERR_ALIGN;
  const int c = chunk < 1 || chunk > M ? M : chunk;
  const size_t need = qlora_lm_head_ce_workspace_bytes(M, V, K, chunk);
  if (!ws || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  int dev;
  if ((st = current_device(&dev)) != QLORA_OK) return st;
  int* err;
  if ((st = error_word_ptr(dev, &err)) != QLORA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Workspace: logits chunk [c, V] bf16 | token losses [M] fp32 | count | GEMM partial sums.
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  auto* z = reinterpret_cast<__nv_bfloat16*>(w8);
  size_t off = align256(static_cast<size_t>(c) * V * 2);
  float* tl = token_loss ? token_loss : reinterpret_cast<float*>(w8 + off);
  off += align256(static_cast<size_t>(M) * 4);
  int* cnt = reinterpret_cast<int*>(w8 + off);
  off += 256;
  void* scratch = w8 + off;
  const size_t scratch_bytes = need - off;

  if ((st = cuda_status(launch_ce_count(labels, M, V, cnt, s))) != QLORA_OK) return st;
  count(1);
  const auto* x = static_cast<const __nv_bfloat16*>(X);
  auto* dx = static_cast<__nv_bfloat16*>(dX);
  for (int m0 = 0; m0 < M; m0 += c) {
    const int mc = std::min(c, M - m0);
    // z = X_c deq(W)^T: the chunk's logits, then its loss rows and (with dX) the gradient
    // dz = (softmax(z) - onehot) / count in place, then dX_c = dz deq(W).
    st = do_gemm(x + static_cast<size_t>(m0) * K, W, false, nullptr, nullptr, mc, 0,
                 single_group(V), z, err, scratch, scratch_bytes, s);
    if (st != QLORA_OK) return st;
    st = cuda_status(launch_ce_rows(z, mc, V, labels + m0, cnt, tl + m0, dX != nullptr, s));
    if (st != QLORA_OK) return st;
    count(1);
    if (dX) {
      st = do_gemm(z, W, true, nullptr, nullptr, mc, 0, single_group(K),
                   dx + static_cast<size_t>(m0) * K, err, scratch, scratch_bytes, s);
      if (st != QLORA_OK) return st;
    }
  }
  st = cuda_status(launch_ce_mean(tl, M, cnt, loss, s));
  if (st == QLORA_OK) count(1);
  return st;
}

qlora_status qlora_cross_entropy_count(const int* labels, int M, int V, int* count_out,
                                       qlora_stream_t stream) {
  if (!labels || !count_out) return QLORA_ERR_NULL;
  if (M < 1 || V < 8 || V % 8) return QLORA_ERR_SHAPE;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_ce_count(labels, M, V, count_out, static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

qlora_status qlora_cross_entropy_rows(void* z, int rows, int V, const int* labels,
                                      const int* count_in, float* token_loss, int write_grad,
                                      qlora_stream_t stream) {
  if (!z || !labels || !count_in || !token_loss) return QLORA_ERR_NULL;
  if (rows < 1 || V < 8 || V % 8) return QLORA_ERR_SHAPE;
  if (!aligned16(z)) return QLORA_ERR_ALIGN;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_ce_rows(static_cast<__nv_bfloat16*>(z), rows, V, labels, count_in,
                                  token_loss, write_grad != 0, static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

qlora_status qlora_cross_entropy_mean(const float* token_loss, int M, const int* count_in,
                                      float* loss, qlora_stream_t stream) {
  if (!token_loss || !count_in || !loss) return QLORA_ERR_NULL;
  if (M < 1) return QLORA_ERR_SHAPE;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  st = cuda_status(launch_ce_mean(token_loss, M, count_in, loss, static_cast<cudaStream_t>(stream)));
  if (st == QLORA_OK) count(1);
  return st;
}

qlora_status qlora_linear_fwd_noalloc(const void* X, const qlora_nf4_weight* W, const void* A,
                                      const void* B, int M, int r, float alpha, void* H,
                                      void* XA_saved, qlora_stream_t stream) {
  if (!X || !A || !B || !H) return QLORA_ERR_NULL;
  qlora_status st = check_weight(W);
  if (st != QLORA_OK) return st;
  if (M < 1 || !rank_ok(r)) return QLORA_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(H) ||
      (XA_saved && !aligned16(XA_saved)))
    return QLORA_ERR_ALIGN;
  // The forward needs s*XA [M, r] bf16; the GEMM's partial sums use what is left of the
  // scratch (whole tiles if they do not fit).
  const size_t sxa_bytes = align256(static_cast<size_t>(M) * r * 2);
  if (sxa_bytes > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;
  int dev;
  if ((st = current_device(&dev)) != QLORA_OK) return st;
  int* err;
  if ((st = error_word_ptr(dev, &err)) != QLORA_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != QLORA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(scratch);
  auto* sxa = reinterpret_cast<__nv_bfloat16*>(w8);
  const float scale = alpha / static_cast<float>(r);
  // Both scratch regions are written in full before they are read: nothing needs clearing.
  st = do_lora_down(X, M, W->K, A, true, r, single_group(W->K), scale, XA_saved, sxa, err, s);
  if (st != QLORA_OK) return st;
  return do_gemm(X, W, false, B, sxa, M, r, single_group(W->N), H, err, w8 + sxa_bytes,
                 kNoAllocScratchBytes - sxa_bytes, s);
}

size_t qlora_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

qlora_status qlora_device_error(int* code) {
  if (!code) return QLORA_ERR_NULL;
  int dev;
  qlora_status st = current_device(&dev);
  if (st != QLORA_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return QLORA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_qlora_error_word, sizeof(int)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  *code = v;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_qlora_error_word, &zero, sizeof(int)) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return QLORA_ERR_TIMEOUT;
  }
  return QLORA_OK;
}

}  // extern "C"

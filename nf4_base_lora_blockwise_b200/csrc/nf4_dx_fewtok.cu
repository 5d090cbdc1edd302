// nf4_dx_fewtok.cu -- dX for few tokens (M <= 32), where streaming the packed weight from HBM is
// the whole cost ("Unsloth vs QLoRA vs Liger-Kernel", section 2, hand-derived backward):
//   dX[M, K] = dY[M, N] . deq(W0) + (s dYB)[M, r] . A
//
// dX reduces over the weight's rows, so a weight row (contiguous along K) contributes to every
// output column.  A CTA owns 256 output columns and a contiguous range of weight rows, and
// streams that panel in steps of 64 rows: the packed codes (64 rows x 128 bytes) and the matching
// 64 columns of dY arrive by TMA in a 4-stage ring; four threads per row decode one 64-element
// block each -- the block's 16 exact results bf16(fp32(level * absmax)) built once in registers,
// the same table the dequant GEMM uses, so the weight enters bit for bit as deq(W0) -- into a
// swizzled bf16 tile [64 rows, 256 columns] in shared memory (double-buffered); the eight warps
// then feed m16n8k16 tensor-core MMAs with dY fragments (tokens x rows) and the tile's
// transposed 8 x 8 blocks (rows x columns), 32 output columns per warp.  Each CTA writes its fp32
// partial [M, 256] to the workspace; a finalize kernel adds the row splits in order, adds the
// LoRA term (s dYB) . A in fp32 and rounds once to bf16, so results do not depend on timing.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "nf4_dequant.cuh"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kFtThreads = 256;           // 8 warps
constexpr int kFtRows = 64;               // weight rows per stage
constexpr int kFtCols = 256;              // output columns per CTA
constexpr uint32_t kFtCodeBytes = kFtRows * kFtCols / 2;  // 8 KB of codes per stage
constexpr uint32_t kFtDecBytes = kFtRows * kFtCols * 2;   // 32 KB decoded bf16 tile

constexpr uint32_t kFtAmBytes = kFtRows * 4 * 4;  // block scales: 64 rows x 4 blocks, fp32
// A ring slot: the codes, dY [16 mb tokens, 64 rows], and (fp32 absmax, K % 256 == 0) the
// stage's block scales.
__host__ __device__ constexpr uint32_t ft_slot_bytes(int mb) {
  return kFtCodeBytes + static_cast<uint32_t>(mb) * 2048u + kFtAmBytes;
}
// TMA ring depth: 4 stages, 3 with 32 tokens, so two CTAs fit on an SM either way.
__host__ __device__ constexpr int ft_stages(int mb) { return mb == 1 ? 4 : 3; }
__host__ __device__ constexpr size_t ft_smem_bytes(int mb) {
  return 1024 + ft_stages(mb) * ft_slot_bytes(mb) + 2 * kFtDecBytes + 8 * ft_stages(mb);
}

struct FtArgs {
  int M, N, K;
  int kblocks;     // K / 64
  int gk;          // CTAs along the output columns (K / 256, rounded up)
  int splits;      // CTAs along the weight rows
  int dq;
  const float* absmax;
  const uint8_t* absmax_q8;
  const float* absmax_scale;
  float* part;     // [splits, M, K] fp32
  int* err;
  Codebook cb;
  int am_tma;      // the block scales arrive in the ring slot (else per-thread loads)
};

// grid (gk x splits): CTA b takes output columns 256 (b % gk) .. and the row steps of split
// b / gk (consecutive CTAs share a row range, so its dY columns are read from L2 once).
template <int MB>
__global__ void __launch_bounds__(kFtThreads, 2)
    nf4_dx_fewtok_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_dy,
                         const __grid_constant__ CUtensorMap tm_am, const FtArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr uint32_t kSlot = ft_slot_bytes(MB);
  constexpr int kFtStages = ft_stages(MB);
  uint8_t* dec = ring + kFtStages * kSlot;
  uint64_t* full = reinterpret_cast<uint64_t*>(dec + 2 * kFtDecBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kg = static_cast<int>(blockIdx.x) % a.gk;
  const int sp = static_cast<int>(blockIdx.x) / a.gk;
  const int nst = a.N / kFtRows;
  const int st0 = static_cast<int>(static_cast<long long>(nst) * sp / a.splits);
  const int n_st = static_cast<int>(static_cast<long long>(nst) * (sp + 1) / a.splits) - st0;
  const int k0 = kg * kFtCols;

  if (tid == 0) {
    for (int s = 0; s < kFtStages; ++s) mbar_init(full + s, 1);
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // dY (and the rank-r operands the finalize reads) are complete
  pdl_trigger();

  // Thread 0 issues stage i (local index) into slot i % kFtStages: the codes of rows
  // 64 (st0 + i) .. + 63 in this CTA's 128-byte column band, and dY's matching 64 columns.
  int issued = 0;
  auto issue = [&](int i) {
    uint8_t* dst = ring + (i % kFtStages) * kSlot;
    uint64_t* bar = full + (i % kFtStages);
    const int n0 = (st0 + i) * kFtRows;
    mbar_arrive_expect_tx(bar, kFtCodeBytes + MB * 2048u + (a.am_tma ? kFtAmBytes : 0u));
    tma_load_2d(dst, &tm_q, bar, k0 / 2, n0);
    tma_load_2d(dst + kFtCodeBytes, &tm_dy, bar, n0, 0);
    if (a.am_tma) tma_load_2d(dst + kFtCodeBytes + MB * 2048u, &tm_am, bar, kg * 4, n0);
    issued = i + 1;
  };
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_dy);
    if (a.am_tma) tma_prefetch_desc(&tm_am);
    for (int i = 0; i < n_st && i < kFtStages; ++i) issue(i);
  }

  // Decode: thread = (row drow of the stage, block dj of the 4 in the column band).
  const int drow = tid >> 2, dj = tid & 3;
  const int kb = kg * 4 + dj;
  auto absmax_of = [&](int i) -> float {
    if (a.am_tma || i >= n_st || kb >= a.kblocks) return 0.f;  // past K: zero weight
    const long long n = static_cast<long long>(st0 + i) * kFtRows + drow;
    return nf4_block_absmax(a.absmax, a.absmax_q8, a.absmax_scale, a.dq, n * a.kblocks + kb);
  };
  // Block scales run kAmAhead stages ahead of their use (their loads are scattered HBM reads).
  constexpr int kAmAhead = 3;
  float am_q[kAmAhead];
#pragma unroll
  for (int j = 0; j < kAmAhead; ++j) am_q[j] = absmax_of(j);

  float acc[MB][4][4];
#pragma unroll
  for (int mb = 0; mb < MB; ++mb)
#pragma unroll
    for (int nb = 0; nb < 4; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mb][nb][e] = 0.f;

  bool failed = false;
  for (int i = 0; i < n_st; ++i) {
    const int slot = i % kFtStages;
    const float am = am_q[0];
    const float am_next = failed ? 0.f : absmax_of(i + kAmAhead);
    if (!failed)
      failed = !mbar_wait_warp(full + slot, static_cast<uint32_t>(i / kFtStages) & 1u,
                               kErrWaitFull, a.err, i);
    uint8_t* d = dec + (i & 1) * kFtDecBytes;
    if (!failed) {
      // (128B-swizzled code tile: 16-byte chunk c of row r sits at chunk c ^ (r & 7).)
      const uint8_t* codes = ring + slot * kSlot + drow * 128;
      const uint32_t cph = static_cast<uint32_t>(drow) & 7u;
      const uint4 c0 = *reinterpret_cast<const uint4*>(codes + (((2u * dj) ^ cph) << 4));
      const uint4 c1 = *reinterpret_cast<const uint4*>(codes + (((2u * dj + 1u) ^ cph) << 4));
      const float scale = a.am_tma ? reinterpret_cast<const float*>(
                                         ring + slot * kSlot + kFtCodeBytes + MB * 2048u)[tid]
                                   : am;
      Nf4Lut lut;
      nf4_build_lut(a.cb, scale, lut);
      uint8_t* row = d + drow * (kFtCols * 2);
      const uint32_t ph = static_cast<uint32_t>(drow) & 7u;
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e)  // 8 elements per 16-byte chunk, chunks 8 dj .. 8 dj + 7
        *reinterpret_cast<uint4*>(row + (((8u * dj + e) ^ ph) << 4)) = nf4_lookup8(lut, w[e]);
    }
    // This thread's reads of the ring (codes now, dY in the previous stage's MMAs) come before
    // the refill below, a TMA (async-proxy) write.
    fence_proxy_async_smem();
    __syncthreads();
    // Every thread is past the previous stage's MMAs: its slot takes stage i - 1 + kFtStages.
    if (tid == 0 && !failed && i >= 1 && i - 1 + kFtStages < n_st) issue(i - 1 + kFtStages);
    if (!failed) {
      const uint32_t dyb = smem_u32(ring + slot * kSlot + kFtCodeBytes);
      const uint32_t db = smem_u32(d);
#pragma unroll
      for (int s16 = 0; s16 < 4; ++s16) {
        uint32_t af[MB][4];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)  // dY [tokens x 16 rows], 128B-swizzled TMA tile
          ldsm_x4(af[mb], dyb + swz_off(static_cast<uint32_t>(16 * mb + (lane & 15)),
                                        static_cast<uint32_t>(2 * s16 + (lane >> 4)), 128u, 7u));
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          // Tile rows 16 s16 .. + 15 (the reduction) x columns 8 (4 warp + 2 p) .. + 15,
          // transposed 8 x 8 loads: b0, b1 of column group 2p, then of 2p + 1.
          const uint32_t r = static_cast<uint32_t>(16 * s16 + (lane & 7) + ((lane >> 3) & 1) * 8);
          const uint32_t ch = static_cast<uint32_t>(4 * warp + 2 * p + (lane >> 4));
          uint32_t b[4];
          ldsm_x4_t(b, db + r * (kFtCols * 2) + ((ch ^ (r & 7u)) << 4));
#pragma unroll
          for (int mb = 0; mb < MB; ++mb) {
            mma16816(acc[mb][2 * p], af[mb], b[0], b[1]);
            mma16816(acc[mb][2 * p + 1], af[mb], b[2], b[3]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j + 1 < kAmAhead; ++j) am_q[j] = am_q[j + 1];
    am_q[kAmAhead - 1] = am_next;
  }

  // This split's partial: tokens 16 mb + lane/4 (+ 8), columns k0 + 32 warp + 8 nb + 2 (lane % 4).
  if (!failed) {
    const int rq = lane >> 2, q = lane & 3;
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
      for (int nb = 0; nb < 4; ++nb)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int m = 16 * mb + rq + 8 * hf;
          const int k = k0 + 32 * warp + 8 * nb + 2 * q;
          if (m < a.M && k < a.K)
            *reinterpret_cast<float2*>(a.part + (static_cast<long long>(sp) * a.M + m) * a.K + k) =
                make_float2(acc[mb][nb][2 * hf], acc[mb][nb][2 * hf + 1]);
        }
  }
  // A failed run may leave copies in flight: they land before the CTA exits.
  if (tid == 0 && failed)
    for (int i = issued > kFtStages ? issued - kFtStages : 0; i < issued; ++i)
      mbar_wait(full + i % kFtStages, static_cast<uint32_t>(i / kFtStages) & 1u, kErrWaitDrain,
                a.err, i);
}

// dX[m, k] = bf16(sum over splits of part[split, m, k], in order, + sum_j sdyb[m, j] A[j, k]);
// two columns per thread.
__global__ void __launch_bounds__(128) nf4_dx_fewtok_finalize(const FtArgs a,
                                                              const __nv_bfloat16* __restrict__ sdyb,
                                                              const __nv_bfloat16* __restrict__ A,
                                                              int R, __nv_bfloat16* __restrict__ dx) {
  pdl_wait();  // the partials are complete
  pdl_trigger();
  const long long pairs = static_cast<long long>(a.M) * (a.K / 2);
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= pairs) return;
  const int m = static_cast<int>(idx / (a.K / 2));
  const int k = static_cast<int>(idx - static_cast<long long>(m) * (a.K / 2)) * 2;
  float v0 = 0.f, v1 = 0.f;
  const long long stride = static_cast<long long>(a.M) * a.K;
  const float* pp = a.part + static_cast<long long>(m) * a.K + k;
  int s = 0;
  for (; s + 8 <= a.splits; s += 8) {  // eight loads in flight, added in split order
    float2 p[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) p[j] = __ldg(reinterpret_cast<const float2*>(pp + (s + j) * stride));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v0 += p[j].x;
      v1 += p[j].y;
    }
  }
  for (; s < a.splits; ++s) {
    const float2 p = __ldg(reinterpret_cast<const float2*>(pp + s * stride));
    v0 += p.x;
    v1 += p.y;
  }
  float l0 = 0.f, l1 = 0.f;
  int j = 0;
  for (; j + 8 <= R; j += 8) {  // eight columns of A in flight
    __nv_bfloat162 w[8];
#pragma unroll
    for (int t = 0; t < 8; ++t)
      w[t] = *reinterpret_cast<const __nv_bfloat162*>(A + static_cast<long long>(j + t) * a.K + k);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float e = __bfloat162float(sdyb[static_cast<long long>(m) * R + j + t]);
      l0 += e * __low2float(w[t]);
      l1 += e * __high2float(w[t]);
    }
  }
  for (; j < R; ++j) {
    const float e = __bfloat162float(sdyb[static_cast<long long>(m) * R + j]);
    const __nv_bfloat162 w =
        *reinterpret_cast<const __nv_bfloat162*>(A + static_cast<long long>(j) * a.K + k);
    l0 += e * __low2float(w);
    l1 += e * __high2float(w);
  }
  *reinterpret_cast<__nv_bfloat162*>(dx + static_cast<long long>(m) * a.K + k) =
      __floats2bfloat162_rn(v0 + l0, v1 + l1);
}

// The few-token backward's last kernel: every block first sums dY B for all tokens from the
// down-projection's partials (in split order, rounded to bf16 -- rank_down_finalize's
// arithmetic) or loads XA, then takes one job by block range:
//   [0, nx)          dX pairs, as nf4_dx_fewtok_finalize with s dYB from shared memory
//   [nx, nx + na)    dA[j, k] = s sum_m dYB[m, j] X[m, k]        (two columns k per thread)
//   [nx + na, ...)   dB[n, j] = s sum_m dY[m, n] XA[m, g(n) r + j]  (eight columns j per thread)
// The sums over the M <= 32 tokens run in token order in fp32.
struct FtTail {
  const float* dpart;  // dY B partials [gsplit][128][R]
  int gsplit;
  int R, r;            // n r packed columns; r per adapter
  float scale;
  const float* xpart;  // dX split partials [splits][M][K] (nx == 0: none)
  int splits;
  int M, N, K;
  const __nv_bfloat16* X;
  const __nv_bfloat16* dY;
  const __nv_bfloat16* XA;
  const __nv_bfloat16* A;
  RowGroups groups;
  __nv_bfloat16* dx;
  float* dA;
  float* dB;
  int nx, na;
};

__global__ void __launch_bounds__(128) nf4_fewtok_bwd_tail(const FtTail t) {
  __shared__ float s_rank[kFewTokDxMaxTokens * kFoldMaxR];
  pdl_wait();  // the partials are complete
  pdl_trigger();
  const int b = static_cast<int>(blockIdx.x);
  const int job = b < t.nx ? 0 : (b < t.nx + t.na ? 1 : 2);
  const int mr = t.M * t.R;
  if (job < 2) {  // job 0: s dYB (the LoRA term of dX); job 1: dYB
    for (int i = threadIdx.x; i < mr; i += blockDim.x) {
      const int m = i / t.R, j = i - m * t.R;
      float v = 0.f;
      for (int g = 0; g < t.gsplit; ++g)
        v += __ldg(t.dpart + (static_cast<long long>(g) * 128 + m) * t.R + j);
      s_rank[i] = __bfloat162float(__float2bfloat16_rn(job == 0 ? t.scale * v : v));
    }
  } else {
    for (int i = threadIdx.x; i < mr; i += blockDim.x) s_rank[i] = __bfloat162float(t.XA[i]);
  }
  __syncthreads();
  const long long idx = static_cast<long long>(job == 0 ? b : (job == 1 ? b - t.nx
                                                                          : b - t.nx - t.na)) *
                            blockDim.x + threadIdx.x;
  if (job == 0) {
    if (idx >= static_cast<long long>(t.M) * (t.K / 2)) return;
    const int m = static_cast<int>(idx / (t.K / 2));
    const int k = static_cast<int>(idx - static_cast<long long>(m) * (t.K / 2)) * 2;
    float v0 = 0.f, v1 = 0.f;
    const long long stride = static_cast<long long>(t.M) * t.K;
    const float* pp = t.xpart + static_cast<long long>(m) * t.K + k;
    int s = 0;
    for (; s + 8 <= t.splits; s += 8) {  // eight loads in flight, added in split order
      float2 p[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        p[j] = __ldg(reinterpret_cast<const float2*>(pp + (s + j) * stride));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v0 += p[j].x;
        v1 += p[j].y;
      }
    }
    for (; s < t.splits; ++s) {
      const float2 p = __ldg(reinterpret_cast<const float2*>(pp + s * stride));
      v0 += p.x;
      v1 += p.y;
    }
    float l0 = 0.f, l1 = 0.f;
    const float* e = s_rank + m * t.R;
    for (int j = 0; j < t.R; ++j) {
      const __nv_bfloat162 w =
          *reinterpret_cast<const __nv_bfloat162*>(t.A + static_cast<long long>(j) * t.K + k);
      l0 += e[j] * __low2float(w);
      l1 += e[j] * __high2float(w);
    }
    *reinterpret_cast<__nv_bfloat162*>(t.dx + static_cast<long long>(m) * t.K + k) =
        __floats2bfloat162_rn(v0 + l0, v1 + l1);
  } else if (job == 1) {
    if (idx >= static_cast<long long>(t.R) * (t.K / 2)) return;
    const int j = static_cast<int>(idx / (t.K / 2));
    const int k = static_cast<int>(idx - static_cast<long long>(j) * (t.K / 2)) * 2;
    float a0 = 0.f, a1 = 0.f;
    for (int m = 0; m < t.M; ++m) {
      const float d = s_rank[m * t.R + j];
      const float2 x = __bfloat1622float2(
          *reinterpret_cast<const __nv_bfloat162*>(t.X + static_cast<long long>(m) * t.K + k));
      a0 = fmaf(d, x.x, a0);
      a1 = fmaf(d, x.y, a1);
    }
    *reinterpret_cast<float2*>(t.dA + static_cast<long long>(j) * t.K + k) =
        make_float2(t.scale * a0, t.scale * a1);
  } else {
    const int groups8 = t.r / 8;
    if (idx >= static_cast<long long>(t.N) * groups8) return;
    const int n = static_cast<int>(idx / groups8);
    const int j0 = static_cast<int>(idx - static_cast<long long>(n) * groups8) * 8;
    const float* xa = s_rank + row_group(t.groups, n) * t.r + j0;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int m = 0; m < t.M; ++m) {
      const float d = __bfloat162float(t.dY[static_cast<long long>(m) * t.N + n]);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(d, xa[m * t.R + i], acc[i]);
    }
    float4* o = reinterpret_cast<float4*>(t.dB + static_cast<long long>(n) * t.r + j0);
    o[0] = make_float4(t.scale * acc[0], t.scale * acc[1], t.scale * acc[2], t.scale * acc[3]);
    o[1] = make_float4(t.scale * acc[4], t.scale * acc[5], t.scale * acc[6], t.scale * acc[7]);
  }
}

}  // namespace

cudaError_t launch_fewtok_bwd_tail(const FewTokTail& tl, const float* xpart, int splits, int M,
                                   int N, int K, __nv_bfloat16* dx, cudaStream_t stream) {
  const int R = tl.groups.n * tl.r;
  if (M < 1 || M > kFewTokDxMaxTokens || R != tl.fold.R || R > kFoldMaxR || tl.r % 8 ||
      K % 2 || !tl.fold.part || tl.fold.gsplit < 1 || (dx && (!xpart || splits < 1)))
    return cudaErrorInvalidValue;
  FtTail t;
  t.dpart = tl.fold.part;
  t.gsplit = tl.fold.gsplit;
  t.R = R;
  t.r = tl.r;
  t.scale = tl.fold.scale;
  t.xpart = xpart;
  t.splits = splits;
  t.M = M;
  t.N = N;
  t.K = K;
  t.X = tl.X;
  t.dY = tl.dY;
  t.XA = tl.XA;
  t.A = tl.A;
  t.groups = tl.groups;
  t.dx = dx;
  t.dA = tl.dA;
  t.dB = tl.dB;
  const long long per = 128;
  t.nx = dx ? static_cast<int>((static_cast<long long>(M) * (K / 2) + per - 1) / per) : 0;
  t.na = static_cast<int>((static_cast<long long>(R) * (K / 2) + per - 1) / per);
  const long long nb = (static_cast<long long>(N) * (tl.r / 8) + per - 1) / per;
  return launch_pdl(nf4_fewtok_bwd_tail, dim3(static_cast<unsigned>(t.nx + t.na + nb)),
                    dim3(128), 0, stream, 1, t);
}

FewTokDxPlan fewtok_dx_plan(int M, int N, int K, int sm_count) {
  FewTokDxPlan p;
  p.gk = (K + kFtCols - 1) / kFtCols;
  // Two CTAs per SM (at most), each with at least two row steps.
  int s = 2 * sm_count / p.gk;
  const int max_s = N / (2 * kFtRows);
  if (s > max_s) s = max_s;
  p.splits = s < 1 ? 1 : s;
  p.grid = p.gk * p.splits;
  p.part_bytes = static_cast<size_t>(p.splits) * M * K * 4;
  p.mb = M <= 16 ? 1 : 2;
  return p;
}

cudaError_t launch_nf4_fewtok_dx(const CUtensorMap& tm_q, const CUtensorMap& tm_dy,
                                 const CUtensorMap* tm_am, const FewTokDxPlan& p, int M, int N,
                                 int K, const float* absmax,
                                 const uint8_t* absmax_q8, const float* absmax_scale, int dq,
                                 const __nv_bfloat16* sdyb, const __nv_bfloat16* A, int R,
                                 __nv_bfloat16* dx, float* part, size_t part_bytes,
                                 const Codebook& cb, int* err, cudaStream_t stream,
                                 bool finalize) {
  if (M < 1 || M > kFewTokDxMaxTokens || N % kFtRows || K % 64 || p.part_bytes > part_bytes ||
      !part)
    return cudaErrorInvalidValue;
  FtArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.kblocks = K / 64;
  a.gk = p.gk;
  a.splits = p.splits;
  a.dq = dq;
  a.absmax = absmax;
  a.absmax_q8 = absmax_q8;
  a.absmax_scale = absmax_scale;
  a.part = part;
  a.err = err;
  a.cb = cb;
  a.am_tma = (tm_am && !dq && K % 256 == 0) ? 1 : 0;
  const CUtensorMap& am_map = a.am_tma ? *tm_am : tm_q;  // (never read without am_tma)
  cudaError_t e;
  if (p.mb == 1) {
    e = cudaFuncSetAttribute(nf4_dx_fewtok_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(ft_smem_bytes(1)));
    if (e == cudaSuccess)
      e = launch_pdl(nf4_dx_fewtok_kernel<1>, dim3(p.grid), dim3(kFtThreads), ft_smem_bytes(1),
                     stream, 1, tm_q, tm_dy, am_map, a);
  } else {
    e = cudaFuncSetAttribute(nf4_dx_fewtok_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(ft_smem_bytes(2)));
    if (e == cudaSuccess)
      e = launch_pdl(nf4_dx_fewtok_kernel<2>, dim3(p.grid), dim3(kFtThreads), ft_smem_bytes(2),
                     stream, 1, tm_q, tm_dy, am_map, a);
  }
  if (e != cudaSuccess || !finalize) return e;
  const long long pairs = static_cast<long long>(M) * (K / 2);
  return launch_pdl(nf4_dx_fewtok_finalize, dim3(static_cast<unsigned>((pairs + 127) / 128)),
                    dim3(128), 0, stream, 1, a, sdyb, A, R, dx);
}

}  // namespace qlora

// nf4_gemv.cu -- the forward dequant product for few tokens (M <= 32), where streaming the
// packed weight from HBM is the whole cost ("Unsloth vs QLoRA vs Liger-Kernel", section 1
// forward formula):
//   h[M, N] = X[M, K] . deq(W0)^T + (s XA)[M, r] . B^T
//
// The tcgen05 kernel moves every 64-deep step of a 128-row weight tile through shared-memory
// rings with several barrier hand-offs; with a handful of tokens those hand-offs, not HBM,
// set the pace.  Here every warp works alone on 16 weight rows: it loads the packed codes with
// plain 8-byte loads straight into registers, turns them into bf16 with byte permutes against
// the unscaled codebook (a constant table), and feeds them as the A operand of warp-level
// m16n8k16 tensor-core MMAs whose B operand (the tokens) sits in shared memory.  The block
// scale is applied to each 64-deep partial sum:
//   sum_k x_k deq_k = sum_blocks absmax_b * sum_{k in b} x_k bf16(c_k)
// i.e. the weight enters the product as bf16(c) * absmax (the codebook value rounded to bf16)
// instead of bf16(c * absmax); each rounds c * absmax within 2^-8 relative, so the two agree
// to about one bf16 rounding of the weight.
//
// Schedule (stream-K): the (128-row tile, 64-block) units, row-tile major, are cut into equal
// contiguous ranges, one per CTA (two CTAs per SM).  A CTA's range covers at most a few row
// tiles; for each it writes fp32 partial sums [tokens, 128 rows] to its own slot, and a
// finalize kernel adds the slots of each row tile in order, adds the LoRA up-projection and
// rounds to bf16 -- deterministic.  Codes, block scales and the X chunk (shared by the CTA's 8
// warps, so X is read from L2 once per 128 weight rows) stream through a 3-4 stage cp.async
// ring, which keeps ~100 KB of weight in flight per SM.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "nf4_dequant.cuh"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kGvWarps = 8;
constexpr int kGvThreads = 32 * kGvWarps;
constexpr int kGvRows = 16 * kGvWarps;  // weight rows per tile
constexpr int kGvBlk = 4;               // 64-blocks per pipeline stage

__device__ __forceinline__ uint32_t gv_saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async8(void* dst, const void* src, bool pred) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(gv_saddr(dst)), "l"(src),
               "r"(pred ? 8 : 0)
               : "memory");
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A stage of the pipeline: up to kGvBlk consecutive 64-blocks of one row tile.  The CTA's
// units [u0, u1) are cut at row-tile ends (segments) and every kGvBlk blocks; a cursor walks
// the stages in order, dividing only when it enters a new segment.
struct GvCursor {
  long long u1;      // end of the CTA's range
  long long seg_u;   // first unit of the current segment
  long long seg_e;   // end of the current segment
  int KB;
  int rt, kb, nblk;  // current stage: row tile, first block, blocks
  int seg;           // segment index within the range
  bool seg_end;      // the stage ends its segment
  __device__ __forceinline__ void enter(long long u) {
    seg_u = u;
    rt = static_cast<int>(u / KB);
    const long long e = static_cast<long long>(rt + 1) * KB;
    seg_e = e < u1 ? e : u1;
    kb = static_cast<int>(u - static_cast<long long>(rt) * KB);
    set_len();
  }
  __device__ __forceinline__ void set_len() {
    const long long left = seg_e - (static_cast<long long>(rt) * KB + kb);
    nblk = left < kGvBlk ? static_cast<int>(left) : kGvBlk;
    seg_end = left <= kGvBlk;
  }
  __device__ __forceinline__ void init(long long u0, long long u1_, int KB_) {
    u1 = u1_;
    KB = KB_;
    seg = 0;
    enter(u0);
  }
  __device__ __forceinline__ void next() {
    if (seg_end) {
      ++seg;
      if (seg_e < u1) enter(seg_e);
    } else {
      kb += kGvBlk;
      set_len();
    }
  }
};

__device__ __forceinline__ int gv_num_stages(long long u0, long long u1, int KB) {
  int n = 0;
  for (long long u = u0; u < u1;) {
    const int rt = static_cast<int>(u / KB);
    const long long e = static_cast<long long>(rt + 1) * KB < u1 ? static_cast<long long>(rt + 1) * KB
                                                                  : u1;
    n += static_cast<int>((e - u + kGvBlk - 1) / kGvBlk);
    u = e;
  }
  return n;
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool pred) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(gv_saddr(dst)), "l"(src),
               "r"(pred ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(gv_saddr(dst)), "l"(src),
               "r"(pred ? 16 : 0)
               : "memory");
}

// Shared-memory stage: the tokens' X chunk in B-fragment order, then every warp's packed codes
// and block scales in the order its lanes read them (conflict-free 8-byte loads).
template <int TT>
struct GvLayout {
  static constexpr int kX = kGvBlk * 4 * TT * 32 * 8;          // [blk][j][tt][lane] x 8 B
  static constexpr int kCodes = kGvWarps * 2 * kGvBlk * 32 * 8;  // [warp][h][blk][lane] x 8 B
  static constexpr int kAm = kGvWarps * 2 * kGvBlk * 8 * 4;      // [warp][h][blk][g] fp32
  static constexpr int kStage = kX + kCodes + kAm;
  static constexpr int kStages = TT <= 2 ? 4 : 3;
};

template <int TT>
__global__ void __launch_bounds__(kGvThreads, 2)
    nf4_gemv_fwd_kernel(const __nv_bfloat16* __restrict__ X, const uint8_t* __restrict__ q,
                        const float* __restrict__ absmax, const uint8_t* __restrict__ absmax_q8,
                        const float* __restrict__ absmax_scale, int dq, int M, int N, int K,
                        long long U, int max_seg, float* __restrict__ partial, Codebook cb) {
  using Lay = GvLayout<TT>;
  constexpr int S = Lay::kStages;
  constexpr int kMp = 8 * TT;  // padded tokens
  extern __shared__ __align__(16) uint8_t gv_smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int KB = K / 64;
  const long long u0 = U * blockIdx.x / gridDim.x;
  const long long u1 = U * (blockIdx.x + 1) / gridDim.x;
  const int nst = gv_num_stages(u0, u1, KB);

  Nf4Lut lut;
  nf4_build_lut(cb, 1.0f, lut);  // the unscaled codebook in bf16
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();

  // Two cursors walk the stage list: loads run S - 1 stages ahead of the compute.
  GvCursor cl, cc;
  cl.init(u0, u1, KB);
  cc.init(u0, u1, KB);
  auto load = [&](int i) {  // stage i == the stage cl points at
    if (i >= nst) return;
    uint8_t* st = gv_smem + (i % S) * Lay::kStage;
    // X chunk: 8-byte pieces (token, 4 consecutive k), zero past M or past the stage's blocks.
    for (int p = tid; p < kGvBlk * 4 * TT * 32; p += kGvThreads) {
      const int ln = p & 31, tt = (p >> 5) % TT, j = (p >> 5) / TT % 4, b = (p >> 5) / (TT * 4);
      const int tok = tt * 8 + (ln >> 2);
      const int k = (cl.kb + b) * 64 + 16 * (ln & 3) + 4 * j;
      const bool ok = tok < M && b < cl.nblk;
      cp_async8(st + static_cast<size_t>(p) * 8, X + (ok ? static_cast<long long>(tok) * K + k : 0),
                ok);
    }
    // Codes: 16-byte pieces = the 8-byte slices of lanes (g, t) and (g, t + 1).
    uint8_t* cs = st + Lay::kX;
    for (int p = tid; p < kGvWarps * 2 * kGvBlk * 16; p += kGvThreads) {
      const int pl = p & 15, b = (p >> 4) % kGvBlk, h = (p >> 4) / kGvBlk % 2,
                w = (p >> 4) / (kGvBlk * 2);
      const int gg = pl >> 1, tt2 = (pl & 1) * 2;  // lanes 4gg + tt2, +1
      const int row = cl.rt * kGvRows + w * 16 + gg + 8 * h;
      const bool ok = row < N && b < cl.nblk;
      const long long blk = static_cast<long long>(row) * KB + cl.kb + b;
      cp_async16(cs + ((static_cast<size_t>(w) * 2 + h) * kGvBlk + b) * 256 + (4 * gg + tt2) * 8,
                 q + (ok ? blk * 32 + 8 * tt2 : 0), ok);
    }
    // Block scales (fp32 absmax; the double-quantised form is read in the compute loop).
    if (!dq) {
      float* as = reinterpret_cast<float*>(st + Lay::kX + Lay::kCodes);
      for (int p = tid; p < kGvWarps * 2 * kGvBlk * 8; p += kGvThreads) {
        const int gg = p & 7, b = (p >> 3) % kGvBlk, h = (p >> 3) / kGvBlk % 2,
                  w = (p >> 3) / (kGvBlk * 2);
        const int row = cl.rt * kGvRows + w * 16 + gg + 8 * h;
        const bool ok = row < N && b < cl.nblk;
        cp_async4(as + p, absmax + (ok ? static_cast<long long>(row) * KB + cl.kb + b : 0), ok);
      }
    }
    cl.next();
  };

  float acc[TT][4];
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) acc[tt][0] = acc[tt][1] = acc[tt][2] = acc[tt][3] = 0.f;

#pragma unroll
  for (int p = 0; p < S - 1; ++p) {
    load(p);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int i = 0; i < nst; ++i) {
    asm volatile("cp.async.wait_group %0;" ::"n"(S - 2) : "memory");
    __syncthreads();
    load(i + S - 1);  // refill the slot every warp finished one iteration ago
    asm volatile("cp.async.commit_group;" ::: "memory");

    const uint8_t* st = gv_smem + (i % S) * Lay::kStage;
    const uint8_t* cs = st + Lay::kX + static_cast<size_t>(warp) * 2 * kGvBlk * 256;
    const float* as = reinterpret_cast<const float*>(st + Lay::kX + Lay::kCodes) +
                      warp * 2 * kGvBlk * 8;
#pragma unroll
    for (int b = 0; b < kGvBlk; ++b) {
      if (b >= cc.nblk) break;
      const uint2 c0 = *reinterpret_cast<const uint2*>(cs + (0 * kGvBlk + b) * 256 + lane * 8);
      const uint2 c1 = *reinterpret_cast<const uint2*>(cs + (1 * kGvBlk + b) * 256 + lane * 8);
      float am0, am1;
      if (!dq) {
        am0 = as[(0 * kGvBlk + b) * 8 + g];
        am1 = as[(1 * kGvBlk + b) * 8 + g];
      } else {
        const int r0 = cc.rt * kGvRows + warp * 16 + g;
        const long long blk0 = static_cast<long long>(r0) * KB + cc.kb + b;
        am0 = r0 < N ? nf4_block_absmax(absmax, absmax_q8, absmax_scale, dq, blk0) : 0.f;
        am1 = r0 + 8 < N ? nf4_block_absmax(absmax, absmax_q8, absmax_scale, dq, blk0 + 8LL * KB)
                         : 0.f;
      }
      // 16 codes per row: word 0 = codes 0..7, word 1 = codes 8..15 of this thread's slice.
      const uint4 r0w0 = nf4_lookup8(lut, c0.x), r0w1 = nf4_lookup8(lut, c0.y);
      const uint4 r1w0 = nf4_lookup8(lut, c1.x), r1w1 = nf4_lookup8(lut, c1.y);
      float tmp[TT][4];
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) tmp[tt][0] = tmp[tt][1] = tmp[tt][2] = tmp[tt][3] = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4& w0 = j < 2 ? r0w0 : r0w1;
        const uint4& w1 = j < 2 ? r1w0 : r1w1;
        uint32_t a[4];
        a[0] = (j & 1) ? w0.z : w0.x;  // row g,     codes 4j, 4j+1
        a[1] = (j & 1) ? w1.z : w1.x;  // row g + 8
        a[2] = (j & 1) ? w0.w : w0.y;  // row g,     codes 4j+2, 4j+3
        a[3] = (j & 1) ? w1.w : w1.y;  // row g + 8
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
          const uint2 bx = *reinterpret_cast<const uint2*>(
              st + ((static_cast<size_t>(b) * 4 + j) * TT + tt) * 256 + lane * 8);
          mma_bf16_16816(tmp[tt], a, bx.x, bx.y);
        }
      }
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        acc[tt][0] = fmaf(tmp[tt][0], am0, acc[tt][0]);
        acc[tt][1] = fmaf(tmp[tt][1], am0, acc[tt][1]);
        acc[tt][2] = fmaf(tmp[tt][2], am1, acc[tt][2]);
        acc[tt][3] = fmaf(tmp[tt][3], am1, acc[tt][3]);
      }
    }
    if (cc.seg_end) {
      // Partial sums of this segment -> slot (CTA, segment): [kMp tokens][128 rows] fp32.
      float* slot =
          partial + (static_cast<long long>(blockIdx.x) * max_seg + cc.seg) * kMp * kGvRows;
      const int r0 = warp * 16 + g;
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        const int c = tt * 8 + 2 * t;
        slot[c * kGvRows + r0] = acc[tt][0];
        slot[(c + 1) * kGvRows + r0] = acc[tt][1];
        slot[c * kGvRows + r0 + 8] = acc[tt][2];
        slot[(c + 1) * kGvRows + r0 + 8] = acc[tt][3];
        acc[tt][0] = acc[tt][1] = acc[tt][2] = acc[tt][3] = 0.f;
      }
    }
    cc.next();
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// h[tok, row] = bf16( sum of the row tile's partial slots, in CTA order
//                    + sum_j ext_act[tok, g, j] * ext_w[row, j] ),  g = the row tile's adapter
// Grid (row tiles, tokens), one row per thread.  Thread 0 finds the CTAs whose ranges cover
// the row tile (one 64-bit division each) and shares them through shared memory.
// With fold.part, the token's scaled rank-r activations are summed here from the
// down-projection's partials (and row tile 0 writes the saved bf16 sums) instead of being read
// from ext_act.
__global__ void __launch_bounds__(kGvRows) nf4_gemv_finalize(
    const float* __restrict__ partial, int M, int N, int K, long long U, int G, int max_seg,
    int Mp, const __nv_bfloat16* __restrict__ ext_act, const __nv_bfloat16* __restrict__ ext_w,
    int r, const RowGroups groups, __nv_bfloat16* __restrict__ out, const RankFold fold) {
  __shared__ int s_first, s_last, s_seg0;
  __shared__ float s_ea[kFoldMaxR];
  pdl_wait();  // the segment partial sums are complete
  pdl_trigger();
  const int KB = K / 64;
  const int rt = blockIdx.x, tok = blockIdx.y;
  if (fold.part) {
    for (int j = threadIdx.x; j < fold.R; j += blockDim.x) {
      float v = 0.f;
      for (int g = 0; g < fold.gsplit; ++g)
        v += __ldg(fold.part + (static_cast<long long>(g) * 128 + tok) * fold.R + j);
      if (rt == 0 && fold.saved)
        fold.saved[static_cast<long long>(tok) * fold.R + j] = __float2bfloat16_rn(v);
      s_ea[j] = __bfloat162float(__float2bfloat16_rn(fold.scale * v));
    }
  }
  if (threadIdx.x == 0) {
    const long long us = static_cast<long long>(rt) * KB, ue = us + KB;
    // CTA holding unit u: the largest b with floor(b U / G) <= u.
    s_first = static_cast<int>(((us + 1) * G - 1) / U);
    s_last = static_cast<int>((ue * G - 1) / U);
    s_seg0 = static_cast<int>(rt - (U * s_first / G) / KB);  // later CTAs start in this tile
  }
  __syncthreads();
  const int row = rt * kGvRows + threadIdx.x;
  if (row >= N) return;
  const int b_first = s_first, b_last = s_last, seg0 = s_seg0;
  const float* base = partial + static_cast<long long>(tok) * kGvRows + threadIdx.x;
  const long long slot_stride = static_cast<long long>(Mp) * kGvRows;
  float v = 0.f;
  for (int b = b_first; b <= b_last; b += 4) {
    float p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int bb = b + i;
      p[i] = bb <= b_last
                 ? __ldg(base + (static_cast<long long>(bb) * max_seg + (bb == b_first ? seg0 : 0)) *
                                    slot_stride)
                 : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (b + i <= b_last) v += p[i];
  }
  float e = 0.f;
  const __nv_bfloat16* ew = ext_w + static_cast<long long>(row) * r;
  if (fold.part) {
    const float* ea = s_ea + row_group(groups, rt * kGvRows) * r;
    for (int j = 0; j < r; j += 8) {
      const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(ew + j));
      const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&w4);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 w = __bfloat1622float2(w2[i]);
        e = fmaf(ea[j + 2 * i], w.x, e);
        e = fmaf(ea[j + 2 * i + 1], w.y, e);
      }
    }
    out[static_cast<long long>(tok) * N + row] = __float2bfloat16_rn(v + e);
    return;
  }
  const __nv_bfloat16* ea = ext_act + static_cast<long long>(tok) * groups.n * r +
                            row_group(groups, rt * kGvRows) * r;
  for (int j = 0; j < r; j += 8) {
    const uint4 a4 = *reinterpret_cast<const uint4*>(ea + j);
    const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(ew + j));
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a4);
    const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&w4);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a = __bfloat1622float2(a2[i]), w = __bfloat1622float2(w2[i]);
      e = fmaf(a.x, w.x, e);
      e = fmaf(a.y, w.y, e);
    }
  }
  out[static_cast<long long>(tok) * N + row] = __float2bfloat16_rn(v + e);
}

int g_gv_sm[64];

}  // namespace

GemvPlan gemv_plan(int M, int N, int K, int sm_count) {
  GemvPlan p;
  p.tt = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
  const long long U = static_cast<long long>((N + kGvRows - 1) / kGvRows) * (K / 64);
  const long long G = 2LL * sm_count < U ? 2LL * sm_count : U;
  p.units = U;
  p.grid = static_cast<int>(G);
  // A range of ceil(U / G) units touches at most ceil(that / KB) + 1 row tiles.
  const long long per = (U + G - 1) / G;
  p.max_seg = static_cast<int>((per + K / 64 - 1) / (K / 64)) + 1;
  p.partial_floats = static_cast<size_t>(p.grid) * p.max_seg * 8 * p.tt * kGvRows;
  p.smem = p.tt == 1 ? GvLayout<1>::kStages * GvLayout<1>::kStage
           : p.tt == 2 ? GvLayout<2>::kStages * GvLayout<2>::kStage
                       : GvLayout<4>::kStages * GvLayout<4>::kStage;
  return p;
}

cudaError_t launch_nf4_gemv_fwd(const __nv_bfloat16* X, const uint8_t* q, const float* absmax,
                                const uint8_t* absmax_q8, const float* absmax_scale, int dq, int M,
                                int N, int K, const __nv_bfloat16* ext_act,
                                const __nv_bfloat16* ext_w, int r, const RowGroups& groups,
                                __nv_bfloat16* out, float* partial, size_t partial_floats,
                                const Codebook& cb, cudaStream_t stream, const RankFold* fold) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_gv_sm[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_gv_sm[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int sms = g_gv_sm[dev] < kGemmMaxCtas ? g_gv_sm[dev] : kGemmMaxCtas;
  const GemvPlan p = gemv_plan(M, N, K, sms);
  if (M > 32 || !partial || p.partial_floats > partial_floats) return cudaErrorInvalidValue;
  switch (p.tt) {
    case 1:
      e = cudaFuncSetAttribute(nf4_gemv_fwd_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(p.smem));
      if (e != cudaSuccess) return e;
      e = launch_pdl(nf4_gemv_fwd_kernel<1>, dim3(p.grid), dim3(kGvThreads), p.smem, stream, 1,
                     X, q, absmax, absmax_q8, absmax_scale, dq, M, N, K, p.units, p.max_seg,
                     partial, cb);
      if (e != cudaSuccess) return e;
      break;
    case 2:
      e = cudaFuncSetAttribute(nf4_gemv_fwd_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(p.smem));
      if (e != cudaSuccess) return e;
      e = launch_pdl(nf4_gemv_fwd_kernel<2>, dim3(p.grid), dim3(kGvThreads), p.smem, stream, 1,
                     X, q, absmax, absmax_q8, absmax_scale, dq, M, N, K, p.units, p.max_seg,
                     partial, cb);
      if (e != cudaSuccess) return e;
      break;
    default:
      e = cudaFuncSetAttribute(nf4_gemv_fwd_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(p.smem));
      if (e != cudaSuccess) return e;
      e = launch_pdl(nf4_gemv_fwd_kernel<4>, dim3(p.grid), dim3(kGvThreads), p.smem, stream, 1,
                     X, q, absmax, absmax_q8, absmax_scale, dq, M, N, K, p.units, p.max_seg,
                     partial, cb);
      if (e != cudaSuccess) return e;
      break;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  RankFold f = {};
  if (fold) {
    if (!fold->part || fold->R > kFoldMaxR || fold->R != groups.n * r || fold->gsplit < 1 || M > 128)
      return cudaErrorInvalidValue;
    f = *fold;
  }
  return launch_pdl(nf4_gemv_finalize, dim3((N + kGvRows - 1) / kGvRows, M), dim3(kGvRows), 0,
                    stream, 1, static_cast<const float*>(partial), M, N, K, p.units, p.grid,
                    p.max_seg, 8 * p.tt, ext_act, ext_w, r, groups, out, f);
}

}  // namespace qlora

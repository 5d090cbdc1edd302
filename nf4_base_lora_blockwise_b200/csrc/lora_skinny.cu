// lora_skinny.cu -- the rank-r products around the dequant GEMM, on the tensor cores through
// warp-level mma.sync (bf16 in, fp32 accumulate).  They are skinny (r <= 128 columns) and
// bound by streaming the [M, C] activation once from HBM.
//
//   lora_down:  out[M, r] = in[M, C] . Wl^T      XA = X A^T (forward, kept for the backward)
//                                                dYB = dY B (backward)
//   lora_grad:  G[C, r]   = s in[M, C]^T . small[M, r]   dB = s dY^T XA,  dA = s (dYB^T X)
// With n adapters packed along the rows of B (q/k/v sharing X), dY B takes the block-diagonal
// B (adapter g's rows feed columns g r_g .. g r_g + r_g - 1 only) and dB takes, for adapter
// g's rows, the columns g r_g .. of XA.  Every 64-row step and 128-column tile lies in one
// adapter, so the zero blocks are skipped, not multiplied.
// ("Unsloth vs QLoRA vs Liger-Kernel", section 1 forward formula, section 2 hand-derived
// backward.)  Long reductions are split across CTAs into fixed-order fp32 partials that a
// second kernel sums in order, so results are deterministic run to run.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"

namespace qlora {

namespace {

constexpr int kTarget = 296;   // CTAs to aim for: two per SM on 148 SMs
constexpr int kWarps = 8;      // 256 threads per CTA
constexpr int kThreadsSk = 32 * kWarps;
constexpr int kBM = 16 * kWarps;  // lora_down: token rows per CTA (16 per warp)
constexpr int kBC = 64;        // lora_down: columns per pipeline step
constexpr int kGC = 16 * kWarps;  // lora_grad: columns (of `big`) per CTA
constexpr int kGM = 64;        // lora_grad: token rows per pipeline step
constexpr int kPad = 8;        // bf16 padding per smem row (keeps ldmatrix conflict-free)

// Pipeline depth: deeper for narrow ranks (small tiles), shallower when r is wide.
__host__ __device__ constexpr int stages_for(int R) { return R <= 64 ? 4 : 3; }
__device__ __forceinline__ void cp_async_wait_n(int n) {
  switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
  }
}

__device__ __forceinline__ uint32_t s_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool pred) {
  const int n = pred ? 16 : 0;  // n == 0 zero-fills the 16 destination bytes
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s_addr(dst)), "l"(src),
               "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait1() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait0() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s_addr(p)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(s_addr(p)));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(s_addr(p)));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// B fragments for n8 tiles [j0, j0 + 8 * NT) of a 16-deep k slice.
//   kn == false: smem rows are n (j), k contiguous      -> ldmatrix
//   kn == true : smem rows are k, n (j) contiguous      -> ldmatrix.trans
template <int NT, bool kn>
__device__ __forceinline__ void load_b_frags(uint32_t (&b)[NT][2], const __nv_bfloat16* base,
                                             int ld, int k0, int lane) {
#pragma unroll
  for (int t = 0; t + 1 < NT; t += 2) {
    uint32_t r[4];
    if (!kn) {
      const int j = t * 8 + (lane & 7) + ((lane >> 4) << 3);
      const int k = k0 + ((lane >> 3) & 1) * 8;
      ldsm_x4(r, base + j * ld + k);
    } else {
      const int k = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int j = t * 8 + (lane >> 4) * 8;
      ldsm_x4_t(r, base + k * ld + j);
    }
    b[t][0] = r[0];
    b[t][1] = r[1];
    b[t + 1][0] = r[2];
    b[t + 1][1] = r[3];
  }
  if (NT & 1) {
    constexpr int t = NT - 1;
    uint32_t r[2];
    const int l = lane & 15;
    if (!kn) {
      ldsm_x2(r, base + (t * 8 + (l & 7)) * ld + k0 + (l >> 3) * 8);
    } else {
      ldsm_x2_t(r, base + (k0 + (l & 7) + (l >> 3) * 8) * ld + t * 8);
    }
    b[t][0] = r[0];
    b[t][1] = r[1];
  }
}

// ------------------------------------------------------------------------------------------
// lora_down: grid (ceil(M/128), split).  8 warps, warp w owns rows 16w..16w+15 of the CTA's
// 128 token rows; a multi-stage cp.async pipeline streams 64-column slices of `in` (and of Wl).
// ------------------------------------------------------------------------------------------
template <int NT, bool kWrc>
__global__ void __launch_bounds__(kThreadsSk) lora_down_kernel(
    const __nv_bfloat16* __restrict__ in, int M, int C, const __nv_bfloat16* __restrict__ w,
    int rg, const RowGroups groups, float scale, __nv_bfloat16* __restrict__ saved,
    __nv_bfloat16* __restrict__ scaled, float* __restrict__ partial, int split) {
  constexpr int R = NT * 8;
  constexpr int S = stages_for(R);
  constexpr int kInLd = kBC + kPad;
  constexpr int kWRows = kWrc ? R : kBC;
  constexpr int kWLd = kWrc ? (kBC + kPad) : (R + kPad);
  extern __shared__ __align__(16) uint8_t dsm_down[];
  auto s_in = reinterpret_cast<__nv_bfloat16(*)[kBM * kInLd]>(dsm_down);
  auto s_w = reinterpret_cast<__nv_bfloat16(*)[kWRows * kWLd]>(
      dsm_down + S * kBM * kInLd * sizeof(__nv_bfloat16));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kBM;
  const int steps = C / kBC;
  const int sb = static_cast<int>((static_cast<long long>(steps) * blockIdx.y) / split);
  const int se = static_cast<int>((static_cast<long long>(steps) * (blockIdx.y + 1)) / split);
  const int n = se - sb;

  auto load = [&](int buf, int step) {
    const int c0 = step * kBC;
#pragma unroll
    for (int i = tid; i < kBM * (kBC / 8); i += kThreadsSk) {
      const int row = i >> 3, ch = i & 7;
      const int m = m0 + row;
      const bool ok = m < M;
      cp_async16(&s_in[buf][row * kInLd + ch * 8],
                 in + static_cast<long long>(ok ? m : 0) * C + c0 + ch * 8, ok);
    }
    if (kWrc) {  // A [r, C]: rows j, 64 contiguous c
      for (int i = tid; i < R * (kBC / 8); i += kThreadsSk) {
        const int j = i >> 3, ch = i & 7;
        cp_async16(&s_w[buf][j * kWLd + ch * 8], w + static_cast<long long>(j) * C + c0 + ch * 8,
                   true);
      }
    } else {  // B [C, rg]: rows c, rg contiguous, placed in columns g rg .. of the R-wide tile
      const int jg = row_group(groups, c0) * rg;
      for (int i = tid; i < kBC * (R / 8); i += kThreadsSk) {
        const int c = i / (R / 8), ch = i % (R / 8);
        const int j = ch * 8 - jg;
        const bool ok = j >= 0 && j < rg;  // other adapters' columns: zero-filled
        cp_async16(&s_w[buf][c * kWLd + ch * 8],
                   w + static_cast<long long>(c0 + c) * rg + (ok ? j : 0), ok);
      }
    }
  };

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  // Prologue: S-1 slices in flight (empty groups keep the group count uniform).
#pragma unroll
  for (int p = 0; p < S - 1; ++p) {
    if (p < n) load(p, sb + p);
    cp_async_commit();
  }
  for (int i = 0; i < n; ++i) {
    cp_async_wait_n(S - 2);
    __syncthreads();
    const int buf = i % S;
    // n8 column tiles this step feeds: all of them, or (B of one adapter) that adapter's.
    const int t_lo = kWrc ? 0 : row_group(groups, (sb + i) * kBC) * (rg / 8);
    const int t_hi = kWrc ? NT : t_lo + rg / 8;
#pragma unroll
    for (int kk = 0; kk < kBC / 16; ++kk) {
      uint32_t a[4];
      ldsm_x4(a, &s_in[buf][(warp * 16 + (lane & 15)) * kInLd + kk * 16 + (lane >> 4) * 8]);
      uint32_t b[NT][2];
      load_b_frags<NT, !kWrc>(b, s_w[buf], kWLd, kk * 16, lane);
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (t >= t_lo && t < t_hi) mma16816(acc[t], a, b[t][0], b[t][1]);
    }
    // Refill the slot consumed one iteration ago (every warp has passed this iteration's
    // barrier, so none still reads it).
    if (i + S - 1 < n) load((i + S - 1) % S, sb + i + S - 1);
    cp_async_commit();
  }
  cp_async_wait0();
  // Let the finalize kernel (launched as a programmatic dependent) be scheduled now; it
  // still waits for this whole grid's results before reading them.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int r_lo = m0 + warp * 16 + (lane >> 2);
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int col = t * 8 + (lane & 3) * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = r_lo + h * 8;
      if (m >= M) continue;
      const float v0 = acc[t][2 * h], v1 = acc[t][2 * h + 1];
      if (split == 1) {
        const long long o = static_cast<long long>(m) * R + col;
        if (saved)
          *reinterpret_cast<__nv_bfloat162*>(saved + o) = __floats2bfloat162_rn(v0, v1);
        *reinterpret_cast<__nv_bfloat162*>(scaled + o) =
            __floats2bfloat162_rn(scale * v0, scale * v1);
      } else {
        const long long o = (static_cast<long long>(blockIdx.y) * M + m) * R + col;
        *reinterpret_cast<float2*>(partial + o) = make_float2(v0, v1);
      }
    }
  }
}

// Fixed-order sum of the split partials [split, n] (n = M * r, a multiple of 8): each thread
// owns 4 consecutive values and issues all of its partial loads before summing, so the kernel
// costs about one memory round trip.
constexpr int kMaxSplit = 16;

__global__ void lora_down_finalize(const float* __restrict__ partial, int split, long long n,
                                   float scale, __nv_bfloat16* __restrict__ saved,
                                   __nv_bfloat16* __restrict__ scaled) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the split kernel's partials are done
  const long long i4 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i4 >= n) return;
  float4 p[kMaxSplit];
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s)
    if (s < split) p[s] = __ldg(reinterpret_cast<const float4*>(partial + s * n + i4));
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s)
    if (s < split) {
      v.x += p[s].x;
      v.y += p[s].y;
      v.z += p[s].z;
      v.w += p[s].w;
    }
  if (saved) {
    *reinterpret_cast<__nv_bfloat162*>(saved + i4) = __floats2bfloat162_rn(v.x, v.y);
    *reinterpret_cast<__nv_bfloat162*>(saved + i4 + 2) = __floats2bfloat162_rn(v.z, v.w);
  }
  *reinterpret_cast<__nv_bfloat162*>(scaled + i4) = __floats2bfloat162_rn(scale * v.x, scale * v.y);
  *reinterpret_cast<__nv_bfloat162*>(scaled + i4 + 2) =
      __floats2bfloat162_rn(scale * v.z, scale * v.w);
}

// ------------------------------------------------------------------------------------------
// lora_grad: grid (C/128, split).  8 warps, warp w owns columns c0+16w..c0+16w+15 of `big`;
// a multi-stage cp.async pipeline streams 64-token slices of `big` and `small`.
// ------------------------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kThreadsSk) lora_grad_kernel(
    const __nv_bfloat16* __restrict__ big, int M, int C, const __nv_bfloat16* __restrict__ small,
    const RowGroups groups, float scale, float* __restrict__ out, int out_cr,
    float* __restrict__ partial, int split) {
  constexpr int R = NT * 8;
  constexpr int S = stages_for(R);
  constexpr int kBigLd = kGC + kPad;
  constexpr int kSmLd = R + kPad;
  extern __shared__ __align__(16) uint8_t dsm_grad[];
  auto s_big = reinterpret_cast<__nv_bfloat16(*)[kGM * kBigLd]>(dsm_grad);
  auto s_sm = reinterpret_cast<__nv_bfloat16(*)[kGM * kSmLd]>(
      dsm_grad + S * kGM * kBigLd * sizeof(__nv_bfloat16));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = blockIdx.x * kGC;
  // small is [M, n R]; the tile's columns of `big` belong to one adapter, whose R columns it reads.
  const int ld_small = groups.n * R;
  const int j0 = row_group(groups, c0) * R;
  const int steps = (M + kGM - 1) / kGM;
  const int sb = static_cast<int>((static_cast<long long>(steps) * blockIdx.y) / split);
  const int se = static_cast<int>((static_cast<long long>(steps) * (blockIdx.y + 1)) / split);
  const int n = se - sb;

  auto load = [&](int buf, int step) {
    const int mb = step * kGM;
#pragma unroll
    for (int i = tid; i < kGM * (kGC / 8); i += kThreadsSk) {
      const int row = i / (kGC / 8), ch = i % (kGC / 8);
      const int m = mb + row;
      const int c = c0 + ch * 8;  // C is a multiple of 64, so a chunk is all in or all out
      const bool ok = m < M && c < C;
      cp_async16(&s_big[buf][row * kBigLd + ch * 8],
                 big + (ok ? static_cast<long long>(m) * C + c : 0), ok);
    }
    for (int i = tid; i < kGM * (R / 8); i += kThreadsSk) {
      const int row = i / (R / 8), ch = i % (R / 8);
      const int m = mb + row;
      const bool ok = m < M;
      cp_async16(&s_sm[buf][row * kSmLd + ch * 8],
                 small + static_cast<long long>(ok ? m : 0) * ld_small + j0 + ch * 8, ok);
    }
  };

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

#pragma unroll
  for (int p = 0; p < S - 1; ++p) {
    if (p < n) load(p, sb + p);
    cp_async_commit();
  }
  for (int i = 0; i < n; ++i) {
    cp_async_wait_n(S - 2);
    __syncthreads();
    const int buf = i % S;
#pragma unroll
    for (int kk = 0; kk < kGM / 16; ++kk) {
      // A = big^T: rows c, k = m; stored [m][c] -> transposed 8x8 loads.
      uint32_t a[4];
      const int q = lane >> 3, i8 = lane & 7;
      ldsm_x4_t(a, &s_big[buf][(kk * 16 + i8 + (q >> 1) * 8) * kBigLd + warp * 16 + (q & 1) * 8]);
      uint32_t b[NT][2];
      load_b_frags<NT, true>(b, s_sm[buf], kSmLd, kk * 16, lane);
#pragma unroll
      for (int t = 0; t < NT; ++t) mma16816(acc[t], a, b[t][0], b[t][1]);
    }
    if (i + S - 1 < n) load((i + S - 1) % S, sb + i + S - 1);
    cp_async_commit();
  }
  cp_async_wait0();
  // Let the finalize kernel (launched as a programmatic dependent) be scheduled now; it
  // still waits for this whole grid's results before reading them.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int c_lo = c0 + warp * 16 + (lane >> 2);
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int j = t * 8 + (lane & 3) * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = c_lo + h * 8;
      if (c >= C) continue;
      const float v0 = acc[t][2 * h], v1 = acc[t][2 * h + 1];
      if (split == 1) {
        if (out_cr) {
          *reinterpret_cast<float2*>(out + static_cast<long long>(c) * R + j) =
              make_float2(scale * v0, scale * v1);
        } else {
          out[static_cast<long long>(j) * C + c] = scale * v0;
          out[static_cast<long long>(j + 1) * C + c] = scale * v1;
        }
      } else {
        *reinterpret_cast<float2*>(partial + (static_cast<long long>(blockIdx.y) * C + c) * R + j) =
            make_float2(v0, v1);
      }
    }
  }
}

// Sum split partials [split, C, r] in order; write scale * sum as [C, r] (out_cr) or [r, C].
// Each thread owns 4 consecutive outputs and issues all of its partial loads first.
__global__ void lora_grad_finalize(const float* __restrict__ partial, int split, int C, int R,
                                   float scale, float* __restrict__ out, int out_cr) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the split kernel's partials are done
  const long long n = static_cast<long long>(C) * R;
  const long long i4 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i4 >= n) return;
  float4 p[kMaxSplit];
  if (out_cr) {  // i4 = c * R + j: 4 consecutive j of one c
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s)
      if (s < split) p[s] = __ldg(reinterpret_cast<const float4*>(partial + s * n + i4));
  } else {       // i4 = j * C + c: 4 consecutive c of one j (coalesced writes)
    const long long j = i4 / C, c = i4 % C;
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s)
      if (s < split) {
        const float* q = partial + s * n + c * R + j;
        p[s] = make_float4(__ldg(q), __ldg(q + R), __ldg(q + 2 * R), __ldg(q + 3 * R));
      }
  }
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s)
    if (s < split) {
      v.x += p[s].x;
      v.y += p[s].y;
      v.z += p[s].z;
      v.w += p[s].w;
    }
  *reinterpret_cast<float4*>(out + i4) =
      make_float4(scale * v.x, scale * v.y, scale * v.z, scale * v.w);
}

// Launches a 256-thread finalize kernel as a programmatic dependent of the kernel before it on
// the stream: it may be scheduled while that kernel's last CTAs run and waits for its results
// with griddepcontrol.wait.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), unsigned blocks, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

int clamp_split(int want, int maxv) { return want < 1 ? 1 : (want > maxv ? maxv : want); }

size_t down_smem(int R, bool w_rc) {
  const int w_rows = w_rc ? R : kBC;
  const int w_ld = w_rc ? (kBC + kPad) : (R + kPad);
  return stages_for(R) * sizeof(__nv_bfloat16) *
         (static_cast<size_t>(kBM) * (kBC + kPad) + static_cast<size_t>(w_rows) * w_ld);
}

size_t grad_smem(int R) {
  return stages_for(R) * sizeof(__nv_bfloat16) *
         (static_cast<size_t>(kGM) * (kGC + kPad) + static_cast<size_t>(kGM) * (R + kPad));
}

template <typename F>
cudaError_t launch_dyn(F kernel, dim3 grid, size_t smem, cudaStream_t stream) {
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  return e;
}

}  // namespace

DownPlan lora_down_plan(int M, int C, int r) {
  const int tiles = (M + kBM - 1) / kBM;  // 128-row tiles
  // As many splits as fit one wave of kTarget CTAs (a partial second wave would double the time).
  const int split = clamp_split(kTarget / tiles < kMaxSplit ? kTarget / tiles : kMaxSplit, C / kBC);
  DownPlan p;
  p.split = split;
  p.partial_floats = split > 1 ? static_cast<size_t>(split) * M * r : 0;
  return p;
}

GradPlan lora_grad_plan(int M, int C, int r) {
  const int tiles = (C + kGC - 1) / kGC;
  const int msteps = (M + kGM - 1) / kGM;
  const int split = clamp_split(kTarget / tiles < kMaxSplit ? kTarget / tiles : kMaxSplit, msteps);
  GradPlan p;
  p.split = split;
  p.partial_floats = split > 1 ? static_cast<size_t>(split) * C * r : 0;
  return p;
}

#define QLORA_DOWN_CASE(NTV)                                                                \
  case NTV:                                                                                 \
    if (w_is_rc) {                                                                          \
      e = launch_dyn(lora_down_kernel<NTV, true>, grid, smem, stream);                      \
      if (e != cudaSuccess) return e;                                                       \
      lora_down_kernel<NTV, true><<<grid, kThreadsSk, smem, stream>>>(                     \
          in, M, C, w, r, groups, scale, saved, scaled, partial, plan.split);               \
    } else {                                                                                \
      e = launch_dyn(lora_down_kernel<NTV, false>, grid, smem, stream);                     \
      if (e != cudaSuccess) return e;                                                       \
      lora_down_kernel<NTV, false><<<grid, kThreadsSk, smem, stream>>>(                    \
          in, M, C, w, r / groups.n, groups, scale, saved, scaled, partial, plan.split);    \
    }                                                                                       \
    break;

cudaError_t launch_lora_down(const __nv_bfloat16* in, int M, int C, const __nv_bfloat16* w,
                             bool w_is_rc, int r, const RowGroups& groups, float scale,
                             __nv_bfloat16* saved, __nv_bfloat16* scaled, float* partial,
                             const DownPlan& plan, cudaStream_t stream) {
  dim3 grid((M + kBM - 1) / kBM, plan.split);
  const size_t smem = down_smem(r, w_is_rc);
  cudaError_t e = cudaSuccess;
  switch (r / 8) {
    QLORA_DOWN_CASE(1)
    QLORA_DOWN_CASE(2)
    QLORA_DOWN_CASE(3)
    QLORA_DOWN_CASE(4)
    QLORA_DOWN_CASE(5)
    QLORA_DOWN_CASE(6)
    QLORA_DOWN_CASE(7)
    QLORA_DOWN_CASE(8)
    QLORA_DOWN_CASE(9)
    QLORA_DOWN_CASE(10)
    QLORA_DOWN_CASE(11)
    QLORA_DOWN_CASE(12)
    QLORA_DOWN_CASE(13)
    QLORA_DOWN_CASE(14)
    QLORA_DOWN_CASE(15)
    QLORA_DOWN_CASE(16)
    default:
      return cudaErrorInvalidValue;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || plan.split == 1) return e;
  const long long n = static_cast<long long>(M) * r;
  return launch_dependent(lora_down_finalize, static_cast<unsigned>((n / 4 + 255) / 256),
                          stream, static_cast<const float*>(partial), plan.split, n, scale,
                          saved, scaled);
}
#undef QLORA_DOWN_CASE

#define QLORA_GRAD_CASE(NTV)                                                               \
  case NTV:                                                                                \
    e = launch_dyn(lora_grad_kernel<NTV>, grid, smem, stream);                             \
    if (e != cudaSuccess) return e;                                                        \
    lora_grad_kernel<NTV><<<grid, kThreadsSk, smem, stream>>>(                            \
        big, M, C, small, groups, scale, out, out_cr ? 1 : 0, partial, plan.split);        \
    break;

cudaError_t launch_lora_grad(const __nv_bfloat16* big, int M, int C, const __nv_bfloat16* small,
                             int r, const RowGroups& groups, float scale, float* out, bool out_cr,
                             float* partial, const GradPlan& plan, cudaStream_t stream) {
  dim3 grid((C + kGC - 1) / kGC, plan.split);
  const size_t smem = grad_smem(r);
  cudaError_t e = cudaSuccess;
  switch (r / 8) {
    QLORA_GRAD_CASE(1)
    QLORA_GRAD_CASE(2)
    QLORA_GRAD_CASE(3)
    QLORA_GRAD_CASE(4)
    QLORA_GRAD_CASE(5)
    QLORA_GRAD_CASE(6)
    QLORA_GRAD_CASE(7)
    QLORA_GRAD_CASE(8)
    QLORA_GRAD_CASE(9)
    QLORA_GRAD_CASE(10)
    QLORA_GRAD_CASE(11)
    QLORA_GRAD_CASE(12)
    QLORA_GRAD_CASE(13)
    QLORA_GRAD_CASE(14)
    QLORA_GRAD_CASE(15)
    QLORA_GRAD_CASE(16)
    default:
      return cudaErrorInvalidValue;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || plan.split == 1) return e;
  const long long n = static_cast<long long>(C) * r;
  return launch_dependent(lora_grad_finalize, static_cast<unsigned>((n / 4 + 255) / 256),
                          stream, static_cast<const float*>(partial), plan.split, C, r, scale,
                          out, out_cr ? 1 : 0);
}
#undef QLORA_GRAD_CASE

}  // namespace qlora

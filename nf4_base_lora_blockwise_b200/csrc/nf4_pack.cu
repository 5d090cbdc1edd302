// nf4_pack.cu -- NF4 blockwise quantise + pack, the double-quantised absmax variant, and
// the dequant export.  One thread owns one 64-element block of a row: it reads the block's
// 128 bytes of bf16, takes the absmax, picks each code by counting codebook midpoints below
// w / absmax, and writes the 32 packed bytes (element 2j in the high nibble of byte j).
//
// "Unsloth vs QLoRA vs Liger-Kernel", FAQ "What is the difference between LoRA and QLoRA?"
// (base weights in 4-bit NormalFloat); "Speed up fine-tuning 2x", internals item 1.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "nf4_dequant.cuh"

namespace qlora {

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ void load_block(const __nv_bfloat16* __restrict__ W, long long blk,
                                           float (&w)[64]) {
  const uint4* src = reinterpret_cast<const uint4*>(W) + blk * 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 v = __ldg(src + i);
    w[8 * i + 0] = bf16_lo(v.x);
    w[8 * i + 1] = bf16_hi(v.x);
    w[8 * i + 2] = bf16_lo(v.y);
    w[8 * i + 3] = bf16_hi(v.y);
    w[8 * i + 4] = bf16_lo(v.z);
    w[8 * i + 5] = bf16_hi(v.z);
    w[8 * i + 6] = bf16_lo(v.w);
    w[8 * i + 7] = bf16_hi(v.w);
  }
}

__device__ __forceinline__ float block_max_abs(const float (&w)[64]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) m = fmaxf(m, fabsf(w[i]));
  return m;
}

// code = #{i : x > mid[i]}, x = fp32(w / a); the exact zero (7) when a == 0.
__device__ __forceinline__ uint32_t pick_code(float w, float a, const Codebook& cb) {
  if (a == 0.f) return 7u;
  const float x = __fdiv_rn(w, a);
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 15; ++i) c += (x > cb.mid[i]) ? 1u : 0u;
  return c;
}

__device__ __forceinline__ void store_codes(uint8_t* __restrict__ q, long long blk,
                                            const float (&w)[64], float a, const Codebook& cb) {
  uint32_t words[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t v = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t hi = pick_code(w[8 * j + 2 * b], a, cb);
      const uint32_t lo = pick_code(w[8 * j + 2 * b + 1], a, cb);
      v |= ((hi << 4) | lo) << (8 * b);
    }
    words[j] = v;
  }
  uint4* dst = reinterpret_cast<uint4*>(q + blk * 32);
  dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
  dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
}

// Single pass: absmax + codes (fp32 absmax variant).
__global__ void nf4_pack_kernel(const __nv_bfloat16* __restrict__ W, long long nblocks,
                                uint8_t* __restrict__ q, float* __restrict__ absmax,
                                const Codebook cb) {
  const long long blk = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blk >= nblocks) return;
  float w[64];
  load_block(W, blk, w);
  const float a = block_max_abs(w);
  absmax[blk] = a;
  store_codes(q, blk, w, a, cb);
}

// Double-quant pass 1: first-level absmax only.
__global__ void nf4_absmax_kernel(const __nv_bfloat16* __restrict__ W, long long nblocks,
                                  float* __restrict__ absmax) {
  const long long blk = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blk >= nblocks) return;
  float w[64];
  load_block(W, blk, w);
  absmax[blk] = block_max_abs(w);
}

// Double-quant pass 2: one warp per group of 256 absmax values.
// scale = fp32(max / 255); q8 = clamp(rint(fp32(absmax / scale)), 0, 255) (q8 = 0 if scale 0).
__global__ void nf4_absmax_dq_kernel(const float* __restrict__ absmax, long long nblocks,
                                     uint8_t* __restrict__ q8, float* __restrict__ scale) {
  const long long grp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long ngroups = (nblocks + 255) >> 8;
  if (grp >= ngroups) return;
  const long long b0 = grp << 8;
  float v[8];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long long b = b0 + lane + 32 * i;
    v[i] = (b < nblocks) ? absmax[b] : 0.f;
    m = fmaxf(m, v[i]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  const float s = __fdiv_rn(m, 255.f);
  if (lane == 0) scale[grp] = s;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long long b = b0 + lane + 32 * i;
    if (b >= nblocks) continue;
    int c = 0;
    if (s != 0.f) {
      c = __float2int_rn(__fdiv_rn(v[i], s));
      c = c < 0 ? 0 : (c > 255 ? 255 : c);
    }
    q8[b] = static_cast<uint8_t>(c);
  }
}

// Double-quant pass 3: codes chosen with the effective absmax fp32(q8 * scale).
__global__ void nf4_pack_dq_kernel(const __nv_bfloat16* __restrict__ W, long long nblocks,
                                   uint8_t* __restrict__ q, const uint8_t* __restrict__ q8,
                                   const float* __restrict__ scale, const Codebook cb) {
  const long long blk = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blk >= nblocks) return;
  float w[64];
  load_block(W, blk, w);
  const float a = __fmul_rn(static_cast<float>(q8[blk]), scale[blk >> 8]);
  store_codes(q, blk, w, a, cb);
}

// Dequant export: the GEMM's table-lookup routine applied to whole blocks.
__global__ void nf4_dequant_kernel(const uint8_t* __restrict__ q, const float* __restrict__ absmax,
                                   const uint8_t* __restrict__ q8, const float* __restrict__ scale,
                                   int dq, long long nblocks, __nv_bfloat16* __restrict__ out,
                                   const Codebook cb) {
  const long long blk = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blk >= nblocks) return;
  const float a = nf4_block_absmax(absmax, q8, scale, dq, blk);
  Nf4Lut lut;
  nf4_build_lut(cb, a, lut);
  const uint4* src = reinterpret_cast<const uint4*>(q + blk * 32);
  const uint4 qa = __ldg(src);
  const uint4 qb = __ldg(src + 1);
  uint4* dst = reinterpret_cast<uint4*>(out) + blk * 8;
  dst[0] = nf4_lookup8(lut, qa.x);
  dst[1] = nf4_lookup8(lut, qa.y);
  dst[2] = nf4_lookup8(lut, qa.z);
  dst[3] = nf4_lookup8(lut, qa.w);
  dst[4] = nf4_lookup8(lut, qb.x);
  dst[5] = nf4_lookup8(lut, qb.y);
  dst[6] = nf4_lookup8(lut, qb.z);
  dst[7] = nf4_lookup8(lut, qb.w);
}

inline unsigned grid_for(long long n, int threads) {
  return static_cast<unsigned>((n + threads - 1) / threads);
}

}  // namespace

cudaError_t launch_nf4_pack(const __nv_bfloat16* W, int N, int K, int dq, uint8_t* q,
                            float* absmax, uint8_t* absmax_q8, float* absmax_scale,
                            const Codebook& cb, cudaStream_t stream) {
  const long long nblocks = static_cast<long long>(N) * (K / 64);
  const int T = 128;
  if (!dq) {
    nf4_pack_kernel<<<grid_for(nblocks, T), T, 0, stream>>>(W, nblocks, q, absmax, cb);
    return cudaGetLastError();
  }
  nf4_absmax_kernel<<<grid_for(nblocks, T), T, 0, stream>>>(W, nblocks, absmax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long ngroups = (nblocks + 255) / 256;
  nf4_absmax_dq_kernel<<<grid_for(ngroups * 32, 256), 256, 0, stream>>>(absmax, nblocks,
                                                                         absmax_q8, absmax_scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  nf4_pack_dq_kernel<<<grid_for(nblocks, T), T, 0, stream>>>(W, nblocks, q, absmax_q8,
                                                             absmax_scale, cb);
  return cudaGetLastError();
}

cudaError_t launch_nf4_dequant(const uint8_t* q, const float* absmax, const uint8_t* q8,
                               const float* scale, int dq, int N, int K, __nv_bfloat16* out,
                               const Codebook& cb, cudaStream_t stream) {
  const long long nblocks = static_cast<long long>(N) * (K / 64);
  const int T = 128;
  nf4_dequant_kernel<<<grid_for(nblocks, T), T, 0, stream>>>(q, absmax, q8, scale, dq, nblocks,
                                                             out, cb);
  return cudaGetLastError();
}

}  // namespace qlora

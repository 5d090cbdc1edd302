// swiglu.cu -- elementwise SwiGLU glue between the gate/up and down projections of the MLP
// workload: a = silu(g) * u, silu(g) = g * sigmoid(g), and its exact derivatives
//   dg = da * u * sig(g) * (1 + g * (1 - sig(g))),   du = da * g * sig(g).
// ("Unsloth vs QLoRA vs Liger-Kernel", section 2: the SwiGLU MLP is one of the
// hand-differentiated ops.)  fp32 math, bf16 in/out, 8 elements per thread per iteration.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace qlora {

namespace {

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 v;
  uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return v;
}

// a = silu(g) * u and its gradients, 8 elements at a time.
__device__ __forceinline__ void swiglu8(const float (&fg)[8], const float (&fu)[8],
                                        float (&fa)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) fa[k] = fg[k] * sigmoid_f(fg[k]) * fu[k];
}

__device__ __forceinline__ void swiglu_grad8(const float (&fg)[8], const float (&fu)[8],
                                             const float (&fd)[8], float (&og)[8],
                                             float (&ou)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float sg = sigmoid_f(fg[k]);
    og[k] = fd[k] * fu[k] * sg * (1.f + fg[k] * (1.f - sg));
    ou[k] = fd[k] * fg[k] * sg;
  }
}

__global__ void swiglu_fwd_kernel(const __nv_bfloat16* __restrict__ g,
                                  const __nv_bfloat16* __restrict__ u,
                                  __nv_bfloat16* __restrict__ a, int64_t n) {
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();
  const int64_t nv = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
       i += stride) {
    float fg[8], fu[8], fa[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(g) + i), fg);
    unpack8(__ldg(reinterpret_cast<const uint4*>(u) + i), fu);
    swiglu8(fg, fu, fa);
    reinterpret_cast<uint4*>(a)[i] = pack8(fa);
  }
  for (int64_t i = nv * 8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride) {
    const float x = __bfloat162float(g[i]);
    a[i] = __float2bfloat16_rn(x * sigmoid_f(x) * __bfloat162float(u[i]));
  }
}

__global__ void swiglu_bwd_kernel(const __nv_bfloat16* __restrict__ g,
                                  const __nv_bfloat16* __restrict__ u,
                                  const __nv_bfloat16* __restrict__ da,
                                  __nv_bfloat16* __restrict__ dg, __nv_bfloat16* __restrict__ du,
                                  int64_t n) {
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();
  const int64_t nv = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
       i += stride) {
    float fg[8], fu[8], fd[8], og[8], ou[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(g) + i), fg);
    unpack8(__ldg(reinterpret_cast<const uint4*>(u) + i), fu);
    unpack8(__ldg(reinterpret_cast<const uint4*>(da) + i), fd);
    swiglu_grad8(fg, fu, fd, og, ou);
    reinterpret_cast<uint4*>(dg)[i] = pack8(og);
    reinterpret_cast<uint4*>(du)[i] = pack8(ou);
  }
  for (int64_t i = nv * 8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride) {
    const float x = __bfloat162float(g[i]), y = __bfloat162float(u[i]),
                d = __bfloat162float(da[i]);
    const float sg = sigmoid_f(x);
    dg[i] = __float2bfloat16_rn(d * y * sg * (1.f + x * (1.f - sg)));
    du[i] = __float2bfloat16_rn(d * x * sg);
  }
}

// Packed gate/up: gu [M, 2I] holds g in columns [0, I) and u in [I, 2I) of every row (the
// output of a packed gate/up layer); a and da are [M, I]; dgu [M, 2I] takes dg and du in the
// same places (the upstream gradient of that layer).  I % 8 == 0.  Blocks walk rows and
// threads the row's 8-element vectors, so no index is divided.
__global__ void swiglu_packed_fwd_kernel(const __nv_bfloat16* __restrict__ gu,
                                         __nv_bfloat16* __restrict__ a, int64_t M, int I) {
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();
  const int per_row = I / 8;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint4* g4 = reinterpret_cast<const uint4*>(gu + m * 2 * I);
    const uint4* u4 = reinterpret_cast<const uint4*>(gu + m * 2 * I + I);
    uint4* a4 = reinterpret_cast<uint4*>(a + m * I);
    for (int c = threadIdx.x; c < per_row; c += blockDim.x) {
      float fg[8], fu[8], fa[8];
      unpack8(__ldg(g4 + c), fg);
      unpack8(__ldg(u4 + c), fu);
      swiglu8(fg, fu, fa);
      a4[c] = pack8(fa);
    }
  }
}

__global__ void swiglu_packed_bwd_kernel(const __nv_bfloat16* __restrict__ gu,
                                         const __nv_bfloat16* __restrict__ da,
                                         __nv_bfloat16* __restrict__ dgu, int64_t M, int I) {
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();
  const int per_row = I / 8;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint4* g4 = reinterpret_cast<const uint4*>(gu + m * 2 * I);
    const uint4* u4 = reinterpret_cast<const uint4*>(gu + m * 2 * I + I);
    const uint4* d4 = reinterpret_cast<const uint4*>(da + m * I);
    uint4* dg4 = reinterpret_cast<uint4*>(dgu + m * 2 * I);
    uint4* du4 = reinterpret_cast<uint4*>(dgu + m * 2 * I + I);
    for (int c = threadIdx.x; c < per_row; c += blockDim.x) {
      float fg[8], fu[8], fd[8], og[8], ou[8];
      unpack8(__ldg(g4 + c), fg);
      unpack8(__ldg(u4 + c), fu);
      unpack8(__ldg(d4 + c), fd);
      swiglu_grad8(fg, fu, fd, og, ou);
      dg4[c] = pack8(og);
      du4[c] = pack8(ou);
    }
  }
}

// Rows per launch of the packed kernels: every row at once up to 16 blocks per SM.
unsigned grid_rows(int64_t M) {
  const int64_t cap = 148 * 16;
  return static_cast<unsigned>(M < 1 ? 1 : (M > cap ? cap : M));
}

unsigned grid_for(int64_t n) {
  const int64_t blocks = (n / 8 + 255) / 256;
  const int64_t cap = 148 * 16;
  return static_cast<unsigned>(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

}  // namespace

cudaError_t launch_swiglu_fwd(const __nv_bfloat16* g, const __nv_bfloat16* u, __nv_bfloat16* a,
                              int64_t n, cudaStream_t stream) {
  return launch_pdl(swiglu_fwd_kernel, dim3(grid_for(n)), dim3(256), 0, stream, 1, g, u, a, n);
}

cudaError_t launch_swiglu_bwd(const __nv_bfloat16* g, const __nv_bfloat16* u,
                              const __nv_bfloat16* da, __nv_bfloat16* dg, __nv_bfloat16* du,
                              int64_t n, cudaStream_t stream) {
  return launch_pdl(swiglu_bwd_kernel, dim3(grid_for(n)), dim3(256), 0, stream, 1, g, u, da, dg, du,
                    n);
}

cudaError_t launch_swiglu_packed_fwd(const __nv_bfloat16* gu, __nv_bfloat16* a, int64_t M, int I,
                                     cudaStream_t stream) {
  return launch_pdl(swiglu_packed_fwd_kernel, dim3(grid_rows(M)), dim3(256), 0, stream, 1, gu, a, M,
                    I);
}

cudaError_t launch_swiglu_packed_bwd(const __nv_bfloat16* gu, const __nv_bfloat16* da,
                                     __nv_bfloat16* dgu, int64_t M, int I, cudaStream_t stream) {
  return launch_pdl(swiglu_packed_bwd_kernel, dim3(grid_rows(M)), dim3(256), 0, stream, 1, gu, da,
                    dgu, M, I);
}

}  // namespace qlora

// cross_entropy.cu -- the row-wise cross-entropy of the LM head over one chunk of tokens:
// loss_m = logsumexp(z_m) - z_m[label_m] and, in place, dz_m = (softmax(z_m) - onehot(label_m))
// / count.  The linear + cross-entropy entry point runs the dequant GEMM for a chunk of tokens
// into a bounded logits buffer, this kernel, and the dX GEMM on the same buffer, so the
// [tokens x vocab] logits never exist at once ("Unsloth vs QLoRA vs Liger-Kernel", section 3,
// fused cross-entropy: chunked softmax reductions instead of the full logit tensor).
// A label outside [0, V) (e.g. -100) marks a token that takes no part: loss 0, gradient 0,
// not counted.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"

namespace qlora {

namespace {

constexpr int kCeThreads = 256;

__device__ __forceinline__ void unpack8_bf16(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Running (max, sum of exp(x - max)) pairs, combined as the online softmax does: eight values
// at a time, so the running pair is rescaled once per vector and the eight exponentials are
// independent of one another.
__device__ __forceinline__ void ms_add8(float& m, float& s, const float (&f)[8]) {
  float m8 = f[0];
#pragma unroll
  for (int k = 1; k < 8; ++k) m8 = fmaxf(m8, f[k]);
  if (m8 > m) {
    s *= __expf(m - m8);
    m = m8;
  }
  float t = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) t += __expf(f[k] - m);
  s += t;
}
__device__ __forceinline__ void ms_merge(float& m, float& s, float m2, float s2) {
  if (m2 > m) {
    s = s * expf(m - m2) + s2;
    m = m2;
  } else if (s2 > 0.f) {
    s += s2 * expf(m2 - m);
  }
}

// Valid-label count of the whole batch (labels in [0, V)), into *count.  One CTA.
__global__ void ce_count_kernel(const int* __restrict__ labels, int M, int V,
                                int* __restrict__ count) {
  __shared__ int part[kCeThreads];
  int c = 0;
  for (int i = threadIdx.x; i < M; i += kCeThreads) c += (labels[i] >= 0 && labels[i] < V) ? 1 : 0;
  part[threadIdx.x] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int i = 0; i < kCeThreads; ++i) t += part[i];
    *count = t;
  }
}

// One CTA per token row of the chunk.  z: [rows, V] bf16 (V % 8 == 0), overwritten by the
// gradient when write_grad; loss: [rows] fp32.
__global__ void __launch_bounds__(kCeThreads) ce_rows_kernel(__nv_bfloat16* __restrict__ z,
                                                             int V, const int* __restrict__ labels,
                                                             const int* __restrict__ count,
                                                             float* __restrict__ loss,
                                                             int write_grad) {
  __shared__ float sm_m[kCeThreads / 32], sm_s[kCeThreads / 32];
  __shared__ float s_lse;
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __nv_bfloat16* zr = z + static_cast<long long>(row) * V;
  const uint4* z4 = reinterpret_cast<const uint4*>(zr);
  const int nv = V / 8;

  float m = -INFINITY, s = 0.f;
  for (int i = tid; i < nv; i += kCeThreads) {
    float f[8];
    unpack8_bf16(z4[i], f);
    ms_add8(m, s, f);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xFFFFFFFFu, m, o);
    const float s2 = __shfl_xor_sync(0xFFFFFFFFu, s, o);
    ms_merge(m, s, m2, s2);
  }
  if (lane == 0) {
    sm_m[warp] = m;
    sm_s[warp] = s;
  }
  __syncthreads();
  if (tid == 0) {
    float mm = sm_m[0], ss = sm_s[0];
    for (int w = 1; w < kCeThreads / 32; ++w) ms_merge(mm, ss, sm_m[w], sm_s[w]);
    s_lse = mm + logf(ss);
  }
  __syncthreads();
  const float lse = s_lse;
  const int lab = labels[row];
  const int label = (lab >= 0 && lab < V) ? lab : -1;
  if (tid == 0) loss[row] = label >= 0 ? lse - __bfloat162float(zr[label]) : 0.f;
  if (!write_grad) return;
  __syncthreads();  // zr[label] is read before any thread overwrites it
  const int cnt = *count;
  const float scale = (label >= 0 && cnt > 0) ? 1.f / static_cast<float>(cnt) : 0.f;
  uint4* w4 = reinterpret_cast<uint4*>(zr);
  for (int i = tid; i < nv; i += kCeThreads) {
    float f[8];
    unpack8_bf16(w4[i], f);
    uint4 out;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int v0 = i * 8 + 2 * k;
      const float g0 = (__expf(f[2 * k] - lse) - (v0 == label ? 1.f : 0.f)) * scale;
      const float g1 = (__expf(f[2 * k + 1] - lse) - (v0 + 1 == label ? 1.f : 0.f)) * scale;
      const __nv_bfloat162 p = __floats2bfloat162_rn(g0, g1);
      ow[k] = *reinterpret_cast<const uint32_t*>(&p);
    }
    w4[i] = out;
  }
}

// loss = sum of the token losses / count (0 when no token counts), in fixed order.
__global__ void ce_mean_kernel(const float* __restrict__ token_loss, int M,
                               const int* __restrict__ count, float* __restrict__ out) {
  __shared__ float part[kCeThreads];
  float a = 0.f;
  for (int i = threadIdx.x; i < M; i += kCeThreads) a += token_loss[i];
  part[threadIdx.x] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < kCeThreads; ++i) t += part[i];
    const int c = *count;
    *out = c > 0 ? t / static_cast<float>(c) : 0.f;
  }
}

}  // namespace

cudaError_t launch_ce_count(const int* labels, int M, int V, int* count, cudaStream_t stream) {
  ce_count_kernel<<<1, kCeThreads, 0, stream>>>(labels, M, V, count);
  return cudaGetLastError();
}

cudaError_t launch_ce_rows(__nv_bfloat16* z, int rows, int V, const int* labels, const int* count,
                           float* loss, bool write_grad, cudaStream_t stream) {
  ce_rows_kernel<<<rows, kCeThreads, 0, stream>>>(z, V, labels, count, loss, write_grad ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_ce_mean(const float* token_loss, int M, const int* count, float* out,
                           cudaStream_t stream) {
  ce_mean_kernel<<<1, kCeThreads, 0, stream>>>(token_loss, M, count, out);
  return cudaGetLastError();
}

}  // namespace qlora

// qlora_gemm.cu -- the NF4 dequant GEMM on the 5th-generation tensor cores (tcgen05, TMEM
// accumulator, TMA operand loads) for sm_100a, with the LoRA up-projection fused as extra
// reduction steps.
//
// One kernel serves both large products of the layer ("Unsloth vs QLoRA vs Liger-Kernel",
// section 1 forward formula; section 2 hand-derived backward):
//   forward  h[M, N]  = X[M, K] . deq(W0)^T + (s XA)[M, r] . B^T
//   dX       dX[M, K] = dY[M, N] . deq(W0)  + (s dYB)[M, r] . A
// The tile is computed transposed, out^T[128 weight rows, bt tokens], so the weight is the
// MMA's A operand (M = 128 rows of W0 for the forward, 128 input features for dX) and the
// tokens are the MMA's N (16..256): small token counts still fill a full 128-row MMA.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: per 64-deep reduction step, the activation tile [bt x 64]
//               (128B swizzle, straight into the MMA layout) and the packed NF4 codes of the
//               weight tile; then the LoRA extension tiles (B or A, and s*XA or s*dYB).
//   warp 1      TMEM allocation; lane 0 issues tcgen05.mma and commits stages back.
//   warps 4-11  two dequant warpgroups taking alternate reduction steps: each thread turns
//               one 64-element block row segment (one absmax) into bf16 and writes it into
//               the weight-operand tile in the canonical 128B-swizzled layout -- K-major for
//               the forward, MN-major for dX (the transposed access costs no extra work).
//               Afterwards they drain the TMEM accumulator to global memory.
// The dequantised weight only ever exists in shared memory.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "nf4_dequant.cuh"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kThreads = 384;
constexpr uint32_t kWBytes = 16384;  // 128 rows x 64 bf16
constexpr uint32_t kQBytes = 4096;   // packed codes of the weight tile
constexpr int kRowsW = 128;          // MMA M
constexpr uint32_t kSmemLimit = 232448;

template <bool kTransW>
__global__ void __launch_bounds__(kThreads, 1)
    qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                      const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_ext_w,
                      const __grid_constant__ CUtensorMap tm_ext_act, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int S = args.stages;
  const int bt = args.bt;
  const uint32_t act_bytes = static_cast<uint32_t>(bt) * 128u;
  const uint32_t stage_bytes = kWBytes + act_bytes + kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);
  uint64_t* full = bars;           // TMA landed (count 1 + tx bytes)
  uint64_t* dqf = bars + S;        // dequantised tile written (count 4 warps)
  uint64_t* empty = bars + 2 * S;  // MMAs reading the stage done (tcgen05.commit)
  uint64_t* accf = bars + 3 * S;   // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 1);

  auto W = [&](int s) { return smem + s * stage_bytes; };
  auto ACT = [&](int s) { return smem + s * stage_bytes + kWBytes; };
  auto Q = [&](int s) { return smem + s * stage_bytes + kWBytes + act_bytes; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRowsW;
  const int tok0 = blockIdx.y * bt;
  const int kt = args.kt;
  const int total = kt + args.n_ext;
  const uint32_t ncols = bt <= 32 ? 32u : (bt <= 64 ? 64u : (bt <= 128 ? 128u : 256u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(dqf + s, 4);
      mbar_init(empty + s, 1);
    }
    mbar_init(accf, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_act);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_ext_w);
      tma_prefetch_desc(&tm_ext_act);
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        if (!mbar_wait(empty + s, ph ^ 1u, kErrWaitEmpty, args.err)) break;
        if (it < kt) {
          mbar_arrive_expect_tx(full + s, act_bytes + kQBytes);
          tma_load_2d(ACT(s), &tm_act, full + s, it * 64, tok0);
          if (!kTransW)
            tma_load_2d(Q(s), &tm_q, full + s, it * 32, row0);       // [128 rows, 32 B]
          else
            tma_load_2d(Q(s), &tm_q, full + s, row0 / 2, it * 64);   // [64 rows, 64 B]
        } else {
          const int e = it - kt;
          mbar_arrive_expect_tx(full + s, kWBytes + act_bytes);
          if (!kTransW) {
            tma_load_2d(W(s), &tm_ext_w, full + s, e * 64, row0);     // B [128 n, 64 j]
          } else {
            tma_load_2d(W(s), &tm_ext_w, full + s, row0, e * 64);     // A [64 j, 64 k]
            tma_load_2d(W(s) + 8192, &tm_ext_w, full + s, row0 + 64, e * 64);
          }
          tma_load_2d(ACT(s), &tm_ext_act, full + s, e * 64, tok0);
        }
        issued = it + 1;
      }
      // Every issued copy must land before the CTA may exit.
      for (int it = issued > S ? issued - S : 0; it < issued; ++it)
        mbar_wait(full + (it % S), static_cast<uint32_t>(it / S) & 1u, kErrWaitDrain, args.err);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, static_cast<uint32_t>(bt), kTransW ? 1u : 0u, 0u);
      for (int it = 0; it < total; ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        if (!mbar_wait(full + s, ph, kErrWaitFull, args.err)) break;
        if (it < kt && !mbar_wait(dqf + s, ph, kErrWaitDequant, args.err)) break;
        tc_fence_after();
        int nk = 4;
        if (it >= kt) {
          const int rem = args.r_pad16 - (it - kt) * 64;
          nk = (rem >= 64 ? 64 : rem) / 16;
        }
        const uint32_t wa = smem_u32(W(s));
        const uint32_t ba = smem_u32(ACT(s));
        for (int j = 0; j < nk; ++j) {
          const uint64_t adesc = kTransW ? smem_desc_sw128(wa + j * 2048u, 8192u, 1024u)
                                         : smem_desc_sw128(wa + j * 32u, 16u, 1024u);
          const uint64_t bdesc = smem_desc_sw128(ba + j * 32u, 16u, 1024u);
          umma_f16_ss(tmem_acc, adesc, bdesc, idesc, (it > 0 || j > 0) ? 1u : 0u);
        }
        umma_commit(empty + s);
      }
      umma_commit(accf);
      mbar_wait(accf, 0, kErrWaitDrain, args.err);  // all MMAs retired before teardown
    }
  } else if (warp >= 4) {
    // ------------------------------ dequant + epilogue ------------------------------------
    const int g = (warp - 4) >> 2;
    const int tid = threadIdx.x - 128 - 128 * g;  // 0..127
    uint32_t w_off, phase, q_off0, q_off1;
    long long blk0, blk_step;
    bool valid;
    if (!kTransW) {
      // Thread = weight row n: writes row `tid` of the K-major [128 x 64] operand tile.
      w_off = static_cast<uint32_t>(tid) * 128u;
      phase = static_cast<uint32_t>(tid) & 7u;
      const uint32_t sw = (static_cast<uint32_t>(tid) >> 2) & 1u;  // 32B swizzle of codes
      q_off0 = tid * 32u + ((0u ^ sw) << 4);
      q_off1 = tid * 32u + ((1u ^ sw) << 4);
      const int n = row0 + tid;
      valid = n < args.N;
      blk0 = static_cast<long long>(n) * args.kblocks;
      blk_step = 1;
    } else {
      // Thread = (64-wide output-feature segment kseg, weight row nl of the 64-row step):
      // writes K-row nl of MN-major atom column kseg.
      const int kseg = tid >> 6;
      const int nl = tid & 63;
      w_off = static_cast<uint32_t>(kseg) * 8192u + static_cast<uint32_t>(nl >> 3) * 1024u +
              static_cast<uint32_t>(nl & 7) * 128u;
      phase = static_cast<uint32_t>(nl) & 7u;
      const uint32_t sw = (static_cast<uint32_t>(nl) >> 1) & 3u;  // 64B swizzle of codes
      q_off0 = nl * 64u + (((2u * kseg + 0u) ^ sw) << 4);
      q_off1 = nl * 64u + (((2u * kseg + 1u) ^ sw) << 4);
      const int kb = row0 / 64 + kseg;
      valid = kb < args.kblocks;
      blk0 = static_cast<long long>(nl) * args.kblocks + kb;
      blk_step = 64LL * args.kblocks;
    }

    bool ok = true;
    for (int it = g; it < kt; it += 2) {
      const int s = it % S;
      const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
      const long long blk = blk0 + (kTransW ? blk_step * it : static_cast<long long>(it));
      const float am =
          valid ? nf4_block_absmax(args.absmax, args.absmax_q8, args.absmax_scale, args.dq, blk)
                : 0.f;
      const bool got = mbar_wait(full + s, ph, kErrWaitFull, args.err);
      if (!__all_sync(0xFFFFFFFFu, got)) {  // keep the warp converged
        ok = false;
        break;
      }
      const uint4 qa = *reinterpret_cast<const uint4*>(Q(s) + q_off0);
      const uint4 qb = *reinterpret_cast<const uint4*>(Q(s) + q_off1);
      Nf4Lut lut;
      nf4_build_lut(args.cb, am, lut);
      uint8_t* dst = W(s) + w_off;
      *reinterpret_cast<uint4*>(dst + ((0u ^ phase) << 4)) = nf4_lookup8(lut, qa.x);
      *reinterpret_cast<uint4*>(dst + ((1u ^ phase) << 4)) = nf4_lookup8(lut, qa.y);
      *reinterpret_cast<uint4*>(dst + ((2u ^ phase) << 4)) = nf4_lookup8(lut, qa.z);
      *reinterpret_cast<uint4*>(dst + ((3u ^ phase) << 4)) = nf4_lookup8(lut, qa.w);
      *reinterpret_cast<uint4*>(dst + ((4u ^ phase) << 4)) = nf4_lookup8(lut, qb.x);
      *reinterpret_cast<uint4*>(dst + ((5u ^ phase) << 4)) = nf4_lookup8(lut, qb.y);
      *reinterpret_cast<uint4*>(dst + ((6u ^ phase) << 4)) = nf4_lookup8(lut, qb.z);
      *reinterpret_cast<uint4*>(dst + ((7u ^ phase) << 4)) = nf4_lookup8(lut, qb.w);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(dqf + s);
    }

    // Epilogue: TMEM lane = weight row, column = token.  Group g takes 8-column chunks
    // c8 = g, g+2, ...
    const bool got = mbar_wait(accf, 0, kErrWaitAcc, args.err);
    tc_fence_after();
    ok = __all_sync(0xFFFFFFFFu, ok && got && *(volatile int*)args.err == 0);
    if (ok) {
      const int quad = warp & 3;
      const int row = row0 + quad * 32 + lane;
      const bool row_ok = row < args.rows_w;
      const uint32_t tbase = tmem_acc + (static_cast<uint32_t>(quad * 32) << 16);
      for (int c8 = g; c8 < bt / 8; c8 += 2) {
        uint32_t v[8];
        tmem_ld_32x32b_x8(tbase + static_cast<uint32_t>(c8 * 8), v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int tok = tok0 + c8 * 8 + j;
          if (row_ok && tok < args.M)
            args.out[static_cast<long long>(tok) * args.rows_w + row] =
                __float2bfloat16_rn(__uint_as_float(v[j]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, ncols);
  }
}

}  // namespace

int gemm_pick_bt(int M) {
  if (M >= 256) return 256;
  const int b = (M + 15) / 16 * 16;
  return b < 16 ? 16 : b;
}

int gemm_pick_stages(int bt) {
  const uint32_t stage = kWBytes + static_cast<uint32_t>(bt) * 128u + kQBytes;
  int s = static_cast<int>((kSmemLimit - 1024u - 256u) / stage);
  if (s > 8) s = 8;
  return s;
}

size_t gemm_smem_bytes(int bt, int stages) {
  const size_t stage = kWBytes + static_cast<size_t>(bt) * 128u + kQBytes;
  return 1024 + stages * stage + 256;
}

cudaError_t launch_qlora_gemm(bool trans_w, const GemmMaps& maps, const GemmArgs& args,
                              cudaStream_t stream) {
  const size_t smem = gemm_smem_bytes(args.bt, args.stages);
  dim3 grid((args.rows_w + kRowsW - 1) / kRowsW, (args.M + args.bt - 1) / args.bt);
  cudaError_t e;
  if (!trans_w) {
    e = cudaFuncSetAttribute(qlora_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    qlora_gemm_kernel<false><<<grid, kThreads, smem, stream>>>(maps.act, maps.q, maps.ext_w,
                                                               maps.ext_act, args);
  } else {
    e = cudaFuncSetAttribute(qlora_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    qlora_gemm_kernel<true><<<grid, kThreads, smem, stream>>>(maps.act, maps.q, maps.ext_w,
                                                              maps.ext_act, args);
  }
  return cudaGetLastError();
}

}  // namespace qlora

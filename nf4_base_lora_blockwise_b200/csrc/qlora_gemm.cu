// qlora_gemm.cu -- the NF4 dequant GEMM on the 5th-generation tensor cores (tcgen05, TMEM
// accumulators, TMA operand loads) for sm_100a, with the LoRA up-projection fused as extra
// reduction steps.
//
// One kernel serves both large products of the layer ("Unsloth vs QLoRA vs Liger-Kernel",
// section 1 forward formula; section 2 hand-derived backward):
//   forward  h[M, N]  = X[M, K] . deq(W0)^T + (s XA)[M, r] . B^T
//   dX       dX[M, K] = dY[M, N] . deq(W0)  + (s dYB)[M, r] . A
// A tile is computed transposed, out^T[128 weight rows, nh x bt tokens]: the weight is the MMA's
// A operand (M = 128 rows of W0 for the forward, 128 input features for dX) and the tokens are
// the MMA's N (bt = 16..256), so small token counts still fill a full 128-row MMA.  With more
// than 256 tokens a tile holds two 256-token halves (nh = 2) that share every dequantised
// weight tile: one dequantised element then feeds 1024 flops.
//
// Persistent CTAs (one per SM) walk the tile list.  Three shared-memory rings decouple the
// stages of a 64-deep reduction step so each one's latency hides behind the others:
//   Q ring  (2 groups x 4 x 4 KB) TMA -> dequant       packed NF4 codes of the weight tile
//   W ring  (2 groups x 2 x 16 KB) dequant -> MMA      bf16 weight operand (never in HBM)
//   X ring  (bt x 128 B slots)   TMA -> MMA            activation operand, 128B-swizzled
// TMEM holds two accumulators (ping-pong, epilogue of one tile overlaps the next mainloop)
// whenever they fit in its 512 columns, else one.
//
// Warp roles (768 threads):
//   warp 0      X producer: activation tiles, then the scaled rank-r tile (s*XA or s*dYB)
//   warp 1      TMEM allocation; lane 0 issues tcgen05.mma and commits slots back
//   warp 2      Q producer: packed code tiles
//   warp 3      idle
//   warps 4-7   epilogue: TMEM -> registers -> bf16 -> global
//   warps 8-23  two dequant groups of 8 warps; group g owns the pipeline steps it = g mod 2
//               (counted across tiles) and W slots 2g, 2g+1.  Each thread turns half of one
//               64-element block row segment (one absmax) into bf16 and writes it into the
//               weight-operand tile in the canonical 128B-swizzled layout -- K-major for the
//               forward, MN-major for dX (the transposed access costs no extra work).  On a LoRA
//               extension step the owning group TMA-loads the LoRA weight tile (B or A) into its
//               slot instead.  A waiting warp polls its barrier with one lane only.
//
// mbarrier waits test phase parity, which cannot tell phases two apart, and TMA copies may land
// out of order; so every ring slot has exactly one producer and one consumer that each visit
// its uses in order: W slots 2g, 2g+1 and Q slots 4g..4g+3 belong to dequant group g (the MMA,
// resp. the Q producer, is the other side), and the X ring has one producer and one consumer.
// A slot that threads read with ordinary loads and TMA then refills (the Q ring) needs a
// generic -> async proxy fence between the reads and the release of the slot; without it the
// refill was seen to overwrite codes not yet read, at large grids and long reductions.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "nf4_dequant.cuh"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kThreads = 768;
constexpr int kGroups = 2;                  // dequant groups (8 warps each)
constexpr int kGroupThreads = 256;
constexpr uint32_t kWBytes = 16384;         // 128 rows x 64 bf16
constexpr uint32_t kQBytes = 4096;          // packed codes of one weight tile step
constexpr int kRowsW = 128;                 // MMA M
constexpr uint32_t kSmemLimit = 232448;
constexpr int kQStages = 8;
constexpr int kWStages = 2 * kGroups;       // two W slots per group
constexpr int kQPerGroup = kQStages / kGroups;

struct Plan {
  int bt;        // tokens per half (MMA N)
  int nh;        // halves per tile
  int sx;        // X half-slots
  int nacc;      // TMEM accumulators (1 or 2)
  uint32_t acc_cols;  // TMEM columns per half accumulator
  uint32_t x_bytes;   // bytes per X half-slot
  size_t smem;
};

__host__ __device__ inline Plan make_plan(int bt, int nh) {
  Plan p;
  p.bt = bt;
  p.nh = nh;
  p.x_bytes = static_cast<uint32_t>(bt) * 128u;
  p.acc_cols = bt <= 16 ? 16u : (bt <= 32 ? 32u : (bt <= 64 ? 64u : (bt <= 128 ? 128u : 256u)));
  p.nacc = (2u * nh * p.acc_cols <= 512u) ? 2 : 1;
  const uint32_t fixed = 1024u + 512u + kQStages * kQBytes + kWStages * kWBytes;
  int sx = static_cast<int>((kSmemLimit - fixed) / p.x_bytes);
  if (sx > 8) sx = 8;
  p.sx = sx;
  p.smem = fixed + static_cast<size_t>(sx) * p.x_bytes;
  return p;
}

// Named barrier among the 256 threads of one dequant group (ids 1, 2).
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");
}

// W slot of pipeline step it: owner group it % 2, alternating between the group's two slots.
__device__ __forceinline__ int w_slot(int it) { return 2 * (it & 1) + ((it >> 1) & 1); }
__device__ __forceinline__ uint32_t w_par(int it) { return static_cast<uint32_t>(it >> 2) & 1u; }

template <bool kTransW>
__global__ void __launch_bounds__(kThreads, 1)
    qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                      const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_ext_w,
                      const __grid_constant__ CUtensorMap tm_ext_act, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const Plan P = make_plan(args.bt, args.nh);
  const int bt = P.bt, nh = P.nh, SX = P.sx;
  constexpr int SW = kWStages, SQ = kQStages;
  uint8_t* w_ring = smem;                     // SW x 16 KB
  uint8_t* q_ring = w_ring + SW * kWBytes;    // SQ x 4 KB
  uint8_t* x_ring = q_ring + SQ * kQBytes;    // SX x bt*128
  uint64_t* bars = reinterpret_cast<uint64_t*>(x_ring + SX * P.x_bytes);
  uint64_t* xfull = bars;
  uint64_t* xempty = xfull + SX;
  uint64_t* wfull = xempty + SX;
  uint64_t* wempty = wfull + SW;
  uint64_t* qfull = wempty + SW;
  uint64_t* qempty = qfull + SQ;
  uint64_t* accfull = qempty + SQ;   // [2]
  uint64_t* accempty = accfull + 2;  // [2]
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  auto WS = [&](int it) { return w_ring + w_slot(it) * kWBytes; };
  auto XS = [&](int hi) { return x_ring + (hi % SX) * P.x_bytes; };
  auto QS = [&](int qi) { return q_ring + (qi % SQ) * kQBytes; };
  auto par = [](int i, int s) { return static_cast<uint32_t>(i / s) & 1u; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kt = args.kt;
  const int total = kt + args.n_ext;
  const int tile_tokens = nh * bt;
  const int row_tiles = (args.rows_w + kRowsW - 1) / kRowsW;
  const int n_tiles = row_tiles * ((args.M + tile_tokens - 1) / tile_tokens);
  const int my_tiles =
      static_cast<int>(blockIdx.x) < n_tiles ? (n_tiles - 1 - static_cast<int>(blockIdx.x)) /
                                                       static_cast<int>(gridDim.x) + 1
                                             : 0;
  const uint32_t tile_cols = static_cast<uint32_t>(nh) * P.acc_cols;
  uint32_t ncols = static_cast<uint32_t>(P.nacc) * tile_cols;
  if (ncols < 32) ncols = 32;
  int* err = args.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      mbar_init(xfull + s, 1);
      mbar_init(xempty + s, 1);
    }
    for (int s = 0; s < SW; ++s) {
      mbar_init(wfull + s, 1);
      mbar_init(wempty + s, 1);
    }
    for (int s = 0; s < SQ; ++s) {
      mbar_init(qfull + s, 1);
      mbar_init(qempty + s, kGroupThreads / 32);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull + b, 1);
      mbar_init(accempty + b, 4);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ X producer -------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_act);
      tma_prefetch_desc(&tm_ext_act);
      int xs = 0;            // ring slot
      uint32_t xph = 0;      // use parity of that slot
      int issued = 0;
      bool ok = true;
      for (int lt = 0; ok && lt < my_tiles; ++lt) {
        const int t = blockIdx.x + lt * gridDim.x;
        const int tok0 = (t / row_tiles) * tile_tokens;
        for (int k = 0; ok && k < total; ++k) {
          for (int h = 0; h < nh; ++h) {
            if (!mbar_wait(xempty + xs, xph ^ 1u, kErrWaitEmpty, err, issued)) {
              ok = false;
              break;
            }
            uint8_t* dst = x_ring + xs * P.x_bytes;
            mbar_arrive_expect_tx(xfull + xs, P.x_bytes);
            if (k < kt)
              tma_load_2d(dst, &tm_act, xfull + xs, k * 64, tok0 + h * bt);
            else
              tma_load_2d(dst, &tm_ext_act, xfull + xs, (k - kt) * 64, tok0 + h * bt);
            ++issued;
            if (++xs == SX) {
              xs = 0;
              xph ^= 1u;
            }
          }
        }
      }
      // Every issued copy lands before the CTA may exit.
      for (int j = issued > SX ? issued - SX : 0; j < issued; ++j)
        mbar_wait(xfull + j % SX, par(j, SX), kErrWaitDrain, err, j);
    }
  } else if (warp == 2) {
    // ------------------------------ Q producer -------------------------------------------
    // Step it's code tile goes to the four-slot Q ring of its owner group g = it % 2, filled and
    // consumed strictly in order (slot 4g + (v & 3) for the group's v-th code tile), so each
    // slot has exactly one producer and one consumer even though TMA copies land out of order.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      int vq0 = 0, vq1 = 0;  // per-group code-tile counters (registers, not an array)
      bool ok = true;
      for (int lt = 0; ok && lt < my_tiles; ++lt) {
        const int t = blockIdx.x + lt * gridDim.x;
        const int row0 = (t % row_tiles) * kRowsW;
        for (int k = 0; k < kt; ++k) {
          const int it = lt * total + k;
          const int g = it & 1;
          const int v = g ? vq1 : vq0;
          const int slot = kQPerGroup * g + (v % kQPerGroup);
          const uint32_t u = static_cast<uint32_t>(v / kQPerGroup);
          if (!mbar_wait(qempty + slot, (u & 1u) ^ 1u, kErrWaitEmpty, err, it)) {
            ok = false;
            break;
          }
          vq0 += g == 0;
          vq1 += g == 1;
          mbar_arrive_expect_tx(qfull + slot, kQBytes);
          if (!kTransW)
            tma_load_2d(QS(slot), &tm_q, qfull + slot, k * 32, row0);      // [128 rows, 32 B]
          else
            tma_load_2d(QS(slot), &tm_q, qfull + slot, row0 / 2, k * 64);  // [64 rows, 64 B]
        }
      }
      // Every issued copy lands before the CTA may exit.
      for (int g = 0; g < kGroups; ++g) {
        const int n = g ? vq1 : vq0;
        for (int v = n > kQPerGroup ? n - kQPerGroup : 0; v < n; ++v)
          mbar_wait(qfull + kQPerGroup * g + (v % kQPerGroup),
                    static_cast<uint32_t>(v / kQPerGroup) & 1u, kErrWaitDrain, err, v);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer -------------------------------------------
    // One thread issues everything, so the loop keeps its per-step work to a few adds: ring
    // positions advance incrementally and the smem descriptors are precomputed, the start
    // address (bits 0-13, >> 4) being the only field that moves.
    if (lane == 0) {
      const uint32_t idesc =
          idesc_bf16_f32(128, static_cast<uint32_t>(bt), kTransW ? 1u : 0u, 0u);
      const uint64_t wdesc0 = kTransW ? smem_desc_sw128(smem_u32(w_ring), 8192u, 1024u)
                                      : smem_desc_sw128(smem_u32(w_ring), 16u, 1024u);
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(x_ring), 16u, 1024u);
      const uint64_t w_kstep = kTransW ? (2048u >> 4) : (32u >> 4);  // per 16-deep K slice
      const uint64_t x_kstep = 32u >> 4;
      const uint64_t w_slot_step = kWBytes >> 4;
      const uint64_t x_slot_step = P.x_bytes >> 4;
      const uint32_t half_cols = P.acc_cols;
      int it = 0, xs = 0;
      uint32_t xph = 0;
      bool ok = true;
      for (int lt = 0; ok && lt < my_tiles; ++lt) {
        const int ab = P.nacc == 2 ? (lt & 1) : 0;
        const int use = P.nacc == 2 ? (lt >> 1) : lt;
        if (!mbar_wait(accempty + ab, (static_cast<uint32_t>(use) & 1u) ^ 1u, kErrWaitAcc, err,
                       lt))
          break;
        tc_fence_after();
        const uint32_t dtm = tmem_base + static_cast<uint32_t>(ab) * tile_cols;
        for (int k = 0; k < total; ++k, ++it) {
          const int ws = w_slot(it);
          bool got = mbar_wait(wfull + ws, w_par(it), kErrWaitDequant, err, it);
          const int xs1 = xs + 1 == SX ? 0 : xs + 1;
          const uint32_t xph1 = xs + 1 == SX ? (xph ^ 1u) : xph;
          if (got) got = mbar_wait(xfull + xs, xph, kErrWaitFull, err, it);
          if (got && nh == 2) got = mbar_wait(xfull + xs1, xph1, kErrWaitFull, err, it);
          if (!got) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = wdesc0 + static_cast<uint64_t>(ws) * w_slot_step;
          const uint64_t bd0 = xdesc0 + static_cast<uint64_t>(xs) * x_slot_step;
          const uint64_t bd1 = xdesc0 + static_cast<uint64_t>(xs1) * x_slot_step;
          const uint32_t acc0 = k > 0 ? 1u : 0u;
          if (k < kt) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t acc = j > 0 ? 1u : acc0;
              umma_f16_ss(dtm, ad + j * w_kstep, bd0 + j * x_kstep, idesc, acc);
              if (nh == 2)
                umma_f16_ss(dtm + half_cols, ad + j * w_kstep, bd1 + j * x_kstep, idesc, acc);
            }
          } else {
            const int rem = args.r_pad16 - (k - kt) * 64;
            const int nk = (rem >= 64 ? 64 : rem) / 16;
            for (int j = 0; j < nk; ++j) {
              umma_f16_ss(dtm, ad + j * w_kstep, bd0 + j * x_kstep, idesc, 1u);
              if (nh == 2) umma_f16_ss(dtm + half_cols, ad + j * w_kstep, bd1 + j * x_kstep, idesc, 1u);
            }
          }
          umma_commit(xempty + xs);
          if (nh == 2) umma_commit(xempty + xs1);
          umma_commit(wempty + ws);
          if (nh == 2) {
            xs = xs1 + 1 == SX ? 0 : xs1 + 1;
            xph = xs1 + 1 == SX ? (xph1 ^ 1u) : xph1;
          } else {
            xs = xs1;
            xph = xph1;
          }
        }
        if (!ok) break;
        umma_commit(accfull + ab);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, kErrWaitDrain, err);  // every MMA retired before teardown
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------ epilogue ---------------------------------------------
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int t = blockIdx.x + lt * gridDim.x;
      const int ab = P.nacc == 2 ? (lt & 1) : 0;
      const int use = P.nacc == 2 ? (lt >> 1) : lt;
      bool got = true;
      if (lane == 0)
        got = mbar_wait_sleepy(accfull + ab, static_cast<uint32_t>(use) & 1u, kErrWaitAcc, err,
                               lt);
      if (!__shfl_sync(0xFFFFFFFFu, got, 0)) break;
      for (int i = 0; i < 64 && !mbar_try_wait(accfull + ab, static_cast<uint32_t>(use) & 1u); ++i) {
      }
      tc_fence_after();
      const int row = (t % row_tiles) * kRowsW + quad * 32 + lane;
      const int tok0 = (t / row_tiles) * tile_tokens;
      const bool row_ok = row < args.rows_w;
      for (int h = 0; h < nh; ++h) {
        const uint32_t tb = tmem_base + lane_base + static_cast<uint32_t>(ab) * tile_cols +
                            static_cast<uint32_t>(h) * P.acc_cols;
        for (int c8 = 0; c8 < bt / 8; ++c8) {
          uint32_t v[8];
          tmem_ld_32x32b_x8(tb + static_cast<uint32_t>(c8 * 8), v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int tok = tok0 + h * bt + c8 * 8 + j;
            if (row_ok && tok < args.M)
              args.out[static_cast<long long>(tok) * args.rows_w + row] =
                  __float2bfloat16_rn(__uint_as_float(v[j]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty + ab);
    }
  } else if (warp >= 8) {
    // ------------------------------ dequant groups ---------------------------------------
    const int g = (warp - 8) >> 3;
    const int tid = threadIdx.x - 256 - kGroupThreads * g;  // 0..255
    uint32_t w_off, phase, q_off;
    int seg_row, seg_kb, hf;  // weight row in the step / 64-block column / half of the segment
    if (!kTransW) {
      // Thread = (weight row n, half hf): writes half of row n of the K-major [128 x 64] tile.
      const int row = tid & 127;
      hf = tid >> 7;
      w_off = static_cast<uint32_t>(row) * 128u;
      phase = static_cast<uint32_t>(row) & 7u;
      const uint32_t sw = (static_cast<uint32_t>(row) >> 2) & 1u;  // 32B swizzle of codes
      q_off = row * 32u + ((static_cast<uint32_t>(hf) ^ sw) << 4);
      seg_row = row;
      seg_kb = 0;
    } else {
      // Thread = (64-wide output-feature segment kseg, weight row nl of the 64-row step, half
      // hf): writes half of K-row nl of MN-major atom column kseg.
      const int nl = tid & 63;
      const int kseg = (tid >> 6) & 1;
      hf = tid >> 7;
      w_off = static_cast<uint32_t>(kseg) * 8192u + static_cast<uint32_t>(nl >> 3) * 1024u +
              static_cast<uint32_t>(nl & 7) * 128u;
      phase = static_cast<uint32_t>(nl) & 7u;
      const uint32_t sw = (static_cast<uint32_t>(nl) >> 1) & 3u;  // 64B swizzle of codes
      q_off = nl * 64u + (((2u * kseg + static_cast<uint32_t>(hf)) ^ sw) << 4);
      seg_row = nl;
      seg_kb = kseg;
    }
    const uint32_t c0 = 4u * static_cast<uint32_t>(hf);  // first 16-byte chunk of this half
    // Effective absmax of this thread's block at reduction step k of tile t (0 outside W0).
    auto absmax_at = [&](int t, int k) -> float {
      const int row0 = (t % row_tiles) * kRowsW;
      long long blk;
      if (!kTransW) {
        const int n = row0 + seg_row;
        if (n >= args.N) return 0.f;
        blk = static_cast<long long>(n) * args.kblocks + k;
      } else {
        const int kb = row0 / 64 + seg_kb;
        if (kb >= args.kblocks) return 0.f;
        blk = static_cast<long long>(k * 64 + seg_row) * args.kblocks + kb;
      }
      return nf4_block_absmax(args.absmax, args.absmax_q8, args.absmax_scale, args.dq, blk);
    };

    // Steps it = g, g + 2, ... of the CTA's pipeline (tile lt = it / total, k = it % total).
    // The block absmax is fetched one owned step ahead to hide its latency.  After a failed
    // wait the group keeps walking its steps (without waiting or writing) so that every
    // thread still meets the group barrier once per step.
    const int n_steps = my_tiles * total;
    int vq = 0;  // code tiles this group has consumed
    bool failed = false;
    int last_ext = -1;
    if (tid == 0) tma_prefetch_desc(&tm_ext_w);
    auto absmax_of_step = [&](int it) -> float {
      const int k = it % total;
      if (it >= n_steps || k >= kt) return 0.f;
      return absmax_at(blockIdx.x + (it / total) * gridDim.x, k);
    };
    float am = absmax_of_step(g);
    for (int it = g; it < n_steps; it += kGroups) {
      const int lt = it / total;
      const int k = it - lt * total;
      const float am_next = failed ? 0.f : absmax_of_step(it + kGroups);
      if (k < kt) {
        const int qslot = kQPerGroup * g + (vq % kQPerGroup);
        const uint32_t qpar = static_cast<uint32_t>(vq / kQPerGroup) & 1u;
        ++vq;
        if (!failed) failed = !mbar_wait_warp(qfull + qslot, qpar, kErrWaitFull, err, it);
        if (!failed) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(QS(qslot) + q_off);
          // The slot's next fill is a TMA write (async proxy): order this generic read before
          // it, or the refill can overwrite the codes before the read has taken them.
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(qempty + qslot);
          Nf4Lut lut;
          nf4_build_lut(args.cb, am, lut);
          const uint4 o0 = nf4_lookup8(lut, q4.x);
          const uint4 o1 = nf4_lookup8(lut, q4.y);
          const uint4 o2 = nf4_lookup8(lut, q4.z);
          const uint4 o3 = nf4_lookup8(lut, q4.w);
          failed = !mbar_wait_warp(wempty + w_slot(it), w_par(it) ^ 1u, kErrWaitEmpty, err, it);
          if (!failed) {
            uint8_t* dst = WS(it) + w_off;
            *reinterpret_cast<uint4*>(dst + (((c0 + 0u) ^ phase) << 4)) = o0;
            *reinterpret_cast<uint4*>(dst + (((c0 + 1u) ^ phase) << 4)) = o1;
            *reinterpret_cast<uint4*>(dst + (((c0 + 2u) ^ phase) << 4)) = o2;
            *reinterpret_cast<uint4*>(dst + (((c0 + 3u) ^ phase) << 4)) = o3;
            fence_proxy_async_smem();
          }
        }
        group_sync(g);
        if (tid == 0 && !failed) mbar_arrive(wfull + w_slot(it));
      } else if (tid < 32) {
        // Extension step: one thread waits for the slot and TMA-loads the LoRA weight tile.
        if (lane == 0 && !failed) {
          const int e = k - kt;
          const int row0 = ((blockIdx.x + lt * gridDim.x) % row_tiles) * kRowsW;
          if (!mbar_wait(wempty + w_slot(it), w_par(it) ^ 1u, kErrWaitEmpty, err, it)) {
            failed = true;
          } else {
            uint64_t* bar = wfull + w_slot(it);
            mbar_arrive_expect_tx(bar, kWBytes);
            if (!kTransW) {
              tma_load_2d(WS(it), &tm_ext_w, bar, e * 64, row0);  // B [128 n, 64 j]
            } else {
              tma_load_2d(WS(it), &tm_ext_w, bar, row0, e * 64);  // A [64 j, 64 k]
              tma_load_2d(WS(it) + 8192, &tm_ext_w, bar, row0 + 64, e * 64);
            }
            last_ext = it;
          }
        }
        failed = __shfl_sync(0xFFFFFFFFu, failed, 0);
      }
      am = am_next;
    }
    // After a failure, copies this thread issued must land before the CTA exits.
    if (failed && last_ext >= 0)
      mbar_wait(wfull + w_slot(last_ext), w_par(last_ext), kErrWaitDrain, err, last_ext);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, ncols);
  }
}

int g_sm_count[64];

}  // namespace

int gemm_pick_bt(int M) {
  if (M >= 256) return 256;
  const int b = (M + 15) / 16 * 16;
  return b < 16 ? 16 : b;
}

int gemm_pick_halves(int M) { return M > 256 ? 2 : 1; }

int gemm_pick_stages(int bt) { return make_plan(bt, 1).sx; }

size_t gemm_smem_bytes(int bt, int nh) { return make_plan(bt, nh).smem; }

cudaError_t launch_qlora_gemm(bool trans_w, const GemmMaps& maps, const GemmArgs& args,
                              cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_sm_count[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = gemm_smem_bytes(args.bt, args.nh);
  const int row_tiles = (args.rows_w + kRowsW - 1) / kRowsW;
  const int tile_tokens = args.bt * args.nh;
  const int n_tiles = row_tiles * ((args.M + tile_tokens - 1) / tile_tokens);
  const int grid = n_tiles < g_sm_count[dev] ? n_tiles : g_sm_count[dev];
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

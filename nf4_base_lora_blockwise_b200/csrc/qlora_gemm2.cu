// qlora_gemm2.cu -- the NF4 dequant GEMM on CTA pairs: 5th-generation tensor-core MMAs with
// M = 256 (tcgen05.mma.cta_group::2) over two SMs, for problems with enough output tiles to
// fill the GPU whole.
//
// It computes the same products as qlora_gemm.cu ("Unsloth vs QLoRA vs Liger-Kernel", section 1
// forward formula; section 2 hand-derived backward):
//   forward  h[M, N]  = X[M, K] . deq(W0)^T + (s XA)[M, r] . B^T
//   dX       dX[M, K] = dY[M, N] . deq(W0)  + (s dYB)[M, r] . A
// on tiles of 256 weight rows x (nh x bt) tokens, shared by the two CTAs of a cluster:
//   * each CTA dequantises its own 128 weight rows into its W ring (the A operand's half);
//   * each CTA TMA-loads half of every token block (bt / 2 tokens) into its X ring (the B
//     operand's half), completing on the first CTA's barrier;
//   * one thread of the first CTA issues every MMA of the pair (M = 256, N = bt): each SM's
//     tensor core reads its own halves from its own shared memory, and each CTA's tensor memory
//     holds its 128 rows for all the tile's tokens;
//   * the commits release both CTAs' slots at once (tcgen05.commit multicast to the pair).
// Against one CTA per 128-row tile, each SM loads and feeds the tensor core half the activation
// bytes per step, so the shared-memory traffic per tensor-core cycle drops by about a third, and
// the X ring can be twice as deep in the same space.
//
// Warp roles and rings are those of the one-SM kernel (X producer, MMA issuer, Q producer,
// epilogue, two dequant groups of 8 warps), with these cross-CTA hand-offs:
//   full[s]      first CTA; completes when both CTAs' dequant groups have published step s's W
//                half and both CTAs' X halves have landed (4 arrivals + bytes)
//   wempty[s]    both CTAs; the MMA's multicast commit
//   accfull      both CTAs; the MMA's multicast commit at the end of a tile
//   accempty     first CTA; both CTAs' epilogue warps (8 arrivals)
// Every wait is bounded (2 s); a wait that runs out sets the device error word and the kernel
// winds down without further waits on the peer.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "nf4_dequant.cuh"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kThreads2 = 768;
constexpr int kGroups2 = 2;
constexpr int kGroupThreads2 = 256;
constexpr uint32_t kWBytes2 = 16384;  // 128 rows x 64 bf16 (this CTA's half of A)
constexpr uint32_t kQBytes2 = 4096;
constexpr int kRows2 = 128;           // weight rows per CTA
constexpr int kPairRows = 256;        // weight rows per pair tile
constexpr int kWStages2 = 4;
constexpr int kAmAhead2 = 3;

struct Plan2 {
  int bt;            // tokens per MMA (N), split bt / 2 per CTA
  int nh;            // MMAs (token blocks) per tile
  int dx, dxlog;     // X ring depth in steps
  int qlog;          // log2 of Q slots per dequant group
  uint32_t acc_cols; // TMEM columns per token block
  uint32_t x_bytes;  // bytes of one CTA's half of one token block (bt / 2 rows x 128 B)
  size_t smem;
};

__host__ __device__ inline Plan2 make_plan2(int bt, int nh) {
  Plan2 p;
  p.bt = bt;
  p.nh = nh;
  p.x_bytes = static_cast<uint32_t>(bt / 2) * 128u;
  p.acc_cols = static_cast<uint32_t>(bt);
  p.qlog = 2;
  p.dx = 4;
  p.dxlog = 2;
  const uint32_t sq = static_cast<uint32_t>(kGroups2) << p.qlog;
  const uint32_t fixed = 1024u + 1024u + sq * kQBytes2 + kWStages2 * kWBytes2;
  p.smem = fixed + static_cast<size_t>(p.dx) * p.nh * p.x_bytes;
  return p;
}

__device__ __forceinline__ int w_slot2(int it) { return 2 * (it & 1) + ((it >> 1) & 1); }
__device__ __forceinline__ uint32_t w_par2(int it) { return static_cast<uint32_t>(it >> 2) & 1u; }

__device__ __forceinline__ void group_sync2(int g) {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");
}

// (tile, reduction step) of a pair-local step index, advanced without dividing.
struct Cursor2 {
  int t, k;
  int row0;  // first weight row (dX: output feature) of this CTA in tile t
  int rp, rofs;  // row pair-tiles, this CTA's row offset in a pair tile
  __device__ __forceinline__ void set(int it, int pair, int n_pairs, int total, int row_pairs,
                                      int rank_rows) {
    rp = row_pairs;
    rofs = rank_rows;
    const int lt = it / total;
    t = pair + lt * n_pairs;
    k = it - lt * total;
    row0 = (t % rp) * kPairRows + rofs;
  }
  __device__ __forceinline__ void advance(int by, int n_pairs, int total) {
    k += by;
    if (k >= total) {
      while (k >= total) {
        k -= total;
        t += n_pairs;
      }
      row0 = (t % rp) * kPairRows + rofs;
    }
  }
};

template <bool kTransW>
__global__ void __launch_bounds__(kThreads2, 1)
    qlora_gemm2_kernel(const __grid_constant__ CUtensorMap tm_act,
                       const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_ext_w,
                       const __grid_constant__ CUtensorMap tm_ext_act, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const Plan2 P = make_plan2(args.bt, args.nh);
  const int bt = P.bt, nh = P.nh, DX = P.dx;
  const int half_bt = bt / 2;
  const int qper = 1 << P.qlog;
  const int SQ = kGroups2 * qper;
  constexpr int SW = kWStages2;
  uint8_t* w_ring = smem;
  uint8_t* q_ring = w_ring + SW * kWBytes2;
  uint8_t* x_ring = q_ring + SQ * kQBytes2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(x_ring + DX * nh * P.x_bytes);
  uint64_t* full = bars;             // [SW]   (used in the first CTA)
  uint64_t* wempty = full + SW;      // [SW]
  uint64_t* qfull = wempty + SW;     // [SQ]
  uint64_t* qempty = qfull + SQ;     // [SQ]
  uint64_t* accfull = qempty + SQ;   // [1]
  uint64_t* accempty = accfull + 1;  // [1]    (used in the first CTA)
  uint64_t* drain = accempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;
  auto WS = [&](int it) { return w_ring + w_slot2(it) * kWBytes2; };
  auto QS = [&](int qi) { return q_ring + qi * kQBytes2; };
  auto x_slot = [&](int it, int h) { return (it & (DX - 1)) * nh + h; };
  // The first CTA's barrier at the same offset (a shared::cluster address).
  auto lead_bar = [&](uint64_t* b) { return mapa_shared(smem_u32(b), 0u); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kt = args.kt;
  const int total = kt + args.n_ext;
  const int tile_tokens = nh * bt;
  const int row_pairs = (args.rows_w + kPairRows - 1) / kPairRows;
  const int n_tiles = row_pairs * ((args.M + tile_tokens - 1) / tile_tokens);
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int n_pairs = static_cast<int>(gridDim.x) >> 1;
  const int my_tiles = pair < n_tiles ? (n_tiles - 1 - pair) / n_pairs + 1 : 0;
  const int n_steps = my_tiles * total;
  // Step it of this pair: tile pair + (it / total) * n_pairs, reduction step it % total.
  auto tile_of = [&](int it) { return pair + (it / total) * n_pairs; };
  auto rows_of = [&](int t) { return (t % row_pairs) * kPairRows + static_cast<int>(rank) * kRows2; };

  const uint32_t tile_cols = static_cast<uint32_t>(nh) * P.acc_cols;
  uint32_t ncols = 32;
  while (ncols < tile_cols) ncols <<= 1;
  int* err = args.err;

  // Two token blocks: warp 1 of the first CTA issues block 0's MMAs and warp 3 block 1's, so
  // every commit barrier takes one (multicast) commit from each issuer.
  const uint32_t n_issuers = nh == 2 ? 2u : 1u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SW; ++s) {
      mbar_init(full + s, 4);
      mbar_init(wempty + s, n_issuers);
    }
    for (int s = 0; s < SQ; ++s) {
      mbar_init(qfull + s, 1);
      mbar_init(qempty + s, kGroupThreads2 / 32);
    }
    mbar_init(accfull, n_issuers);
    mbar_init(accempty, 8);
    mbar_init(drain, n_issuers);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, ncols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either arrives on the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // the previous kernel's outputs (activations, rank-r operand) are complete
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------ X producer (both CTAs) --------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_act);
      tma_prefetch_desc(&tm_ext_act);
      int issued = 0;
      Cursor2 cur;
      cur.set(0, pair, n_pairs, total, row_pairs, static_cast<int>(rank) * kRows2);
      for (int it = 0; it < n_steps; ++it, cur.advance(1, n_pairs, total)) {
        const int t = cur.t;
        const int k = cur.k;
        const int tok0 = (t / row_pairs) * tile_tokens + static_cast<int>(rank) * half_bt;
        const int eg = kTransW ? 0 : row_group(args.groups, cur.row0);
        // Step it reuses the X slots of step it - DX: wait until that step's MMAs are done.
        if (it >= DX &&
            !mbar_wait(wempty + w_slot2(it - DX), w_par2(it - DX), kErrWaitEmpty, err, it))
          break;
        const uint32_t fb = lead_bar(full + w_slot2(it));
        mbar_arrive_expect_tx_cl(fb, static_cast<uint32_t>(nh) * P.x_bytes);
        for (int h = 0; h < nh; ++h) {
          uint8_t* dst = x_ring + x_slot(it, h) * P.x_bytes;
          if (k < kt)
            tma_load_2d_pair(dst, &tm_act, fb, k * 64, tok0 + h * bt);
          else
            tma_load_3d_pair(dst, &tm_ext_act, fb, (k - kt) * 64, eg, tok0 + h * bt);
        }
        issued = it + 1;
      }
      // The copies land on the first CTA's barriers; this CTA's shared memory must outlive
      // them, which the closing cluster barrier (after the MMA thread's drain) guarantees.
      (void)issued;
    }
  } else if (warp == 2) {
    // ------------------------------ Q producer (both CTAs) --------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      int vq0 = 0, vq1 = 0;
      bool ok = true;
      Cursor2 cur;
      cur.set(0, pair, n_pairs, total, row_pairs, static_cast<int>(rank) * kRows2);
      for (int it = 0; ok && it < n_steps; ++it, cur.advance(1, n_pairs, total)) {
        const int k = cur.k;
        if (k >= kt) continue;
        const int row0 = cur.row0;
        const int g = it & 1;
        const int v = g ? vq1 : vq0;
        const int slot = (g << P.qlog) + (v & (qper - 1));
        const uint32_t u = static_cast<uint32_t>(v >> P.qlog);
        if (!mbar_wait(qempty + slot, (u & 1u) ^ 1u, kErrWaitEmpty, err, it)) {
          ok = false;
          break;
        }
        vq0 += g == 0;
        vq1 += g == 1;
        mbar_arrive_expect_tx(qfull + slot, kQBytes2);
        if (!kTransW)
          tma_load_2d(QS(slot), &tm_q, qfull + slot, k * 32, row0);
        else
          tma_load_2d(QS(slot), &tm_q, qfull + slot, row0 / 2, k * 64);
      }
      for (int g = 0; g < kGroups2; ++g) {
        const int n = g ? vq1 : vq0;
        for (int v = n > qper ? n - qper : 0; v < n; ++v)
          mbar_wait(qfull + (g << P.qlog) + (v & (qper - 1)),
                    static_cast<uint32_t>(v >> P.qlog) & 1u, kErrWaitDrain, err, v);
      }
    }
  } else if (warp == 1 || (warp == 3 && nh == 2)) {
    // ------------------------------ MMA issuers (first CTA) -------------------------------
    if (lane == 0 && lead) {
      const int h_lo = nh == 2 ? (warp == 1 ? 0 : 1) : 0;
      const int h_hi = nh == 2 ? h_lo + 1 : nh;
      const uint32_t idesc =
          idesc_bf16_f32(256, static_cast<uint32_t>(bt), kTransW ? 1u : 0u, 0u);
      const uint64_t wdesc0 = kTransW ? smem_desc_sw128(smem_u32(w_ring), 8192u, 1024u)
                                      : smem_desc_sw128(smem_u32(w_ring), 16u, 1024u);
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(x_ring), 16u, 1024u);
      const uint64_t w_kstep = kTransW ? (2048u >> 4) : (32u >> 4);
      const uint64_t x_kstep = 32u >> 4;
      const uint64_t w_slot_step = kWBytes2 >> 4;
      const uint64_t x_slot_step = P.x_bytes >> 4;
      bool ok = true;
      int it = 0;
      for (int tl = 0; ok && tl < my_tiles; ++tl) {
        if (!mbar_wait(accempty, (static_cast<uint32_t>(tl) & 1u) ^ 1u, kErrWaitAcc, err, tl))
          break;
        tc_fence_after();
        for (int k = 0; k < total; ++k, ++it) {
          const int ws = w_slot2(it);
          if (!mbar_wait(full + ws, w_par2(it), kErrWaitDequant, err, it)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = wdesc0 + static_cast<uint64_t>(ws) * w_slot_step;
          const uint64_t bd0 =
              xdesc0 + static_cast<uint64_t>((it & (DX - 1)) * nh) * x_slot_step;
          const int nk = k < kt ? 4 : ((args.r_pad16 - (k - kt) * 64 >= 64
                                            ? 64
                                            : args.r_pad16 - (k - kt) * 64) /
                                       16);
          for (int j = 0; j < nk; ++j) {
            const uint32_t acc = (k > 0 || j > 0) ? 1u : 0u;
            for (int h = h_lo; h < h_hi; ++h)
              umma_f16_ss_pair(tmem_base + static_cast<uint32_t>(h) * P.acc_cols,
                               ad + j * w_kstep,
                               bd0 + static_cast<uint64_t>(h) * x_slot_step + j * x_kstep, idesc,
                               acc);
          }
          umma_commit_pair(wempty + ws, 3);  // releases the W slot (and the X slots DX on)
        }
        if (!ok) break;
        umma_commit_pair(accfull, 3);
      }
      umma_commit_pair(drain, 1);
      mbar_wait(drain, 0, kErrWaitDrain, err);  // every MMA retired before teardown
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------ epilogue (both CTAs) ----------------------------------
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t ae = lead_bar(accempty);
    for (int tl = 0; tl < my_tiles; ++tl) {
      const int t = pair + tl * n_pairs;
      bool got = true;
      if (lane == 0) got = mbar_wait(accfull, static_cast<uint32_t>(tl) & 1u, kErrWaitAcc, err, tl);
      if (!__shfl_sync(0xFFFFFFFFu, got, 0)) break;
      __syncwarp();
      tc_fence_after();
      const int row = rows_of(t) + quad * 32 + lane;
      const int tok0 = (t / row_pairs) * tile_tokens;
      const bool row_ok = row < args.rows_w;
      for (int h = 0; h < nh; ++h) {
        const uint32_t tb = tmem_base + lane_base + static_cast<uint32_t>(h) * P.acc_cols;
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
      if (lane == 0) mbar_arrive_cl(ae);
    }
  } else if (warp >= 8) {
    // ------------------------------ dequant groups (both CTAs) ----------------------------
    const int g = (warp - 8) >> 3;
    const int tid = threadIdx.x - 256 - kGroupThreads2 * g;
    uint32_t w_off, phase, q_off;
    int seg_row, seg_kb, hf;
    if (!kTransW) {
      const int row = tid & 127;
      hf = tid >> 7;
      w_off = static_cast<uint32_t>(row) * 128u;
      phase = static_cast<uint32_t>(row) & 7u;
      const uint32_t sw = (static_cast<uint32_t>(row) >> 2) & 1u;
      q_off = row * 32u + ((static_cast<uint32_t>(hf) ^ sw) << 4);
      seg_row = row;
      seg_kb = 0;
    } else {
      const int nl = tid & 63;
      const int kseg = (tid >> 6) & 1;
      hf = tid >> 7;
      w_off = static_cast<uint32_t>(kseg) * 8192u + static_cast<uint32_t>(nl >> 3) * 1024u +
              static_cast<uint32_t>(nl & 7) * 128u;
      phase = static_cast<uint32_t>(nl) & 7u;
      const uint32_t sw = (static_cast<uint32_t>(nl) >> 1) & 3u;
      q_off = nl * 64u + (((2u * kseg + static_cast<uint32_t>(hf)) ^ sw) << 4);
      seg_row = nl;
      seg_kb = kseg;
    }
    const uint32_t c0 = 4u * static_cast<uint32_t>(hf);
    auto absmax_at = [&](int row0, int k) -> float {
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
    auto absmax_of_step = [&](int it) -> float {  // set-up only (divides)
      if (it >= n_steps) return 0.f;
      const int k = it % total;
      return k < kt ? absmax_at(rows_of(tile_of(it)), k) : 0.f;
    };
    const uint32_t fb0 = lead_bar(full);  // first CTA's full[0]; slot s at + 8 s
    int vq = 0;
    bool failed = false;
    if (tid == 0) tma_prefetch_desc(&tm_ext_w);
    static_assert(kGroups2 == 2 && kAmAhead2 == 3, "absmax prefetch walks owned steps");
    float am0 = absmax_of_step(g);
    float am1 = absmax_of_step(g + kGroups2);
    float am2 = absmax_of_step(g + 2 * kGroups2);
    Cursor2 cur, ahead;  // step it, and step it + kAmAhead2 * kGroups2
    cur.set(g, pair, n_pairs, total, row_pairs, static_cast<int>(rank) * kRows2);
    ahead.set(g + kAmAhead2 * kGroups2, pair, n_pairs, total, row_pairs,
              static_cast<int>(rank) * kRows2);
    for (int it = g; it < n_steps; it += kGroups2, cur.advance(kGroups2, n_pairs, total),
             ahead.advance(kGroups2, n_pairs, total)) {
      const int k = cur.k;
      const int row0 = cur.row0;
      const float am_next =
          (failed || it + kAmAhead2 * kGroups2 >= n_steps || ahead.k >= kt)
              ? 0.f
              : absmax_at(ahead.row0, ahead.k);
      const uint32_t fb = fb0 + 8u * static_cast<uint32_t>(w_slot2(it));
      if (k < kt) {
        const int qslot = (g << P.qlog) + (vq & (qper - 1));
        const uint32_t qpar = static_cast<uint32_t>(vq >> P.qlog) & 1u;
        ++vq;
        if (!failed) failed = !mbar_wait_warp(qfull + qslot, qpar, kErrWaitFull, err, it);
        if (!failed) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(QS(qslot) + q_off);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(qempty + qslot);
          Nf4Lut lut;
          nf4_build_lut(args.cb, am0, lut);
          const uint4 o0 = nf4_lookup8(lut, q4.x);
          const uint4 o1 = nf4_lookup8(lut, q4.y);
          const uint4 o2 = nf4_lookup8(lut, q4.z);
          const uint4 o3 = nf4_lookup8(lut, q4.w);
          failed = !mbar_wait_warp(wempty + w_slot2(it), w_par2(it) ^ 1u, kErrWaitEmpty, err, it);
          if (!failed) {
            uint8_t* dst = WS(it) + w_off;
            *reinterpret_cast<uint4*>(dst + (((c0 + 0u) ^ phase) << 4)) = o0;
            *reinterpret_cast<uint4*>(dst + (((c0 + 1u) ^ phase) << 4)) = o1;
            *reinterpret_cast<uint4*>(dst + (((c0 + 2u) ^ phase) << 4)) = o2;
            *reinterpret_cast<uint4*>(dst + (((c0 + 3u) ^ phase) << 4)) = o3;
            fence_proxy_async_smem();
          }
        }
        group_sync2(g);
        if (tid == 0 && !failed) mbar_arrive_cl(fb);
      } else {
        // Extension step: the lead thread TMA-loads this CTA's half of the LoRA weight tile.
        if (!failed)
          failed = !mbar_wait_warp(wempty + w_slot2(it), w_par2(it) ^ 1u, kErrWaitEmpty, err, it);
        group_sync2(g);
        if (tid == 0 && !failed) {
          const int e = k - kt;
          mbar_arrive_expect_tx_cl(fb, kWBytes2);
          if (!kTransW) {
            tma_load_2d_pair(WS(it), &tm_ext_w, fb, e * 64, row0);  // B [128 n, 64 j]
          } else {
            tma_load_2d_pair(WS(it), &tm_ext_w, fb, row0, e * 64);  // A [64 j, 64 k]
            tma_load_2d_pair(WS(it) + 8192, &tm_ext_w, fb, row0 + 64, e * 64);
          }
        }
      }
      am0 = am1;
      am1 = am2;
      am2 = am_next;
    }
  }

  tc_fence_before();
  // Neither CTA leaves (or frees its tensor memory) while the pair's MMAs, copies or remote
  // arrivals may still touch it: the first CTA's MMA thread drained every MMA above, and every
  // copy completed on a barrier some waiter saw, before its warps reach this barrier.
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, ncols);
  }
}

}  // namespace

size_t gemm2_smem_bytes(int bt, int nh) { return make_plan2(bt, nh).smem; }

GemmTile gemm2_pick_tile(int M, int rows_w, int steps_per_tile, int sm_count) {
  // Tokens per tile = 2 x bt (bt <= 256 per MMA, a multiple of 16, split bt / 2 per CTA): the
  // widest bt unless a narrower one shortens the busiest pair by at least 2 % under the
  // one-SM kernel's per-step cost model (its rounds of tiles, each with its exposed drain).
  GemmTile best{256, 2};
  const int pairs = (sm_count < kGemmMaxCtas ? sm_count : kGemmMaxCtas) / 2;
  if (pairs < 1) return best;
  const long long rp = (rows_w + kPairRows - 1) / kPairRows;
  auto cost = [&](int bt) {
    const int tt = 2 * bt;
    const long long tiles = rp * ((M + tt - 1) / tt);
    const long long rounds = (tiles + pairs - 1) / pairs;
    return static_cast<double>(rounds) * (steps_per_tile * (745.0 + 2.12 * tt) + 37.0 * tt);
  };
  const double wide = cost(256);
  double best_cost = wide;
  for (int bt = 240; bt >= 128; bt -= 16) {
    const double c = cost(bt);
    if (c < best_cost) {
      best_cost = c;
      best.bt = bt;
    }
  }
  if (best_cost > 0.98 * wide) best.bt = 256;
  return best;
}

bool gemm2_applies(int M, int rows_w, int steps_per_tile, int sm_count,
                   const RowGroups& groups) {
  // Whole pair tiles must fill every pair, and a pair tile must not straddle two adapters
  // (its MMA's extension operand is shared by both CTAs' rows).
  const GemmTile t = gemm2_pick_tile(M, rows_w, steps_per_tile, sm_count);
  const int pairs = (sm_count < kGemmMaxCtas ? sm_count : kGemmMaxCtas) / 2;
  const long long tiles =
      static_cast<long long>((rows_w + kPairRows - 1) / kPairRows) * ((M + 2 * t.bt - 1) / (2 * t.bt));
  if (pairs < 1 || tiles < pairs) return false;
  for (int i = 0; i + 1 < groups.n; ++i)
    if (groups.end[i] % kPairRows) return false;
  return true;
}

cudaError_t launch_qlora_gemm2(bool trans_w, const GemmMaps& maps, const GemmArgs& args,
                               cudaStream_t stream, int* launched) {
  *launched = 0;
  int sms = 0;
  cudaError_t e = gemm_device_sms(&sms);
  if (e != cudaSuccess) return e;
  const int pairs = (sms < kGemmMaxCtas ? sms : kGemmMaxCtas) / 2;
  const int tile_tokens = args.bt * args.nh;
  const long long tiles = static_cast<long long>((args.rows_w + kPairRows - 1) / kPairRows) *
                          ((args.M + tile_tokens - 1) / tile_tokens);
  const int grid = 2 * static_cast<int>(tiles < pairs ? tiles : pairs);
  const size_t smem = gemm2_smem_bytes(args.bt, args.nh);
  if (!trans_w) {
    e = cudaFuncSetAttribute(qlora_gemm2_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(qlora_gemm2_kernel<false>, dim3(grid), dim3(kThreads2), smem, stream, 2,
                   maps.act, maps.q, maps.ext_w, maps.ext_act, args);
  } else {
    e = cudaFuncSetAttribute(qlora_gemm2_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(qlora_gemm2_kernel<true>, dim3(grid), dim3(kThreads2), smem, stream, 2,
                   maps.act, maps.q, maps.ext_w, maps.ext_act, args);
  }
  if (e == cudaSuccess) *launched = 1;
  return e;
}

}  // namespace qlora

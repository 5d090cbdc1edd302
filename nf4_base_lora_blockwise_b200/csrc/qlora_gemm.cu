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
// the MMA's N (bt = 16..256), so small token counts still fill a full 128-row MMA.  With
// several adapters packed along W0's rows (q/k/v sharing X), a forward row tile takes the
// extension operand's columns of its own adapter, (s XA)[M, g, 0..r), so one launch computes
// every adapter's output ("Speed Up Fine-Tuning 2x with Unsloth", "How it works internally",
// item 3: several LoRA adapters packed into one tensor).  With more
// than 256 tokens a tile holds two 256-token halves (nh = 2) that share every dequantised
// weight tile: one dequantised element then feeds 1024 flops.
//
// Persistent CTAs (one per SM) walk the work in one of two modes:
//   tiles     (enough tiles to fill the GPU): CTA b takes tiles b, b + G, b + 2G, ... whole;
//   stream-K  (fewer tiles than SMs, i.e. few tokens or few output features): the tiles'
//             reduction steps, laid end to end, are cut into G equal contiguous ranges, one per
//             CTA.  A tile cut between CTAs leaves fp32 partial sums in the workspace (two slots
//             per CTA: the head segment of its range and the tail segment), and a finalize
//             kernel adds them in step order, so results do not depend on timing.
// Three shared-memory rings decouple the stages of a 64-deep reduction step so each one's
// latency hides behind the others:
//   Q ring  (2 groups x 4..16 x 4 KB) TMA -> dequant   packed NF4 codes of the weight tile
//   W ring  (2 groups x 2 x 16 KB) dequant -> MMA      bf16 weight operand (never in HBM)
//   X ring  (2-4 steps)          TMA -> MMA            activation operand, 128B-swizzled
// TMEM holds two accumulators (ping-pong, epilogue of one tile overlaps the next mainloop)
// whenever they fit in its 512 columns, else one.
//
// Warp roles (768 threads):
//   warp 0      X producer: activation tiles, then the scaled rank-r tile (s*XA or s*dYB)
//   warp 1      TMEM allocation; lane 0 issues tcgen05.mma and commits slots back
//   warp 2      Q producer: packed code tiles
//   warp 3      with two token halves, lane 0 issues half 1's MMAs (warp 1 then issues half 0's)
//   warps 4-7   epilogue: TMEM -> registers -> bf16 -> global
//   warps 8-23  two dequant groups of 8 warps; group g owns the pipeline steps it = g mod 2
//               (counted across tiles) and W slots 2g, 2g+1.  Each thread turns half of one
//               64-element block row segment (one absmax) into bf16 and writes it into the
//               weight-operand tile in the canonical 128B-swizzled layout -- K-major for the
//               forward, MN-major for dX (the transposed access costs no extra work).  On a LoRA
//               extension step the owning group TMA-loads the LoRA weight tile (B or A) into its
//               slot instead.  A waiting warp polls its barrier with one lane only.
//
// The MMA thread issues every tensor-core instruction of the CTA and is the pipeline's
// tightest resource, so it commits to one barrier per step (W empty): the X producer recycles
// X slots on the W ring's empty barriers instead of X barriers of their own.
//
// mbarrier waits test phase parity, which cannot tell phases two apart, and TMA copies may land
// out of order; so every ring slot has exactly one producer and one consumer that each visit
// its uses in order, and a waiter that only observes a barrier must gate its next phase:
// W slots 2g, 2g+1 and Q slots g*q..g*q+q-1 belong to dequant group g (the MMA, resp. the Q
// producer, is the other side); the X ring is filled by the X producer and consumed by the MMA
// thread, and an X slot is refilled only after the W slot of the step DX earlier is released
// (DX <= 4 steps, the W ring's reuse distance, so that release cannot move on without the new
// X tile).
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
constexpr int kWStages = 2 * kGroups;       // two W slots per group
constexpr int kAmAhead = 3;                 // owned steps the block absmax is fetched ahead

struct Plan {
  int bt;        // tokens per half (MMA N)
  int nh;        // halves per tile
  int dx;        // X ring depth in steps (2 or 4)
  int dxlog;     // log2(dx)
  int sx;        // X half-slots = dx * nh
  int nacc;      // TMEM accumulators (1 or 2)
  int qlog;      // log2 of the Q slots per dequant group
  uint32_t acc_cols;  // TMEM columns per half accumulator
  uint32_t x_bytes;   // bytes per X half-slot
  uint32_t rank_slot; // fused down-projection: bytes of one rank-operand tile (0: not fused)
  int rank_slots;     // tiles of its ring: dx (one per X ring step), 0 when it does not fit
  size_t smem;
};

constexpr uint32_t kSmemMax = 232448;  // dynamic shared memory of one CTA (227 KB)

// Small token tiles leave shared memory for a deeper code ring: with few tokens a step is
// short and the weight stream is the whole job, so more code tiles stay in flight.  A fused
// launch puts the rank operand's ring (one rank_slot-byte tile per X ring step) after the
// barriers, giving up code-ring depth if it would not fit otherwise.
__host__ __device__ inline Plan make_plan(int bt, int nh, uint32_t rank_slot = 0) {
  Plan p;
  p.bt = bt;
  p.nh = nh;
  p.x_bytes = static_cast<uint32_t>(bt) * 128u;
  // (Fused launches keep the accumulator at exactly bt columns: the rank window follows it.)
  p.acc_cols = rank_slot ? static_cast<uint32_t>(bt)
                         : (bt <= 16 ? 16u : (bt <= 32 ? 32u : (bt <= 64 ? 64u : (bt <= 128 ? 128u : 256u))));
  p.nacc = (2u * nh * p.acc_cols <= 512u) ? 2 : 1;
  p.qlog = bt <= 64 ? 4 : (bt <= 128 ? 3 : 2);
  // X slots are recycled on the W ring's empty barriers, which allows at most 4 steps of X
  // in flight.
  p.dx = nh == 2 ? 2 : 4;
  p.dxlog = nh == 2 ? 1 : 2;
  p.sx = p.dx * nh;
  p.rank_slot = rank_slot;
  p.rank_slots = 0;
  for (;;) {
    const uint32_t sq = static_cast<uint32_t>(kGroups) << p.qlog;
    const uint32_t fixed = 1024u + 1024u + sq * kQBytes + kWStages * kWBytes;
    p.smem = fixed + static_cast<size_t>(p.sx) * p.x_bytes;
    if (rank_slot == 0) break;
    const size_t ring = static_cast<size_t>(p.dx) * rank_slot;  // one tile per X ring step
    if (p.smem + ring <= kSmemMax || p.qlog <= 1) {
      p.rank_slots = p.smem + ring <= kSmemMax ? p.dx : 0;
      p.smem += static_cast<size_t>(p.rank_slots) * rank_slot;
      break;
    }
    --p.qlog;
  }
  return p;
}

// Where the CTA's it-th reduction step lies: tile t and step k within the tile.
struct StepMap {
  int total;       // steps per tile
  int streamk;     // 0: whole tiles b, b + G, ...; 1: contiguous range [g0, g0 + n_steps)
  long long g0;    // stream-K: first global step of this CTA
  int glu_rt;      // SwiGLU pairs: gate row tiles (half of row_tiles); 0: off
  int row_tiles;
  __device__ __forceinline__ void at(int it, int& t, int& k) const {
    if (streamk) {
      const long long g = g0 + it;
      t = static_cast<int>(g / total);
      k = static_cast<int>(g - static_cast<long long>(t) * total);
    } else {
      const int lt = it / total;
      if (glu_rt) {
        // Local tiles 2 i and 2 i + 1: pair q = b + i G, its gate row tile, then its up row tile.
        const int q = static_cast<int>(blockIdx.x) + (lt >> 1) * static_cast<int>(gridDim.x);
        const int tq = q / glu_rt;
        t = tq * row_tiles + (q - tq * glu_rt) + (lt & 1) * glu_rt;
      } else {
        t = static_cast<int>(blockIdx.x) + lt * static_cast<int>(gridDim.x);
      }
      k = it - lt * total;
    }
  }
};

// (tile, step) of a CTA-local step index that advances by kGroups at a time, without
// dividing (every tile has at least 2 steps, so one advance wraps at most once).
struct StepCursor {
  int t, k;
  int row0;  // first weight row (or output feature, dX) of tile t
  int lt, j, tq;  // SwiGLU pairs: local tile, gate row tile and token tile of its pair
  __device__ __forceinline__ void set(const StepMap& m, int it, int row_tiles) {
    m.at(it, t, k);
    row0 = (t % row_tiles) * kRowsW;
    if (m.glu_rt) {
      lt = it / m.total;
      const int q = static_cast<int>(blockIdx.x) + (lt >> 1) * static_cast<int>(gridDim.x);
      tq = q / m.glu_rt;
      j = q - tq * m.glu_rt;
    }
  }
  __device__ __forceinline__ void advance(const StepMap& m, int row_tiles) {
    if (m.glu_rt) {  // paired tiles: the next pair is G pairs on, walked without dividing
      k += 2;
      if (k >= m.total) {
        k -= m.total;
        ++lt;
        if ((lt & 1) == 0) {
          j += static_cast<int>(gridDim.x);
          while (j >= m.glu_rt) {
            j -= m.glu_rt;
            ++tq;
          }
        }
        const int rt = j + (lt & 1) * m.glu_rt;
        t = tq * row_tiles + rt;
        row0 = rt * kRowsW;
      }
      return;
    }
    k += 2;
    if (k >= m.total) {
      k -= m.total;
      t += m.streamk ? 1 : static_cast<int>(gridDim.x);
      row0 = (t % row_tiles) * kRowsW;
    }
  }
};

// First global step of stream-K CTA b: floor(b * T / G).
__host__ __device__ __forceinline__ long long sk_start(long long b, long long T, long long G) {
  return b * T / G;
}

// Named barrier among the 256 threads of one dequant group (ids 1, 2).
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");
}

// W slot of pipeline step it: owner group it % 2, alternating between the group's two slots.
__device__ __forceinline__ int w_slot(int it) { return 2 * (it & 1) + ((it >> 1) & 1); }
__device__ __forceinline__ uint32_t w_par(int it) { return static_cast<uint32_t>(it >> 2) & 1u; }

// ---------------------------------------------------------------------------------------------
// Fused rank-r down-projection (forward X A^T, dX dY B_bd) on the tensor cores.  A token tile's
// rank product is cut into 128-token windows, two per token half of 128 < bt <= 240 tokens:
// rows 0-127 of the half, and rows bt-128 .. bt-1, which writes rows 128 .. bt-1.  Window w is
// computed by the token tile's w-th tile, which runs in the first wave of tiles that reaches the
// token tile (the host checks), so every other tile of it starts no earlier.  On each activation
// step that tile's MMA thread adds four M = 128 MMAs: the window's rows of the activation tile
// already in shared memory (A operand, K-major) times the step's rank-operand tile (B operand:
// forward, A's n r rows [K-major]; dX, B's 64 rows [MN-major]), accumulated in TMEM columns past
// the tile's accumulator.  After the last activation step the epilogue warps read the window,
// write its rank values (bf16) and count it in the token tile's flag (one count per warp, four
// per window), which the extension step of every tile of that token tile waits on.
// ---------------------------------------------------------------------------------------------
constexpr int kRankMaxCols = 32;  // n r of a fused launch

struct RankWindow {
  int has;   // this tile computes a window
  int h;     // token half of the window
  int w0;    // first row of the window within the half
  int own0;  // first window row it writes (it writes rows own0 .. 127)
  int nwin;  // windows of the token tile
};

// Windows of a token half with `toks` valid tokens.
__host__ __device__ inline int half_windows(int toks) {
  return toks <= 0 ? 0 : (toks <= 128 ? 1 : 2);
}

__host__ __device__ inline RankWindow rank_window(int t, int row_tiles, int M, int bt, int nh) {
  RankWindow w;
  const int tt = bt * nh;
  const int tq = t / row_tiles;
  const int rt = t - tq * row_tiles;
  const int rest = M - tq * tt;
  const int n0 = half_windows(rest < bt ? rest : bt);
  const int n1 = nh == 2 ? half_windows(rest - bt < bt ? rest - bt : bt) : 0;
  w.nwin = n0 + n1;
  w.has = rt < w.nwin ? 1 : 0;
  w.h = rt < n0 ? 0 : 1;
  const int which = rt - (w.h ? n0 : 0);
  w.w0 = which == 0 ? 0 : bt - 128;
  w.own0 = which == 0 ? 0 : 256 - bt;
  return w;
}

// Tiles of token tile tq in the first wave of G tiles that reaches it.
__host__ __device__ inline int first_wave_tiles(int tq, int row_tiles, int G) {
  const long long t0 = static_cast<long long>(tq) * row_tiles;
  const long long wave_end = (t0 / G + 1) * G;
  return static_cast<int>(wave_end - t0 < row_tiles ? wave_end - t0 : row_tiles);
}

template <bool kTransW, bool kFused, bool kGlu = false>
__global__ void __launch_bounds__(kThreads, 1)
    qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                      const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_ext_w,
                      const __grid_constant__ CUtensorMap tm_ext_act,
                      const __grid_constant__ CUtensorMap tm_rank, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const Plan P = make_plan(args.bt, args.nh, kFused ? args.rank_slot : 0u);
  const int bt = P.bt, nh = P.nh, SX = P.sx, DX = P.dx, DXLOG = P.dxlog;
  const int qper = 1 << P.qlog;          // Q slots per dequant group
  const int SQ = kGroups * qper;
  constexpr int SW = kWStages;
  uint8_t* w_ring = smem;                     // SW x 16 KB
  uint8_t* q_ring = w_ring + SW * kWBytes;    // SQ x 4 KB
  uint8_t* x_ring = q_ring + SQ * kQBytes;    // SX x bt*128
  uint64_t* bars = reinterpret_cast<uint64_t*>(x_ring + SX * P.x_bytes);
  uint64_t* xfull = bars;
  uint64_t* wfull = xfull + SX;
  uint64_t* wempty = wfull + SW;
  uint64_t* qfull = wempty + SW;
  uint64_t* qempty = qfull + SQ;
  uint64_t* accfull = qempty + SQ;   // [2]
  uint64_t* accempty = accfull + 2;  // [2]
  uint64_t* drain = accempty + 2;
  uint64_t* rank_full = drain + 1;  // fused: the window's MMAs have retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rank_full + 1);
  uint8_t* rank_ring = x_ring + SX * P.x_bytes + 1024;  // fused: DX rank-operand tiles

  auto WS = [&](int it) { return w_ring + w_slot(it) * kWBytes; };
  auto QS = [&](int qi) { return q_ring + qi * kQBytes; };
  // X half-slot of step it, half h, and the parity of that use.
  auto x_slot = [&](int it, int h) { return (it & (DX - 1)) * nh + h; };
  auto x_par = [&](int it) { return static_cast<uint32_t>(it >> DXLOG) & 1u; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kt = args.kt;
  const int total = kt + args.n_ext;
  const int tile_tokens = nh * bt;
  const int row_tiles = (args.rows_w + kRowsW - 1) / kRowsW;
  const int n_tiles = row_tiles * ((args.M + tile_tokens - 1) / tile_tokens);

  // This CTA's reduction steps: whole tiles, or one contiguous stream-K range.
  StepMap map;
  map.total = total;
  map.streamk = args.streamk;
  map.row_tiles = row_tiles;
  map.glu_rt = (kGlu && !args.streamk) ? args.glu_I / kRowsW : 0;
  int n_steps;
  if (map.glu_rt) {
    map.g0 = 0;
    const int pairs = map.glu_rt * (n_tiles / row_tiles);
    const int my_pairs = static_cast<int>(blockIdx.x) < pairs
                             ? (pairs - 1 - static_cast<int>(blockIdx.x)) /
                                       static_cast<int>(gridDim.x) + 1
                             : 0;
    n_steps = 2 * my_pairs * total;
  } else if (args.streamk) {
    const long long T = static_cast<long long>(n_tiles) * total;
    map.g0 = sk_start(blockIdx.x, T, gridDim.x);
    n_steps = static_cast<int>(sk_start(blockIdx.x + 1, T, gridDim.x) - map.g0);
  } else {
    map.g0 = 0;
    const int my_tiles = static_cast<int>(blockIdx.x) < n_tiles
                             ? (n_tiles - 1 - static_cast<int>(blockIdx.x)) /
                                       static_cast<int>(gridDim.x) + 1
                             : 0;
    n_steps = my_tiles * total;
  }
  // Segment of the range starting at step it: tile t, steps [k0, k0 + len) of that tile.
  auto segment = [&](int it, int& t, int& k0, int& len) {
    map.at(it, t, k0);
    len = total - k0 < n_steps - it ? total - k0 : n_steps - it;
  };

  const uint32_t tile_cols = static_cast<uint32_t>(nh) * P.acc_cols;
  uint32_t ncols = static_cast<uint32_t>(P.nacc) * tile_cols;
  if (ncols < 32) ncols = 32;
  // Fused: the rank window's columns follow the accumulator (the allocation is a power of 2).
  const uint32_t rank_col0 = tile_cols;
  if (kFused) ncols = 512;
  const uint32_t rank_bytes = P.rank_slot;
  int* err = args.err;
  // Two token halves: warp 1 issues half 0's MMAs and warp 3 half 1's, each thread waiting only
  // for its own half's X tile and committing its own MMAs (the halves' accumulators are
  // disjoint TMEM columns), so the empty and accumulator barriers take one commit from each.
  // A lone MMA thread's serial chain of barrier operations and issues idles the tensor pipe
  // between steps.  (Fused launches keep one issuer: the window MMAs read either half.)
  const bool dual = !kFused && nh == 2;
  const uint32_t n_issuers = dual ? 2u : 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) mbar_init(xfull + s, 1);
    for (int s = 0; s < SW; ++s) {
      mbar_init(wfull + s, 1);
      mbar_init(wempty + s, n_issuers);  // one commit per MMA-issuing thread
    }
    for (int s = 0; s < SQ; ++s) {
      mbar_init(qfull + s, 1);
      mbar_init(qempty + s, kGroupThreads / 32);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull + b, n_issuers);
      mbar_init(accempty + b, 4);
    }
    mbar_init(drain, n_issuers);
    mbar_init(rank_full, 1);
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
  pdl_wait();  // the previous kernel's outputs (activations, rank-r operand) are complete
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------ X producer -------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_act);
      tma_prefetch_desc(&tm_ext_act);
      if (kFused) tma_prefetch_desc(&tm_rank);
      int issued = 0;  // steps whose X tiles were issued
      bool ok = true;
      for (int it = 0; ok && it < n_steps;) {
        int t, k0, len;
        segment(it, t, k0, len);
        const int tq = t / row_tiles;
        const int tok0 = tq * tile_tokens;
        const RankWindow win = kFused ? rank_window(t, row_tiles, args.M, bt, nh) : RankWindow{};
        // Forward: the tile's adapter picks its r columns of the packed [M, n, r] operand.
        const int eg = kTransW ? 0 : row_group(args.groups, (t - tq * row_tiles) * kRowsW);
        for (int k = k0; k < k0 + len; ++k, ++it) {
          // Step it reuses the X slots of step it - DX: wait until that step's MMAs are done.
          if (it >= DX &&
              !mbar_wait(wempty + w_slot(it - DX), w_par(it - DX), kErrWaitEmpty, err, it)) {
            ok = false;
            break;
          }
          // Fused: the extension operand of this token tile is complete once all of its windows
          // are published (acquire), and the TMA read below is ordered after that.
          if (kFused && k == kt) {
            if (!wait_count(args.rank_flags + tq, 4u * static_cast<unsigned>(win.nwin),
                            kErrWaitRank, err, it)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
          }
          // Fused, on a window's tile: the step's rank-operand tile rides on half 0's barrier.
          const bool rank_step = win.has && k < kt;
          for (int h = 0; h < nh; ++h) {
            const int xs = x_slot(it, h);
            uint8_t* dst = x_ring + xs * P.x_bytes;
            mbar_arrive_expect_tx(xfull + xs, P.x_bytes + (rank_step && h == 0 ? rank_bytes : 0u));
            if (k < kt)
              tma_load_2d(dst, &tm_act, xfull + xs, k * 64, tok0 + h * bt);
            else
              tma_load_3d(dst, &tm_ext_act, xfull + xs, (k - kt) * 64, eg, tok0 + h * bt);
          }
          if (rank_step) {
            uint8_t* rdst = rank_ring + (it & (DX - 1)) * rank_bytes;
            uint64_t* bar = xfull + x_slot(it, 0);
            if (!kTransW)
              tma_load_2d(rdst, &tm_rank, bar, k * 64, 0);  // A [n r rows, 64 k]
            else
              tma_load_2d(rdst, &tm_rank, bar, 0, k * 64);  // B [64 n rows, r]
          }
          issued = it + 1;
        }
      }
      // Every issued copy lands before the CTA may exit.
      for (int j = issued > DX ? issued - DX : 0; j < issued; ++j)
        for (int h = 0; h < nh; ++h) mbar_wait(xfull + x_slot(j, h), x_par(j), kErrWaitDrain, err, j);
    }
  } else if (warp == 2) {
    // ------------------------------ Q producer -------------------------------------------
    // Step it's code tile goes to the Q ring of its owner group g = it % 2, filled and
    // consumed strictly in order (slot g * qper + (v % qper) for the group's v-th code tile),
    // so each slot has exactly one producer and one consumer even though TMA copies land out
    // of order.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      int vq0 = 0, vq1 = 0;  // per-group code-tile counters (registers, not an array)
      bool ok = true;
      for (int it = 0; ok && it < n_steps;) {
        int t, k0, len;
        segment(it, t, k0, len);
        const int row0 = (t % row_tiles) * kRowsW;
        const int kq_end = k0 + len < kt ? k0 + len : kt;
        for (int k = k0; k < kq_end; ++k) {
          const int step = it + (k - k0);
          const int g = step & 1;
          const int v = g ? vq1 : vq0;
          const int slot = (g << P.qlog) + (v & (qper - 1));
          const uint32_t u = static_cast<uint32_t>(v >> P.qlog);
          if (!mbar_wait(qempty + slot, (u & 1u) ^ 1u, kErrWaitEmpty, err, step)) {
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
        it += len;
      }
      // Every issued copy lands before the CTA may exit.
      for (int g = 0; g < kGroups; ++g) {
        const int n = g ? vq1 : vq0;
        for (int v = n > qper ? n - qper : 0; v < n; ++v)
          mbar_wait(qfull + (g << P.qlog) + (v & (qper - 1)),
                    static_cast<uint32_t>(v >> P.qlog) & 1u, kErrWaitDrain, err, v);
      }
    }
  } else if (warp == 1 || (warp == 3 && dual)) {
    // ------------------------------ MMA issuer(s) ----------------------------------------
    // The issuing thread keeps its per-step work to a few adds: ring positions advance
    // incrementally and the smem descriptors are precomputed, the start address (bits 0-13,
    // >> 4) being the only field that moves.  h_lo .. h_hi - 1: the token halves it issues.
    if (lane == 0) {
      const int h_lo = dual ? (warp == 1 ? 0 : 1) : 0;
      const int h_hi = dual ? h_lo + 1 : nh;
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
      // Fused rank window: M = 128 tokens x N = the rank columns (forward: n r rounded up to 16,
      // B K-major; dX: one adapter's r, B MN-major in rows of 2r bytes, 32B or 64B swizzle).
      const uint32_t rank_r = static_cast<uint32_t>(args.rank_r);
      const uint32_t rank_n =
          kTransW ? rank_r : static_cast<uint32_t>((args.rank_cols + 15) / 16 * 16);
      const uint32_t idesc_rank = idesc_bf16_f32(128, rank_n < 16 ? 16u : rank_n, 0u,
                                                 kTransW ? 1u : 0u);
      const uint32_t rank_base = smem_u32(rank_ring);
      const uint32_t rank_pitch = 2u * rank_r;  // dX tile row bytes
      const uint32_t rank_layout = rank_r == 16 ? 6u : 4u;
      int it = 0, seg = 0;
      bool ok = true;
      while (ok && it < n_steps) {
        int t, k0, len;
        segment(it, t, k0, len);
        const RankWindow win = kFused ? rank_window(t, row_tiles, args.M, bt, nh) : RankWindow{};
        const int ab = P.nacc == 2 ? (seg & 1) : 0;
        const int use = P.nacc == 2 ? (seg >> 1) : seg;
        if (!mbar_wait(accempty + ab, (static_cast<uint32_t>(use) & 1u) ^ 1u, kErrWaitAcc, err,
                       seg))
          break;
        tc_fence_after();
        const uint32_t dtm = tmem_base + static_cast<uint32_t>(ab) * tile_cols;
        for (int k = k0; k < k0 + len; ++k, ++it) {
          const int ws = w_slot(it);
          const int xs = (it & (DX - 1)) * nh;
          bool got = mbar_wait(wfull + ws, w_par(it), kErrWaitDequant, err, it);
          for (int h = h_lo; got && h < h_hi; ++h)
            got = mbar_wait(xfull + xs + h, x_par(it), kErrWaitFull, err, it);
          if (!got) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = wdesc0 + static_cast<uint64_t>(ws) * w_slot_step;
          const uint64_t bd0 = xdesc0 + static_cast<uint64_t>(xs) * x_slot_step;
          const uint64_t bd1 = bd0 + x_slot_step;
          const uint32_t acc0 = k > k0 ? 1u : 0u;  // the segment's first step starts the sum
          if (k < kt) {
            if (dual) {  // this thread's half only
              const uint32_t dh = dtm + static_cast<uint32_t>(h_lo) * half_cols;
              const uint64_t bh = h_lo ? bd1 : bd0;
#pragma unroll
              for (int j = 0; j < 4; ++j)
                umma_f16_ss(dh, ad + j * w_kstep, bh + j * x_kstep, idesc, j > 0 ? 1u : acc0);
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t acc = j > 0 ? 1u : acc0;
                umma_f16_ss(dtm, ad + j * w_kstep, bd0 + j * x_kstep, idesc, acc);
                if (nh == 2)
                  umma_f16_ss(dtm + half_cols, ad + j * w_kstep, bd1 + j * x_kstep, idesc, acc);
              }
            }
            if (win.has) {
              // The window's rows of this step's activation tile times its rank-operand tile.
              const uint64_t wa = xdesc0 + static_cast<uint64_t>(xs + win.h) * x_slot_step +
                                  static_cast<uint64_t>(win.w0 * 8);  // w0 rows of 128 B
              const uint32_t rs = rank_base + static_cast<uint32_t>(it & (DX - 1)) * rank_bytes;
              if (!kTransW) {
                const uint64_t rb = smem_desc_sw128(rs, 16u, 1024u);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  umma_f16_ss(tmem_base + rank_col0, wa + j * x_kstep, rb + j * (32u >> 4),
                              idesc_rank, (k > 0 || j > 0) ? 1u : 0u);
              } else {
                // Adapter g of these 64 rows of B adds to its r columns only; its first step
                // starts their sum.
                const int g = row_group(args.rank_groups, k * 64);
                int first_row = 0;
#pragma unroll
                for (int q = 0; q < kMaxGroups - 1; ++q)
                  if (q + 1 < args.rank_groups.n && q + 1 <= g) first_row = args.rank_groups.end[q];
                const uint32_t d = tmem_base + rank_col0 + static_cast<uint32_t>(g) * rank_r;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const uint64_t rb =
                      smem_desc(rs + static_cast<uint32_t>(j) * 16u * rank_pitch, 0u,
                                8u * rank_pitch, rank_layout);
                  umma_f16_ss(d, wa + j * x_kstep, rb, idesc_rank,
                              (k * 64 > first_row || j > 0) ? 1u : 0u);
                }
              }
              if (k == kt - 1) umma_commit(rank_full);
            }
          } else {
            const int rem = args.r_pad16 - (k - kt) * 64;
            const int nk = (rem >= 64 ? 64 : rem) / 16;
            for (int j = 0; j < nk; ++j) {
              const uint32_t acc = j > 0 ? 1u : acc0;
              for (int h = h_lo; h < h_hi; ++h)
                umma_f16_ss(dtm + static_cast<uint32_t>(h) * half_cols, ad + j * w_kstep,
                            (h ? bd1 : bd0) + j * x_kstep, idesc, acc);
            }
          }
          umma_commit(wempty + ws);  // releases the W slot and, DX steps on, the X slots
        }
        if (!ok) break;
        umma_commit(accfull + ab);
        ++seg;
      }
      umma_commit(drain);
      mbar_wait(drain, 0, kErrWaitDrain, err);  // every MMA retired before teardown
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------ epilogue ---------------------------------------------
    // A segment that covers its whole tile goes straight to the bf16 output; a cut one goes
    // as fp32 to this CTA's head (0) or tail (1) partial slot of the workspace.
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int seg = 0, nwin_done = 0;
    for (int it = 0; it < n_steps; ++seg) {
      int t, k0, len;
      segment(it, t, k0, len);
      if (kFused) {
        // Fused: publish this tile's rank window (if any) as soon as its MMAs retire, before the
        // tile's extension step can run.  Lane = window row = token.
        const RankWindow win = rank_window(t, row_tiles, args.M, bt, nh);
        if (win.has) {
          bool got = true;
          if (lane == 0)
            got = mbar_wait(rank_full, static_cast<uint32_t>(nwin_done) & 1u, kErrWaitAcc, err,
                            seg);
          if (!__shfl_sync(0xFFFFFFFFu, got, 0)) break;
          __syncwarp();
          tc_fence_after();
          ++nwin_done;
          const int wrow = quad * 32 + lane;
          const int tq = t / row_tiles;
          const int tok = tq * tile_tokens + win.h * bt + win.w0 + wrow;
          const bool mine = wrow >= win.own0 && tok < args.M;
          const int R = args.rank_cols;
          const uint32_t tb = tmem_base + lane_base + rank_col0;
          for (int c8 = 0; c8 < R / 8; ++c8) {
            uint32_t v[8];
            tmem_ld_32x32b_x8(tb + static_cast<uint32_t>(c8 * 8), v);
            tmem_ld_wait();
            if (mine) {
              const long long o = static_cast<long long>(tok) * R + c8 * 8;
#pragma unroll
              for (int e = 0; e < 8; e += 2) {
                const float v0 = __uint_as_float(v[e]), v1 = __uint_as_float(v[e + 1]);
                if (args.rank_saved)
                  *reinterpret_cast<__nv_bfloat162*>(args.rank_saved + o + e) =
                      __floats2bfloat162_rn(v0, v1);
                *reinterpret_cast<__nv_bfloat162*>(args.rank_scaled + o + e) =
                    __floats2bfloat162_rn(args.rank_scale * v0, args.rank_scale * v1);
              }
            }
          }
          tc_fence_before();
          __threadfence();
          fence_proxy_async_global();
          __syncwarp();
          // Each epilogue warp counts its own 32 rows (no barrier across the warps, which a
          // failed wait in one of them could leave waiting): a window is 4 counts.
          if (lane == 0) atomicAdd(args.rank_flags + tq, 1u);
        }
      }
      const bool whole = k0 == 0 && len == total;
      const int slot = it == 0 ? 0 : 1;
      it += len;
      const int ab = P.nacc == 2 ? (seg & 1) : 0;
      const int use = P.nacc == 2 ? (seg >> 1) : seg;
      bool got = true;
      if (lane == 0)
        got = mbar_wait(accfull + ab, static_cast<uint32_t>(use) & 1u, kErrWaitAcc, err, seg);
      if (!__shfl_sync(0xFFFFFFFFu, got, 0)) break;
      __syncwarp();  // lane 0's acquire, passed on to the warp
      tc_fence_after();
      const int row_l = quad * 32 + lane;
      const int row = (t % row_tiles) * kRowsW + row_l;
      const int tok0 = (t / row_tiles) * tile_tokens;
      const bool row_ok = row < args.rows_w;
      float* part = args.partial +
                    ((static_cast<long long>(blockIdx.x) * 2 + slot) * tile_tokens) * kRowsW;
      // (Two separate loops: a branch inside the drain loop measurably slows the bf16 path.)
      if (kGlu && whole && map.glu_rt && (t % row_tiles) >= map.glu_rt) {
        // Up tile of a SwiGLU pair: u as usual, and a = silu(g) u from the g this thread wrote
        // for the same tokens and the gate row (row - I) one tile earlier: bf16 g and u, fp32
        // math in the packed SwiGLU kernel's order, so a has that kernel's bits.
        const int I = args.glu_I;
        const long long ld = args.rows_w;
        for (int h = 0; h < nh; ++h) {
          const uint32_t tb = tmem_base + lane_base + static_cast<uint32_t>(ab) * tile_cols +
                              static_cast<uint32_t>(h) * P.acc_cols;
          // g of 16 tokens is loaded ahead of their u (16 independent L2 reads in flight).
          for (int c32 = 0; c32 < bt / 8; c32 += 2) {
            const int tk0 = tok0 + h * bt + c32 * 8;
            __nv_bfloat16 gq[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              gq[j] = (c32 * 8 + j < bt && tk0 + j < args.M)
                          ? args.out[static_cast<long long>(tk0 + j) * ld + row - I]
                          : __float2bfloat16_rn(0.f);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              if (c32 + q >= bt / 8) break;
              uint32_t v[8];
              tmem_ld_32x32b_x8(tb + static_cast<uint32_t>((c32 + q) * 8), v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int tok = tk0 + q * 8 + j;
                if (tok < args.M) {
                  const __nv_bfloat16 ub = __float2bfloat16_rn(__uint_as_float(v[j]));
                  args.out[static_cast<long long>(tok) * ld + row] = ub;
                  const float g = __bfloat162float(gq[q * 8 + j]);
                  args.glu_out[static_cast<long long>(tok) * I + row - I] =
                      __float2bfloat16_rn(g * (1.f / (1.f + expf(-g))) * __bfloat162float(ub));
                }
              }
            }
          }
        }
      } else if (whole) {
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
      } else {
        for (int h = 0; h < nh; ++h) {
          const uint32_t tb = tmem_base + lane_base + static_cast<uint32_t>(ab) * tile_cols +
                              static_cast<uint32_t>(h) * P.acc_cols;
          for (int c8 = 0; c8 < bt / 8; ++c8) {
            uint32_t v[8];
            tmem_ld_32x32b_x8(tb + static_cast<uint32_t>(c8 * 8), v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int tl = h * bt + c8 * 8 + j;
              part[static_cast<long long>(tl) * kRowsW + row_l] = __uint_as_float(v[j]);
            }
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
    // Effective absmax of this thread's block at reduction step k of the tile whose first
    // row is row0 (0 outside W0).
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

    // Steps it = g, g + 2, ... of the CTA's range.  The block absmax is fetched kAmAhead owned
    // steps ahead to hide its latency.  After a failed wait the group keeps walking its steps
    // (without waiting or writing) so that every thread still meets the group barrier once
    // per step.
    int vq = 0;  // code tiles this group has consumed
    bool failed = false;
    int last_ext = -1;
    if (tid == 0) tma_prefetch_desc(&tm_ext_w);
    auto absmax_of_step = [&](int it) -> float {
      if (it >= n_steps) return 0.f;
      int t, k;
      map.at(it, t, k);
      return k < kt ? absmax_at((t % row_tiles) * kRowsW, k) : 0.f;
    };
    static_assert(kGroups == 2 && kAmAhead == 3, "the step cursors advance by two steps");
    float am0 = absmax_of_step(g);
    float am1 = absmax_of_step(g + kGroups);
    float am2 = absmax_of_step(g + 2 * kGroups);
    StepCursor cur, ahead;  // step it, and step it + kAmAhead * kGroups
    cur.set(map, g, row_tiles);
    ahead.set(map, g + kAmAhead * kGroups, row_tiles);
    for (int it = g; it < n_steps;
         it += kGroups, cur.advance(map, row_tiles), ahead.advance(map, row_tiles)) {
      const int k = cur.k;
      const float am_next =
          (failed || it + kAmAhead * kGroups >= n_steps || ahead.k >= kt)
              ? 0.f
              : absmax_at(ahead.row0, ahead.k);
      if (k < kt) {
        const int qslot = (g << P.qlog) + (vq & (qper - 1));
        const uint32_t qpar = static_cast<uint32_t>(vq >> P.qlog) & 1u;
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
          nf4_build_lut(args.cb, am0, lut);
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
      } else {
        // Extension step: the lead thread TMA-loads the LoRA weight tile into the W slot.  Every
        // warp of the group first sees the slot's previous use released and the group syncs:
        // a warp that skipped this use could otherwise meet the slot's barrier two phases on.
        if (!failed) failed = !mbar_wait_warp(wempty + w_slot(it), w_par(it) ^ 1u, kErrWaitEmpty,
                                              err, it);
        group_sync(g);
        if (tid == 0 && !failed) {
          {
            const int e = k - kt;
            const int row0 = cur.row0;
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
      }
      am0 = am1;
      am1 = am2;
      am2 = am_next;
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

// Stream-K finalize.  A tile cut between CTAs b_first..b_last gets the sum of their partials
// in that (step) order, rounded once to bf16; an uncut tile was written whole.  Grid (chunks of
// 1024 tile elements, tiles); each thread owns 4 consecutive output features of one token and
// issues its partial loads four contributors at a time before adding them in order.
__global__ void __launch_bounds__(256) qlora_gemm_finalize(const float* __restrict__ partial,
                                                           int M, int rows_w, int tile_tokens,
                                                           int total, long long T, int G,
                                                           __nv_bfloat16* __restrict__ out) {
  pdl_wait();  // the GEMM's partial sums are complete
  pdl_trigger();
  const int row_tiles = (rows_w + kRowsW - 1) / kRowsW;
  const int t = blockIdx.y;
  const long long gs = static_cast<long long>(t) * total;
  // CTA holding global step g: the largest b with floor(b T / G) <= g.
  auto owner = [&](long long g) { return static_cast<int>(((g + 1) * G - 1) / T); };
  const int b_first = owner(gs);
  const int b_last = owner(gs + total - 1);
  if (b_first == b_last) return;
  const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4;  // element of the tile
  if (e >= tile_tokens * kRowsW) return;
  const int tl = e / kRowsW, rl = e - tl * kRowsW;
  const int tok = (t / row_tiles) * tile_tokens + tl;
  const int row = (t % row_tiles) * kRowsW + rl;
  if (tok >= M || row >= rows_w) return;  // rows_w % 64 == 0: the 4 features are all in or out
  const long long slot_elems = static_cast<long long>(tile_tokens) * kRowsW;
  const float* base = partial + e;
  auto slot_ptr = [&](int b) {
    const int slot = sk_start(b, T, G) >= gs ? 0 : 1;  // tile t heads b's range, or ends it
    return base + (static_cast<long long>(b) * 2 + slot) * slot_elems;
  };
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int b = b_first; b <= b_last; b += 4) {
    float4 p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (b + i <= b_last) p[i] = __ldg(reinterpret_cast<const float4*>(slot_ptr(b + i)));
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (b + i <= b_last) {
        v.x += p[i].x;
        v.y += p[i].y;
        v.z += p[i].z;
        v.w += p[i].w;
      }
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + static_cast<long long>(tok) * rows_w + row) = pk;
}

int g_sm_count[64];

}  // namespace

namespace {

// Relative duration (cycles of the busiest CTA) of a whole-tile schedule with token tiles of
// nh x bt, from the kernel's per-step profile at 512-token tiles: besides ~2.12 tensor cycles
// per token, the MMA thread spends ~745 cycles per 64-deep step on barriers, descriptors and
// the commit; and when one accumulator fills TMEM (more than 256 token columns) the epilogue's
// drain, ~37 cycles per token column, is exposed at every tile switch instead of overlapping
// the next tile's mainloop.
// Measured on a B200 (4096-token q_proj backward): one CTA of the side kernel, alone on its SM
// with a 12-stage TMA ring, streams ~26 GB/s while the GEMM holds the other SMs (the SM's
// outstanding-miss limit, not HBM); the cluster kernels on the whole GPU ~2.2 TB/s.
constexpr double kSideBytesPerUsPerSm = 26e3;
constexpr double kSerialBytesPerUs = 2.2e6;
constexpr double kClockMhz = 1965.0;  // cycles of the model per microsecond
constexpr int kSideMaxSms = 32;

double whole_tile_cycles(int M, int rows_w, int steps, int G, int bt, int nh) {
  const int tt = bt * nh;
  const long long tiles =
      static_cast<long long>((rows_w + kRowsW - 1) / kRowsW) * ((M + tt - 1) / tt);
  const long long rounds = (tiles + G - 1) / G;
  const double step = 745.0 + 2.12 * tt;
  const double drain = 37.0 * tt;
  const bool exposed = make_plan(bt, nh).nacc == 1;
  return static_cast<double>(rounds) * (steps * step + (exposed ? drain : 0.0)) +
         (exposed ? 0.0 : drain);
}

}  // namespace

GemmTile gemm_pick_tile(int M, int rows_w, int steps_per_tile, int sm_count, bool fused) {
  GemmTile t;
  if (fused && M > 256) {
    // The fused down-projection's windows need two halves of 128 < bt <= 240 tokens: take the
    // cheapest such tile by the same model.
    const int G = sm_count < kGemmMaxCtas ? sm_count : kGemmMaxCtas;
    double best = 0.0;
    t.nh = 2;
    t.bt = 240;
    for (int bt = 240; bt >= 144; bt -= 16) {
      const double c = whole_tile_cycles(M, rows_w, steps_per_tile, G, bt, 2);
      if (bt == 240 || c < best) {
        best = c;
        t.bt = bt;
      }
    }
    return t;
  }
  if (M <= 256) {  // one half: as many tokens as there are, in steps of 16
    t.bt = M < 16 ? 16 : (M + 15) / 16 * 16;
    t.nh = 1;
    return t;
  }
  t.bt = 256;
  t.nh = 2;
  const int G = sm_count < kGemmMaxCtas ? sm_count : kGemmMaxCtas;
  const long long tiles =
      static_cast<long long>((rows_w + kRowsW - 1) / kRowsW) * ((M + 511) / 512);
  if (tiles < G) return t;  // stream-K over the widest tiles
  // Whole tiles: the last round of tiles is usually part-full, so narrower token tiles can
  // shorten the busiest CTA's work at the same number of rounds.  Keep 512 tokens unless the
  // model gives at least 2 %.
  const double wide = whole_tile_cycles(M, rows_w, steps_per_tile, G, 256, 2);
  double best = wide;
  int best_bt = 256;
  for (int bt = 240; bt >= 128; bt -= 16) {
    const double c = whole_tile_cycles(M, rows_w, steps_per_tile, G, bt, 2);
    if (c < best) {
      best = c;
      best_bt = bt;
    }
  }
  if (best <= 0.98 * wide) t.bt = best_bt;
  return t;
}

cudaError_t gemm_device_sms(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_sm_count[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  *sms = g_sm_count[dev];
  return cudaSuccess;
}

size_t gemm_smem_bytes(int bt, int nh) { return make_plan(bt, nh).smem; }

bool gemm_glu_ok(int M, int I, int steps_per_tile, int sm_count) {
  if (I < kRowsW || I % kRowsW) return false;
  return !gemm_schedule(M, 2 * I, steps_per_tile, sm_count, false).streamk;
}

GemmSchedule gemm_schedule(int M, int rows_w, int steps_per_tile, int sm_count, bool fused) {
  GemmSchedule sc;
  const GemmTile tl = gemm_pick_tile(M, rows_w, steps_per_tile, sm_count, fused);
  const int tile_tokens = tl.bt * tl.nh;
  sc.n_tiles = ((rows_w + kRowsW - 1) / kRowsW) * ((M + tile_tokens - 1) / tile_tokens);
  const int G = sm_count < kGemmMaxCtas ? sm_count : kGemmMaxCtas;
  if (sc.n_tiles >= G) {
    sc.streamk = 0;
    sc.grid = G;
  } else {
    // Fewer tiles than SMs: cut the reduction so every SM streams its share of the weight
    // (every CTA gets at least one step).
    const long long T = static_cast<long long>(sc.n_tiles) * steps_per_tile;
    sc.streamk = 1;
    sc.grid = T < G ? static_cast<int>(T) : G;
  }
  sc.partial_floats = sc.streamk ? static_cast<size_t>(sc.grid) * 2 * tile_tokens * kRowsW : 0;
  return sc;
}

bool gemm_rank_fusable(int M, int rows_w, int steps_per_tile, int sm_count, int rank_cols,
                       unsigned rank_slot) {
  if (rank_cols < 8 || rank_cols > kRankMaxCols || rank_cols % 8 != 0 || rank_slot == 0)
    return false;
  if (M <= 256) return false;
  const GemmTile tl = gemm_pick_tile(M, rows_w, steps_per_tile, sm_count, true);
  const GemmSchedule sc = gemm_schedule(M, rows_w, steps_per_tile, sm_count, true);
  if (sc.streamk) return false;
  // Worth it while the fused tile costs the GEMM at most 4 % over its own choice of tile (the
  // separate down-projection it replaces streams all of the activations once more).
  const GemmTile own = gemm_pick_tile(M, rows_w, steps_per_tile, sm_count, false);
  const GemmSchedule own_sc = gemm_schedule(M, rows_w, steps_per_tile, sm_count, false);
  if (own_sc.streamk) return false;
  const int G = sc.grid;
  if (whole_tile_cycles(M, rows_w, steps_per_tile, G, tl.bt, tl.nh) >
      1.04 * whole_tile_cycles(M, rows_w, steps_per_tile, G, own.bt, own.nh))
    return false;
  // The window's columns after the 2 bt accumulator columns, within TMEM's 512.
  if (2 * tl.bt + (rank_cols + 15) / 16 * 16 > 512) return false;
  const Plan p = make_plan(tl.bt, tl.nh, rank_slot);
  if (p.rank_slots < p.dx || p.nacc != 1) return false;
  const int tile_tokens = tl.bt * tl.nh;
  const int row_tiles = (rows_w + kRowsW - 1) / kRowsW;
  const int token_tiles = (M + tile_tokens - 1) / tile_tokens;
  for (int tq = 0; tq < token_tiles; ++tq) {
    const RankWindow w = rank_window(tq * row_tiles, row_tiles, M, tl.bt, tl.nh);
    if (w.nwin > first_wave_tiles(tq, row_tiles, G)) return false;
  }
  return true;
}

int gemm_side_sms(int M, int rows_w, int steps_per_tile, int sm_count, double side_bytes,
                  bool force, double* us) {
  const int G = sm_count < kGemmMaxCtas ? sm_count : kGemmMaxCtas;
  *us = 0.0;
  if (M <= 256 || G < 64 || side_bytes <= 0.0 ||
      gemm_schedule(M, rows_w, steps_per_tile, G).streamk)
    return 0;
  const GemmTile t0 = gemm_pick_tile(M, rows_w, steps_per_tile, G);
  const double alone = whole_tile_cycles(M, rows_w, steps_per_tile, G, t0.bt, t0.nh) / kClockMhz;
  int best = 0;
  double best_us = 0.0;
  for (int spare = 2; spare <= kSideMaxSms; spare += 2) {
    const int g = G - spare;
    if (gemm_schedule(M, rows_w, steps_per_tile, g).streamk) break;
    const GemmTile t = gemm_pick_tile(M, rows_w, steps_per_tile, g);
    const double gemm = whole_tile_cycles(M, rows_w, steps_per_tile, g, t.bt, t.nh) / kClockMhz;
    const double side = side_bytes / (spare * kSideBytesPerUsPerSm);
    const double both = gemm > side ? gemm : side;
    if (best == 0 || both < best_us) {
      best = spare;
      best_us = both;
    }
  }
  // After the launch instead: the cluster kernels stream at ~2.2 TB/s on the whole GPU, plus
  // ~5 us for their launch and tail.
  const double serial = alone + side_bytes / kSerialBytesPerUs + 5.0;
  if (best == 0 || (!force && best_us > 0.97 * serial)) return 0;
  *us = best_us;
  return best;
}

size_t gemm_rank_flag_bytes(int M) { return 4 * (static_cast<size_t>(M) / 128 + 2); }

size_t gemm_partial_bytes_bound(int M, int rows_w, int steps_per_tile) {
  return 4 * gemm_schedule(M, rows_w, steps_per_tile, kGemmMaxCtas).partial_floats;
}

cudaError_t launch_qlora_gemm(bool trans_w, const GemmMaps& maps, GemmArgs args,
                              size_t partial_floats_avail, cudaStream_t stream, int* launched) {
  *launched = 0;
  int sms = 0;
  cudaError_t e = gemm_device_sms(&sms);
  if (e != cudaSuccess) return e;
  if (args.sm_limit > 0 && args.sm_limit < sms) {
    if (args.fuse) return cudaErrorInvalidValue;  // its windows assume every SM's first wave
    sms = args.sm_limit;
  }
  // The caller's tile (TMA boxes, smem plan) must be the one the schedule assumes.
  const GemmTile tl = gemm_pick_tile(args.M, args.rows_w, args.kt + args.n_ext, sms, args.fuse);
  if (tl.bt != args.bt || tl.nh != args.nh) return cudaErrorInvalidValue;
  GemmSchedule sc = gemm_schedule(args.M, args.rows_w, args.kt + args.n_ext, sms, args.fuse);
  if (sc.streamk && (!args.partial || sc.partial_floats > partial_floats_avail)) {
    // No room for the partial sums: whole tiles, one CTA per tile.
    sc.streamk = 0;
    sc.grid = sc.n_tiles;
  }
  args.streamk = sc.streamk;
  if (args.glu_I > 0 && (trans_w || args.fuse || sc.streamk || !args.glu_out ||
                         args.glu_I % kRowsW || args.rows_w != 2 * args.glu_I))
    return cudaErrorInvalidValue;
  if (args.fuse && (sc.streamk || !gemm_rank_fusable(args.M, args.rows_w, args.kt + args.n_ext,
                                                      sms, args.rank_cols, args.rank_slot)))
    return cudaErrorInvalidValue;
  const size_t smem = make_plan(args.bt, args.nh, args.fuse ? args.rank_slot : 0u).smem;
  // The fused down-projection is a separate instantiation, so the plain kernel carries none of
  // its code.
  // The SwiGLU epilogue is a third instance (forward, unfused), so the others carry none of it.
  auto kernel = trans_w ? (args.fuse ? qlora_gemm_kernel<true, true> : qlora_gemm_kernel<true, false>)
                        : (args.fuse ? qlora_gemm_kernel<false, true>
                                     : (args.glu_I > 0 ? qlora_gemm_kernel<false, false, true>
                                                       : qlora_gemm_kernel<false, false>));
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(kernel, dim3(sc.grid), dim3(kThreads), smem, stream, 1, maps.act, maps.q,
                 maps.ext_w, maps.ext_act, maps.rank, args);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  *launched = 1;
  if (!sc.streamk) return e;
  const int total = args.kt + args.n_ext;
  const long long T = static_cast<long long>(sc.n_tiles) * total;
  const int tile_elems = args.bt * args.nh * kRowsW;
  const dim3 fgrid((tile_elems / 4 + 255) / 256, sc.n_tiles);
  e = launch_pdl(qlora_gemm_finalize, fgrid, dim3(256), 0, stream, 1,
                 static_cast<const float*>(args.partial), args.M, args.rows_w,
                 args.bt * args.nh, total, T, sc.grid, args.out);
  if (e == cudaSuccess) *launched = 2;
  return e;
}

}  // namespace qlora

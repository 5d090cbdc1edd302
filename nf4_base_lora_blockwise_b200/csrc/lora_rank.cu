// lora_rank.cu -- the rank-r products around the dequant GEMM, streamed from HBM once at full
// bandwidth: TMA loads of 128 x 64 activation tiles into a swizzled shared-memory ring, warp-level
// mma.sync (bf16 in, fp32 accumulate) on the 16-column-wide tensor work, and the reduction split
// over the CTAs of a thread-block cluster and summed in a fixed order through distributed shared
// memory, so one launch writes the finished result and needs no scratch in HBM.
//
//   down:  out[M, R]  = in[M, C] . Wl^T         XA = X A^T (forward, kept for the backward),
//                                               dYB = dY B (backward)
//   grad:  G[C, R]    = s in[M, C]^T . small[M, R]   dB = s dY^T XA,  dA = s (dYB^T X)
// ("Unsloth vs QLoRA vs Liger-Kernel", section 1 forward formula and its "save the small
// product" remark; section 2, hand-derived backward.)
//
// With n adapters packed along the rows of B (q/k/v or gate/up sharing X), dY B takes the
// block-diagonal B: adapter g's rows of dY feed columns g r .. g r + r - 1 only, so each 64-row
// step multiplies by that adapter's r columns and the zero blocks are neither loaded nor
// multiplied; dB takes, for adapter g's columns of dY, the columns g r .. of XA.
//
// A tile is 128 rows of the output (tokens for down, columns of `in` for grad).  The reduction
// (C for down, M for grad) runs in 64-deep steps, split into S equal ranges over the S CTAs of
// one cluster (S = 1, 2, 4 or 8).  Warp roles (288 threads):
//   warps 0-7   consumers: warp w owns rows 16w .. 16w + 15 of the tile (mma.sync m16n8k16)
//   warp 8      lane 0 issues the TMA loads of the ring
// After the reduction each CTA leaves its fp32 partial [128 x R] in its own shared memory; CTA q
// of the cluster then sums rows q*128/S .. of all S partials in rank order (deterministic) and
// writes them.
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace qlora {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kRankThreads = 32 * (kConsumerWarps + 1);
constexpr int kTileRows = 128;
constexpr uint32_t kBigTileBytes = kTileRows * 64 * 2;  // 128 rows x 64 bf16
constexpr int kMaxSplit = 8;

__device__ __forceinline__ uint32_t sw128_off(uint32_t row, uint32_t chunk) {
  return swz_off(row, chunk, 128u, 7u);
}

// ---------------------------------- cluster helpers ---------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster arrives, then waits for all of them (release /
// acquire: shared-memory writes before the barrier are visible to the cluster after it).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(remote));
  return v;
}
__device__ __forceinline__ float ld_dsmem_f1(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote));
  return v;
}

// Shared-memory plan of one launch (the same on host and device).
struct RankLayout {
  uint32_t small_bytes;  // per stage: the Wl / small tile
  uint32_t stage_bytes;  // big tile + small tile
  uint32_t ring_bytes;   // max(stages x stage_bytes, the fp32 partial)
  int stages;
  size_t smem;
};

__host__ __device__ inline uint32_t partial_pitch(int R) { return static_cast<uint32_t>(R + 4); }

__host__ __device__ inline RankLayout rank_layout(uint32_t small_bytes, int R, int budget,
                                                  int max_stages = 8) {
  RankLayout L;
  L.small_bytes = (small_bytes + 1023u) & ~1023u;
  L.stage_bytes = kBigTileBytes + L.small_bytes;
  int st = static_cast<int>((static_cast<uint32_t>(budget) - 2048u) / L.stage_bytes);
  L.stages = st < 2 ? 2 : (st > max_stages ? max_stages : st);
  const uint32_t ring = static_cast<uint32_t>(L.stages) * L.stage_bytes;
  const uint32_t part = static_cast<uint32_t>(kTileRows) * partial_pitch(R) * 4u;
  L.ring_bytes = ring > part ? ring : part;
  L.smem = 1024 + L.ring_bytes + 2 * 8 * L.stages;
  return L;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// Kernel arguments (shared by both kernels).
// ------------------------------------------------------------------------------------------
struct RankArgs {
  int M, C;          // `in` / `big` is [M, C]
  int R;             // accumulator columns (NT * 8)
  int rg;            // down, B form: columns per adapter (R = n rg); grad: R
  int steps;         // 64-deep reduction steps in total
  int split;         // CTAs per cluster
  int stages;
  uint32_t stage_bytes, small_bytes, ring_bytes;
  uint32_t small_pitch;  // bytes per row of a small-tile block
  uint32_t small_mask;   // its swizzle mask (0: unswizzled)
  int small_blocks;      // 2: two 64-column SW128 blocks (128 columns), else 1
  int ld_small;          // grad: columns of small ([M, ld_small])
  float scale;
  RowGroups groups;
  __nv_bfloat16* saved;   // down: bf16(out) (nullable)
  __nv_bfloat16* scaled;  // down: bf16(scale * out)
  float* out;             // grad: scale * G, [C, R] (out_cr) or [R, C]
  int out_cr;
  int* err;
  int gsplit;             // down: clusters per row tile along the reduction
  float* gpart;           // down, gsplit > 1: fp32 partials [tiles][gsplit][128][R]
};

namespace {

// Offset of 16-byte chunk `ch` of row `row` of the small tile (rows of the reduction).
__device__ __forceinline__ uint32_t small_off(const RankArgs& a, int row, uint32_t ch) {
  if (a.small_blocks == 2) return (ch >> 3) * 8192u + sw128_off(row, ch & 7u);
  return swz_off(static_cast<uint32_t>(row), ch, a.small_pitch, a.small_mask);
}

// Producer: lane 0 of warp 8 fills the ring in order; stage i waits for the consumers to
// release its previous use.  `load(i, dst, bar)` issues step i's copies.  Before the CTA moves
// on, the copies it issued have all landed (they have, when the consumers saw every stage).
template <typename Load>
__device__ __forceinline__ void rank_produce(const RankArgs& a, uint8_t* ring, uint64_t* full,
                                             uint64_t* empty, int n, Load load) {
  int issued = 0;
  for (int i = 0; i < n; ++i) {
    const int st = i % a.stages;
    const int use = i / a.stages;
    if (use > 0 && !mbar_wait(empty + st, static_cast<uint32_t>(use - 1) & 1u, kErrWaitEmpty,
                              a.err, i))
      break;
    uint8_t* dst = ring + st * a.stage_bytes;
    mbar_arrive_expect_tx(full + st, a.stage_bytes);
    load(i, dst, full + st);
    issued = i + 1;
  }
  for (int i = issued > a.stages ? issued - a.stages : 0; i < issued; ++i)
    mbar_wait(full + i % a.stages, static_cast<uint32_t>(i / a.stages) & 1u, kErrWaitDrain, a.err,
              i);
}

// ------------------------------------------------------------------------------------------
// down: grid (tiles x S), cluster S.  Tile rows = tokens.  kWrc: Wl is A [R, C] (K-major rows
// j, SW128); otherwise Wl is B [C, rg] (rows c, rg contiguous; block-diagonal over adapters).
// ------------------------------------------------------------------------------------------
template <int NT, bool kWrc>
__global__ void __launch_bounds__(kRankThreads, NT <= 8 ? 2 : 1)
    rank_down_kernel(const __grid_constant__ CUtensorMap tm_in,
                     const __grid_constant__ CUtensorMap tm_w, const RankArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + a.ring_bytes);
  uint64_t* empty = full + a.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  // Cluster gc of tile `tile` takes part gc of the reduction; CTA `rank` of it, its own share.
  const int per_tile = a.split * a.gsplit;
  const int tile = static_cast<int>(blockIdx.x) / per_tile;
  const int gc = (static_cast<int>(blockIdx.x) / a.split) % a.gsplit;
  const int row0 = tile * kTileRows;
  const int part_idx = gc * a.split + static_cast<int>(rank);
  const int s0 = static_cast<int>(static_cast<long long>(a.steps) * part_idx / per_tile);
  const int n = static_cast<int>(static_cast<long long>(a.steps) * (part_idx + 1) / per_tile) - s0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_in);
      tma_prefetch_desc(&tm_w);
      rank_produce(a, ring, full, empty, n, [&](int i, uint8_t* dst, uint64_t* bar) {
        const int c0 = (s0 + i) * 64;
        tma_load_2d(dst, &tm_in, bar, c0, row0);
        uint8_t* w = dst + kBigTileBytes;
        if (kWrc) {
          tma_load_2d(w, &tm_w, bar, c0, 0);  // A [R rows, 64 c]
        } else {
          tma_load_2d(w, &tm_w, bar, 0, c0);  // B [64 c, rg] (one or two column blocks)
          if (a.small_blocks == 2) tma_load_2d(w + 8192, &tm_w, bar, 64, c0);
        }
      });
    }
  } else {
    bool failed = false;
    const int ar = 16 * warp + (lane & 15);  // A-fragment row this lane addresses
    for (int i = 0; i < n; ++i) {
      const int st = i % a.stages;
      if (!failed)
        failed = !mbar_wait_warp(full + st, static_cast<uint32_t>(i / a.stages) & 1u,
                                 kErrWaitFull, a.err, i);
      if (!failed) {
        const uint32_t xb = smem_u32(ring + st * a.stage_bytes);
        const uint32_t wb = xb + kBigTileBytes;
        // Adapter of this step's rows of B (its n-tiles are the only ones fed).
        const int g = kWrc ? 0 : row_group(a.groups, (s0 + i) * 64);
        const int t_lo = kWrc ? 0 : g * (a.rg / 8);
        const int t_hi = kWrc ? NT : t_lo + a.rg / 8;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t af[4];
          ldsm_x4(af, xb + sw128_off(ar, 2 * kk + (lane >> 4)));
          if (kWrc) {
#pragma unroll
            for (int t = 0; t + 1 < NT; t += 2) {
              const int j = t * 8 + (lane & 7) + ((lane >> 4) << 3);
              uint32_t b[4];
              ldsm_x4(b, wb + sw128_off(j, 2 * kk + ((lane >> 3) & 1)));
              mma16816(acc[t], af, b[0], b[1]);
              mma16816(acc[t + 1], af, b[2], b[3]);
            }
            if (NT & 1) {
              constexpr int t = NT - 1;
              const int l = lane & 15;
              uint32_t b[2];
              ldsm_x2(b, wb + sw128_off(t * 8 + (l & 7), 2 * kk + (l >> 3)));
              mma16816(acc[t], af, b[0], b[1]);
            }
          } else {
            const int l = lane & 15;
            const int k = 16 * kk + (l & 7) + ((l >> 3) << 3);  // row c of the B tile
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              if (t >= t_lo && t < t_hi) {
                const uint32_t ch = static_cast<uint32_t>(t - t_lo);  // 16-byte column chunk
                uint32_t b[2];
                ldsm_x2_t(b, wb + small_off(a, k, ch));
                mma16816(acc[t], af, b[0], b[1]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + st);
    }
  }

  // ---- fixed-order reduction over the cluster through distributed shared memory ----------
  cluster_sync_all();  // every warp of every CTA is done with its ring
  float* part = reinterpret_cast<float*>(ring);
  const uint32_t pp = partial_pitch(a.R);
  if (warp < kConsumerWarps) {
    const int r_lo = 16 * warp + (lane >> 2);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int col = t * 8 + (lane & 3) * 2;
      *reinterpret_cast<float2*>(part + r_lo * pp + col) = make_float2(acc[t][0], acc[t][1]);
      *reinterpret_cast<float2*>(part + (r_lo + 8) * pp + col) =
          make_float2(acc[t][2], acc[t][3]);
    }
  }
  cluster_sync_all();  // every CTA's partial is complete and visible to the cluster
  const int rows = kTileRows / a.split;
  const int r_first = static_cast<int>(rank) * rows;
  const int items = rows * (a.R / 4);
  for (int it = threadIdx.x; it < items; it += kRankThreads) {
    const int rl = r_first + it / (a.R / 4);
    const int c4 = (it % (a.R / 4)) * 4;
    const int m = row0 + rl;
    const uint32_t la = smem_u32(part + rl * pp + c4);
    float4 p[kMaxSplit];
#pragma unroll
    for (int q = 0; q < kMaxSplit; ++q)
      if (q < a.split) p[q] = ld_dsmem_f4(la, static_cast<uint32_t>(q));
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < kMaxSplit; ++q)
      if (q < a.split) {
        v.x += p[q].x;
        v.y += p[q].y;
        v.z += p[q].z;
        v.w += p[q].w;
      }
    if (a.gsplit > 1) {
      // This cluster's share of the reduction, for the finalize to add in cluster order.
      float* dst = a.gpart + ((static_cast<long long>(tile) * a.gsplit + gc) * kTileRows + rl) * a.R + c4;
      *reinterpret_cast<float4*>(dst) = v;
    } else if (m < a.M) {
      const long long o = static_cast<long long>(m) * a.R + c4;
      if (a.saved) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(a.saved + o) = pk;
      }
      __nv_bfloat162 lo = __floats2bfloat162_rn(a.scale * v.x, a.scale * v.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(a.scale * v.z, a.scale * v.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(a.scaled + o) = pk;
    }
  }
  cluster_sync_all();  // no CTA leaves while another still reads its partial
}

// The second-level split's sum: out[m, c4 .. c4+3] adds the gsplit cluster partials of m's
// tile in cluster order, then rounds to bf16 (saved) and scales (scaled).
__global__ void __launch_bounds__(256) rank_down_finalize(const RankArgs a) {
  pdl_wait();  // the partials are complete
  pdl_trigger();
  const int items = a.M * (a.R / 4);
  const int it = static_cast<int>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (it >= items) return;
  const int m = it / (a.R / 4);
  const int c4 = (it - m * (a.R / 4)) * 4;
  const int tile = m / kTileRows, rl = m - tile * kTileRows;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int g = 0; g < a.gsplit; ++g) {
    const float4 p = __ldg(reinterpret_cast<const float4*>(
        a.gpart + ((static_cast<long long>(tile) * a.gsplit + g) * kTileRows + rl) * a.R + c4));
    v.x += p.x;
    v.y += p.y;
    v.z += p.z;
    v.w += p.w;
  }
  const long long o = static_cast<long long>(m) * a.R + c4;
  if (a.saved) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(a.saved + o) = pk;
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(a.scale * v.x, a.scale * v.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(a.scale * v.z, a.scale * v.w);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(a.scaled + o) = pk;
}

// ------------------------------------------------------------------------------------------
// grad: grid (tiles x S), cluster S.  Tile rows = 128 columns c of `big`; the reduction runs
// over tokens in steps of 64.  A = big^T (transposed 8x8 loads of the [64 tokens x 128 c]
// tile, two SW128 blocks of 64 columns), B = small [64 tokens x R] (rows tokens).
// ------------------------------------------------------------------------------------------
// Two independent problems (dB and dA of one backward) may share a launch: CTAs below `grid1`
// take the first (maps *1, a1), the rest the second, so neither waits for the other's tail.
template <int NT>
__global__ void __launch_bounds__(kRankThreads, NT <= 8 ? 2 : 1)
    rank_grad_kernel(const __grid_constant__ CUtensorMap tm_big1,
                     const __grid_constant__ CUtensorMap tm_small1, const __grid_constant__ RankArgs a1,
                     const __grid_constant__ CUtensorMap tm_big2,
                     const __grid_constant__ CUtensorMap tm_small2, const __grid_constant__ RankArgs a2,
                     int grid1) {
  const bool second = static_cast<int>(blockIdx.x) >= grid1;
  const RankArgs& a = second ? a2 : a1;
  const CUtensorMap& tm_big = second ? tm_big2 : tm_big1;
  const CUtensorMap& tm_small = second ? tm_small2 : tm_small1;
  const int bid = second ? static_cast<int>(blockIdx.x) - grid1 : static_cast<int>(blockIdx.x);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + a.ring_bytes);
  uint64_t* empty = full + a.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int tile = bid / a.split;
  const int c0 = tile * kTileRows;
  // This tile's columns belong to one adapter, whose R columns of `small` it reads.
  const int j0 = row_group(a.groups, c0) * a.R;
  const int s0 = static_cast<int>(static_cast<long long>(a.steps) * rank / a.split);
  const int n = static_cast<int>(static_cast<long long>(a.steps) * (rank + 1) / a.split) - s0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_big);
      tma_prefetch_desc(&tm_small);
      rank_produce(a, ring, full, empty, n, [&](int i, uint8_t* dst, uint64_t* bar) {
        const int m0 = (s0 + i) * 64;
        tma_load_2d(dst, &tm_big, bar, c0, m0);             // [64 tokens, c0 .. c0 + 63]
        tma_load_2d(dst + 8192, &tm_big, bar, c0 + 64, m0);  // [64 tokens, c0 + 64 ..]
        uint8_t* sm = dst + kBigTileBytes;
        tma_load_2d(sm, &tm_small, bar, j0, m0);
        if (a.small_blocks == 2) tma_load_2d(sm + 8192, &tm_small, bar, j0 + 64, m0);
      });
    }
  } else {
    bool failed = false;
    const int q = lane >> 3, i8 = lane & 7;
    const int cl = 16 * warp + (q & 1) * 8;  // column block of big this lane addresses
    const uint32_t cblk = static_cast<uint32_t>(cl >> 6) * 8192u;
    const uint32_t cch = static_cast<uint32_t>(cl & 63) >> 3;
    for (int i = 0; i < n; ++i) {
      const int st = i % a.stages;
      if (!failed)
        failed = !mbar_wait_warp(full + st, static_cast<uint32_t>(i / a.stages) & 1u,
                                 kErrWaitFull, a.err, i);
      if (!failed) {
        const uint32_t bb = smem_u32(ring + st * a.stage_bytes);
        const uint32_t sb = bb + kBigTileBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t af[4];
          const int tok = 16 * kk + i8 + (q >> 1) * 8;
          ldsm_x4_t(af, bb + cblk + sw128_off(tok, cch));
          const int l = lane & 15;
          const int k = 16 * kk + (l & 7) + ((l >> 3) << 3);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            uint32_t b[2];
            ldsm_x2_t(b, sb + small_off(a, k, static_cast<uint32_t>(t)));
            mma16816(acc[t], af, b[0], b[1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + st);
    }
  }

  cluster_sync_all();
  float* part = reinterpret_cast<float*>(ring);
  const uint32_t pp = partial_pitch(a.R);
  if (warp < kConsumerWarps) {
    const int r_lo = 16 * warp + (lane >> 2);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int col = t * 8 + (lane & 3) * 2;
      *reinterpret_cast<float2*>(part + r_lo * pp + col) = make_float2(acc[t][0], acc[t][1]);
      *reinterpret_cast<float2*>(part + (r_lo + 8) * pp + col) =
          make_float2(acc[t][2], acc[t][3]);
    }
  }
  cluster_sync_all();
  const int rows = kTileRows / a.split;
  const int r_first = static_cast<int>(rank) * rows;
  if (a.out_cr) {  // out [C, R]: 4 consecutive j of one column c
    const int items = rows * (a.R / 4);
    for (int it = threadIdx.x; it < items; it += kRankThreads) {
      const int rl = r_first + it / (a.R / 4);
      const int j4 = (it % (a.R / 4)) * 4;
      const uint32_t la = smem_u32(part + rl * pp + j4);
      float4 p[kMaxSplit];
#pragma unroll
      for (int qq = 0; qq < kMaxSplit; ++qq)
        if (qq < a.split) p[qq] = ld_dsmem_f4(la, static_cast<uint32_t>(qq));
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int qq = 0; qq < kMaxSplit; ++qq)
        if (qq < a.split) {
          v.x += p[qq].x;
          v.y += p[qq].y;
          v.z += p[qq].z;
          v.w += p[qq].w;
        }
      const int c = c0 + rl;
      if (c < a.C)
        *reinterpret_cast<float4*>(a.out + static_cast<long long>(c) * a.R + j4) =
            make_float4(a.scale * v.x, a.scale * v.y, a.scale * v.z, a.scale * v.w);
    }
  } else {  // out [R, C]: 4 consecutive columns c of one j (coalesced rows of dA)
    const int items = (rows / 4) * a.R;
    for (int it = threadIdx.x; it < items; it += kRankThreads) {
      const int j = it / (rows / 4);
      const int rl = r_first + (it % (rows / 4)) * 4;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      for (int qq = 0; qq < a.split; ++qq) {
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          p[e] = ld_dsmem_f1(smem_u32(part + (rl + e) * pp + j), static_cast<uint32_t>(qq));
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] += p[e];
      }
      const int c = c0 + rl;  // C % 64 == 0, so the 4 columns are all in or all out
      if (c < a.C)
        *reinterpret_cast<float4*>(a.out + static_cast<long long>(j) * a.C + c) =
            make_float4(a.scale * v[0], a.scale * v[1], a.scale * v[2], a.scale * v[3]);
    }
  }
  cluster_sync_all();
}

// ------------------------------------------------------------------------------------------
// grad beside another kernel (rank_grad_loop_kernel): a few CTAs, one per SM, each walking
// whole tiles -- CTA b of a problem takes tiles b, b + nb, ... -- so the launch occupies only
// the SMs it is given while a GEMM holds the rest.  A tile's reduction over M runs in the same
// S contiguous step ranges as the cluster kernel's S CTAs: each range is summed on its own and
// the range sums are added in range order, exactly the cluster kernel's arithmetic, so both
// kernels give the same bits.  The ring runs on across tiles (the copies of the next tile
// overlap the end of this one) and each tile is written straight from the accumulators.
// ------------------------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kRankThreads, 1)
    rank_grad_loop_kernel(const __grid_constant__ CUtensorMap tm_big1,
                          const __grid_constant__ CUtensorMap tm_small1,
                          const __grid_constant__ RankArgs a1,
                          const __grid_constant__ CUtensorMap tm_big2,
                          const __grid_constant__ CUtensorMap tm_small2,
                          const __grid_constant__ RankArgs a2, int grid1) {
  const bool second = static_cast<int>(blockIdx.x) >= grid1;
  const RankArgs& a = second ? a2 : a1;
  const CUtensorMap& tm_big = second ? tm_big2 : tm_big1;
  const CUtensorMap& tm_small = second ? tm_small2 : tm_small1;
  const int bid = second ? static_cast<int>(blockIdx.x) - grid1 : static_cast<int>(blockIdx.x);
  const int nb = second ? static_cast<int>(gridDim.x) - grid1 : grid1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + a.ring_bytes);
  uint64_t* empty = full + a.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (a.C + kTileRows - 1) / kTileRows;
  const int my_tiles = bid < tiles ? (tiles - bid + nb - 1) / nb : 0;
  const int n = my_tiles * a.steps;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_big);
      tma_prefetch_desc(&tm_small);
      // The big operand is read once here: evict-first, so the stream does not push out of L2
      // the activation tiles the GEMM beside this kernel keeps re-reading.
      const uint64_t once = l2_policy_evict_first();
      rank_produce(a, ring, full, empty, n, [&](int i, uint8_t* dst, uint64_t* bar) {
        const int ti = i / a.steps;
        const int c0 = (bid + ti * nb) * kTileRows;
        const int m0 = (i - ti * a.steps) * 64;
        const int j0 = row_group(a.groups, c0) * a.R;
        tma_load_2d_hint(dst, &tm_big, bar, c0, m0, once);
        tma_load_2d_hint(dst + 8192, &tm_big, bar, c0 + 64, m0, once);
        uint8_t* sm = dst + kBigTileBytes;
        tma_load_2d(sm, &tm_small, bar, j0, m0);
        if (a.small_blocks == 2) tma_load_2d(sm + 8192, &tm_small, bar, j0 + 64, m0);
      });
    }
    return;
  }
  bool failed = false;
  const int q = lane >> 3, i8 = lane & 7;
  const int cl = 16 * warp + (q & 1) * 8;
  const uint32_t cblk = static_cast<uint32_t>(cl >> 6) * 8192u;
  const uint32_t cch = static_cast<uint32_t>(cl & 63) >> 3;
  const int r_lo = 16 * warp + (lane >> 2);
  int i = 0;  // ring position (steps consumed by this CTA)
  for (int ti = 0; ti < my_tiles; ++ti) {
    const int c0 = (bid + ti * nb) * kTileRows;
    float tot[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) tot[t][0] = tot[t][1] = tot[t][2] = tot[t][3] = 0.f;
    for (int rq = 0; rq < a.split; ++rq) {
      const int s0 = static_cast<int>(static_cast<long long>(a.steps) * rq / a.split);
      const int s1 = static_cast<int>(static_cast<long long>(a.steps) * (rq + 1) / a.split);
      float acc[NT][4];
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
      for (int s = s0; s < s1; ++s, ++i) {
        const int st = i % a.stages;
        if (!failed)
          failed = !mbar_wait_warp(full + st, static_cast<uint32_t>(i / a.stages) & 1u,
                                   kErrWaitFull, a.err, i);
        if (!failed) {
          const uint32_t bb = smem_u32(ring + st * a.stage_bytes);
          const uint32_t sb = bb + kBigTileBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint32_t af[4];
            const int tok = 16 * kk + i8 + (q >> 1) * 8;
            ldsm_x4_t(af, bb + cblk + sw128_off(tok, cch));
            const int l = lane & 15;
            const int k = 16 * kk + (l & 7) + ((l >> 3) << 3);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              uint32_t b[2];
              ldsm_x2_t(b, sb + small_off(a, k, static_cast<uint32_t>(t)));
              mma16816(acc[t], af, b[0], b[1]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + st);
      }
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) tot[t][e] += acc[t][e];
    }
    if (failed) continue;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int col = t * 8 + (lane & 3) * 2;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = c0 + r_lo + 8 * h;
        if (c >= a.C) continue;
        const float v0 = a.scale * tot[t][2 * h], v1 = a.scale * tot[t][2 * h + 1];
        if (a.out_cr)  // out [C, R]
          *reinterpret_cast<float2*>(a.out + static_cast<long long>(c) * a.R + col) =
              make_float2(v0, v1);
        else {  // out [R, C]
          a.out[static_cast<long long>(col) * a.C + c] = v0;
          a.out[static_cast<long long>(col + 1) * a.C + c] = v1;
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// down, many tokens (rank_down_rows_kernel): each warp owns 16 token rows over the whole
// reduction, so there is nothing to reduce across warps or CTAs.  A CTA (2 consumer warps, 32
// rows) streams its rows in stages of 256 columns -- 512 contiguous bytes of every row, four
// 64-column SW128 boxes -- together with the matching 256 columns of Wl (A [R, C]: four boxes
// of R rows; B [C, rg]: one box of 256 rows).  For R <= 32, where Wl's slice is no larger than
// the activation's.
// ------------------------------------------------------------------------------------------
constexpr int kRowWarps = 2;
constexpr int kRowThreads = 32 * (kRowWarps + 1);
constexpr int kRowRows = 16 * kRowWarps;
constexpr uint32_t kRowXBytes = kRowRows * 512u;  // 32 rows x 256 bf16

template <int NT, bool kWrc>
__global__ void __launch_bounds__(kRowThreads, 2)
    rank_down_rows_kernel(const __grid_constant__ CUtensorMap tm_in,
                          const __grid_constant__ CUtensorMap tm_w, const RankArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + a.ring_bytes);
  uint64_t* empty = full + a.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = static_cast<int>(blockIdx.x) * kRowRows;
  const int n = a.steps;  // stages of 256 columns

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kRowWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // the previous kernel's outputs are complete
  pdl_trigger();

  if (warp == kRowWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_in);
      tma_prefetch_desc(&tm_w);
      rank_produce(a, ring, full, empty, n, [&](int i, uint8_t* dst, uint64_t* bar) {
        const int c0 = i * 256;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          tma_load_2d(dst + b * (kRowXBytes / 4), &tm_in, bar, c0 + 64 * b, row0);
        uint8_t* w = dst + kRowXBytes;
        if (kWrc) {
#pragma unroll
          for (int b = 0; b < 4; ++b)
            tma_load_2d(w + b * (a.small_bytes / 4), &tm_w, bar, c0 + 64 * b, 0);  // A [R, 64]
        } else {
          tma_load_2d(w, &tm_w, bar, 0, c0);  // B [256 c, rg]
        }
      });
    }
    return;
  }
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  bool failed = false;
  const int ar = 16 * warp + (lane & 15);
  for (int i = 0; i < n; ++i) {
    const int st = i % a.stages;
    if (!failed)
      failed = !mbar_wait_warp(full + st, static_cast<uint32_t>(i / a.stages) & 1u,
                               kErrWaitFull, a.err, i);
    if (!failed) {
      const uint32_t xb = smem_u32(ring + st * a.stage_bytes);
      const uint32_t wb = xb + kRowXBytes;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t xbb = xb + b * (kRowXBytes / 4);
        const int g = kWrc ? 0 : row_group(a.groups, i * 256 + 64 * b);
        const int t_lo = kWrc ? 0 : g * (a.rg / 8);
        const int t_hi = kWrc ? NT : t_lo + a.rg / 8;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t af[4];
          ldsm_x4(af, xbb + sw128_off(ar, 2 * kk + (lane >> 4)));
          if (kWrc) {
            const uint32_t wbb = wb + b * (a.small_bytes / 4);
#pragma unroll
            for (int t = 0; t + 1 < NT; t += 2) {
              const int j = t * 8 + (lane & 7) + ((lane >> 4) << 3);
              uint32_t bb[4];
              ldsm_x4(bb, wbb + sw128_off(j, 2 * kk + ((lane >> 3) & 1)));
              mma16816(acc[t], af, bb[0], bb[1]);
              mma16816(acc[t + 1], af, bb[2], bb[3]);
            }
            if (NT & 1) {
              constexpr int t = NT - 1;
              const int l = lane & 15;
              uint32_t bb[2];
              ldsm_x2(bb, wbb + sw128_off(t * 8 + (l & 7), 2 * kk + (l >> 3)));
              mma16816(acc[t], af, bb[0], bb[1]);
            }
          } else {
            const int l = lane & 15;
            const int k = 64 * b + 16 * kk + (l & 7) + ((l >> 3) << 3);  // row c of the B tile
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              if (t >= t_lo && t < t_hi) {
                uint32_t bb[2];
                ldsm_x2_t(bb, wb + small_off(a, k, static_cast<uint32_t>(t - t_lo)));
                mma16816(acc[t], af, bb[0], bb[1]);
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + st);
  }
  const int r_lo = row0 + 16 * warp + (lane >> 2);
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int col = t * 8 + (lane & 3) * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = r_lo + 8 * h;
      if (m >= a.M) continue;
      const float v0 = acc[t][2 * h], v1 = acc[t][2 * h + 1];
      const long long o = static_cast<long long>(m) * a.R + col;
      if (a.saved)
        *reinterpret_cast<__nv_bfloat162*>(a.saved + o) = __floats2bfloat162_rn(v0, v1);
      *reinterpret_cast<__nv_bfloat162*>(a.scaled + o) =
          __floats2bfloat162_rn(a.scale * v0, a.scale * v1);
    }
  }
}

// Launch with the cluster dimension (S CTAs along x), as a programmatic dependent.
template <typename K>
cudaError_t launch_clustered(K kernel, int grid, int split, size_t smem, cudaStream_t stream,
                             const CUtensorMap& m0, const CUtensorMap& m1, const RankArgs& a,
                             int threads = kRankThreads) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kernel, dim3(static_cast<unsigned>(grid)), dim3(threads), smem, stream,
                    split, m0, m1, a);
}

// CTAs per cluster: the largest power of two (<= 8, <= the steps) that keeps the grid within
// two CTAs per SM.
int pick_split(int tiles, int steps, int sm_count) {
  int s = 1;
  while (s < kMaxSplit && tiles * s * 2 <= 2 * sm_count && s * 2 <= steps) s *= 2;
  return s;
}

}  // namespace

// Layout of a [64 rows, w columns] bf16 tile (w a multiple of 8, at most 128) as TMA writes
// it: w = 8, 16, 32, 64 fill rows of 16..128 bytes with the swizzle of the same span
// (conflict-free transposed 8x8 loads); w = 128 takes two 64-column SW128 blocks; any other w
// keeps unswizzled rows of 2w bytes (an odd number of 16-byte chunks, or at most a 2- to
// 4-way bank conflict).
SmallTile small_tile(int w) {
  SmallTile t;
  t.blocks = 1;
  t.box_w = w;
  t.pitch = static_cast<uint32_t>(2 * w);
  t.mask = 0;
  t.swizzle = 0;
  if (w == 128) {
    t.blocks = 2;
    t.box_w = 64;
    t.pitch = 128;
    t.mask = 7;
    t.swizzle = 128;
  } else if (w == 16 || w == 32 || w == 64) {
    t.mask = t.pitch / 16 - 1;
    t.swizzle = static_cast<int>(t.pitch);
  }
  t.bytes = 64u * t.pitch * static_cast<uint32_t>(t.blocks);
  return t;
}

namespace {

}  // namespace

RankPlan rank_down_plan(int M, int C, int R, int rg, bool w_rc, int sm_count,
                        size_t scratch_bytes) {
  RankPlan p;
  p.gsplit = 1;
  p.part_bytes = 0;
  const int row_ctas = (M + kRowRows - 1) / kRowRows;
  // (A [R, C] only: with B the 256-row box of narrow rows measured slower than the cluster kernel.)
  if (w_rc && R <= 32 && 3 * row_ctas >= 2 * sm_count) {
    // Many tokens and a narrow rank: whole rows per warp, no reduction across CTAs.
    p.rows = 1;
    p.split = 1;
    p.grid = row_ctas;
    p.box_rows_in = kRowRows;
    p.small = w_rc ? SmallTile{1, 64, 128u, 7u, 128, static_cast<uint32_t>(R) * 512u}
                   : small_tile(rg);
    if (!w_rc) p.small.bytes = 256u * p.small.pitch;  // one box of 256 rows of B
    p.box_rows_w = w_rc ? R : 256;
    const uint32_t stage = kRowXBytes + ((p.small.bytes + 1023u) & ~1023u);
    p.stages = static_cast<int>((110u * 1024u - 2048u) / stage);
    if (p.stages > 8) p.stages = 8;
    p.smem = 1024 + static_cast<size_t>(p.stages) * stage + 2 * 8 * p.stages;
    return p;
  }
  p.rows = 0;
  const int tiles = (M + kTileRows - 1) / kTileRows;
  p.split = pick_split(tiles, C / 64, sm_count);
  // Few tokens: too few clusters to stream `in` at full rate, so split the reduction further
  // over gsplit clusters (at least two steps each, within two CTAs per SM) when the workspace
  // holds their partials.
  while (tiles * p.split * p.gsplit * 2 <= 2 * sm_count &&
         p.split * p.gsplit * 2 * 2 <= C / 64 &&
         static_cast<size_t>(tiles) * p.gsplit * 2 * kTileRows * R * 4 <= scratch_bytes)
    p.gsplit *= 2;
  if (p.gsplit > 1)
    p.part_bytes = static_cast<size_t>(tiles) * p.gsplit * kTileRows * R * 4;
  p.grid = tiles * p.split * p.gsplit;
  p.box_rows_in = kTileRows;
  p.small = w_rc ? SmallTile{1, 64, 128u, 7u, 128, static_cast<uint32_t>(R) * 128u}
                 : small_tile(rg);
  p.box_rows_w = w_rc ? R : 64;
  const RankLayout L = rank_layout(p.small.bytes, R, R <= 64 ? 110 * 1024 : 200 * 1024);
  p.stages = L.stages;
  p.smem = L.smem;
  return p;
}

RankPlan rank_grad_plan(int M, int C, int R, int sm_count) {
  RankPlan p;
  p.gsplit = 1;
  p.part_bytes = 0;
  p.rows = 0;
  p.box_rows_in = 64;
  p.box_rows_w = 64;
  const int tiles = (C + kTileRows - 1) / kTileRows;
  p.split = pick_split(tiles, (M + 63) / 64, sm_count);
  p.grid = tiles * p.split;
  p.small = small_tile(R);
  const RankLayout L = rank_layout(p.small.bytes, R, R <= 64 ? 110 * 1024 : 200 * 1024);
  p.stages = L.stages;
  p.smem = L.smem;
  return p;
}

cudaError_t launch_down_cluster(const RankMaps& maps, const RankPlan& p, int R, bool w_rc,
                                const RankArgs& a, cudaStream_t stream);

#define QLORA_RANK_DOWN_CASE(NTV)                                                              \
  case NTV:                                                                                   \
    return w_rc ? launch_clustered(rank_down_kernel<NTV, true>, p.grid, p.split, p.smem, stream, \
                                   maps.big, maps.small, a)                                   \
                : launch_clustered(rank_down_kernel<NTV, false>, p.grid, p.split, p.smem,      \
                                   stream, maps.big, maps.small, a);

#define QLORA_RANK_ROWS_CASE(NTV)                                                              \
  case NTV:                                                                                   \
    return w_rc ? launch_clustered(rank_down_rows_kernel<NTV, true>, p.grid, 1, p.smem, stream,  \
                                   maps.big, maps.small, a, kRowThreads)                      \
                : launch_clustered(rank_down_rows_kernel<NTV, false>, p.grid, 1, p.smem,       \
                                   stream, maps.big, maps.small, a, kRowThreads);

cudaError_t launch_rank_down(const RankMaps& maps, const RankPlan& p, int M, int C, int R, int rg,
                             bool w_rc, const RowGroups& groups, float scale,
                             __nv_bfloat16* saved, __nv_bfloat16* scaled, int* err,
                             cudaStream_t stream, float* scratch, bool finalize) {
  RankArgs a = {};
  a.gsplit = 1;
  a.gpart = nullptr;
  a.M = M;
  a.C = C;
  a.R = R;
  a.rg = rg;
  a.steps = C / 64;
  a.split = p.split;
  if (p.rows) {
    a.steps = (C + 255) / 256;
    a.stages = p.stages;
    a.small_bytes = (p.small.bytes + 1023u) & ~1023u;
    a.stage_bytes = kRowXBytes + a.small_bytes;
    a.ring_bytes = static_cast<uint32_t>(p.stages) * a.stage_bytes;
    a.small_pitch = p.small.pitch;
    a.small_mask = p.small.mask;
    a.small_blocks = p.small.blocks;
    a.scale = scale;
    a.groups = groups;
    a.saved = saved;
    a.scaled = scaled;
    a.err = err;
    if (a.small_bytes != p.small.bytes || p.small.blocks != 1) return cudaErrorInvalidValue;
    switch (R / 8) {
      QLORA_RANK_ROWS_CASE(1)
      QLORA_RANK_ROWS_CASE(2)
      QLORA_RANK_ROWS_CASE(3)
      QLORA_RANK_ROWS_CASE(4)
      default:
        return cudaErrorInvalidValue;
    }
  }
  const RankLayout L = rank_layout(p.small.bytes, R, R <= 64 ? 110 * 1024 : 200 * 1024);
  a.stages = L.stages;
  a.stage_bytes = L.stage_bytes;
  a.small_bytes = L.small_bytes;
  a.ring_bytes = L.ring_bytes;
  a.small_pitch = p.small.pitch;
  a.small_mask = p.small.mask;
  a.small_blocks = p.small.blocks;
  // The ring's expected bytes per stage are exactly what its copies deliver.
  if (L.small_bytes != p.small.bytes) return cudaErrorInvalidValue;
  a.scale = scale;
  a.groups = groups;
  a.saved = saved;
  a.scaled = scaled;
  a.err = err;
  if (p.gsplit > 1) {
    if (!scratch || R % 4 != 0) return cudaErrorInvalidValue;
    a.gsplit = p.gsplit;
    a.gpart = scratch;
    const cudaError_t e = launch_down_cluster(maps, p, R, w_rc, a, stream);
    if (e != cudaSuccess || !finalize) return e;
    const int items = M * (R / 4);
    return launch_pdl(rank_down_finalize, dim3((items + 255) / 256), dim3(256), 0, stream, 1, a);
  }
  return launch_down_cluster(maps, p, R, w_rc, a, stream);
}

cudaError_t launch_down_cluster(const RankMaps& maps, const RankPlan& p, int R, bool w_rc,
                                const RankArgs& a, cudaStream_t stream) {
  switch (R / 8) {
    QLORA_RANK_DOWN_CASE(1)
    QLORA_RANK_DOWN_CASE(2)
    QLORA_RANK_DOWN_CASE(3)
    QLORA_RANK_DOWN_CASE(4)
    QLORA_RANK_DOWN_CASE(5)
    QLORA_RANK_DOWN_CASE(6)
    QLORA_RANK_DOWN_CASE(7)
    QLORA_RANK_DOWN_CASE(8)
    QLORA_RANK_DOWN_CASE(9)
    QLORA_RANK_DOWN_CASE(10)
    QLORA_RANK_DOWN_CASE(11)
    QLORA_RANK_DOWN_CASE(12)
    QLORA_RANK_DOWN_CASE(13)
    QLORA_RANK_DOWN_CASE(14)
    QLORA_RANK_DOWN_CASE(15)
    QLORA_RANK_DOWN_CASE(16)
    default:
      return cudaErrorInvalidValue;
  }
}
#undef QLORA_RANK_DOWN_CASE
#undef QLORA_RANK_ROWS_CASE

namespace {

RankArgs grad_args(const RankPlan& p, int M, int C, int R, int ld_small, const RowGroups& groups,
                   float scale, float* out, bool out_cr, int* err, bool* ok) {
  RankArgs a = {};
  a.M = M;
  a.C = C;
  a.R = R;
  a.rg = R;
  a.steps = (M + 63) / 64;
  a.split = p.split;
  const RankLayout L = rank_layout(p.small.bytes, R, R <= 64 ? 110 * 1024 : 200 * 1024);
  a.stages = L.stages;
  a.stage_bytes = L.stage_bytes;
  a.small_bytes = L.small_bytes;
  a.ring_bytes = L.ring_bytes;
  a.small_pitch = p.small.pitch;
  a.small_mask = p.small.mask;
  a.small_blocks = p.small.blocks;
  // The ring's expected bytes per stage are exactly what its copies deliver.
  *ok = L.small_bytes == p.small.bytes;
  a.ld_small = ld_small;
  a.scale = scale;
  a.groups = groups;
  a.out = out;
  a.out_cr = out_cr ? 1 : 0;
  a.err = err;
  return a;
}

template <int NT>
cudaError_t launch_grad_nt(const RankMaps& m1, const RankArgs& a1, int grid1, const RankMaps& m2,
                           const RankArgs& a2, int grid2, int split, size_t smem,
                           cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(rank_grad_kernel<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(rank_grad_kernel<NT>, dim3(static_cast<unsigned>(grid1 + grid2)),
                    dim3(kRankThreads), smem, stream, split, m1.big, m1.small, a1, m2.big,
                    m2.small, a2, grid1);
}

cudaError_t launch_grad_any(int R, const RankMaps& m1, const RankArgs& a1, int grid1,
                            const RankMaps& m2, const RankArgs& a2, int grid2, int split,
                            size_t smem, cudaStream_t stream) {
  switch (R / 8) {
#define QLORA_RANK_GRAD_CASE(NTV) \
  case NTV:                       \
    return launch_grad_nt<NTV>(m1, a1, grid1, m2, a2, grid2, split, smem, stream);
    QLORA_RANK_GRAD_CASE(1)
    QLORA_RANK_GRAD_CASE(2)
    QLORA_RANK_GRAD_CASE(3)
    QLORA_RANK_GRAD_CASE(4)
    QLORA_RANK_GRAD_CASE(5)
    QLORA_RANK_GRAD_CASE(6)
    QLORA_RANK_GRAD_CASE(7)
    QLORA_RANK_GRAD_CASE(8)
    QLORA_RANK_GRAD_CASE(9)
    QLORA_RANK_GRAD_CASE(10)
    QLORA_RANK_GRAD_CASE(11)
    QLORA_RANK_GRAD_CASE(12)
    QLORA_RANK_GRAD_CASE(13)
    QLORA_RANK_GRAD_CASE(14)
    QLORA_RANK_GRAD_CASE(15)
    QLORA_RANK_GRAD_CASE(16)
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_rank_grad(const RankMaps& maps, const RankPlan& p, int M, int C, int R,
                             int ld_small, const RowGroups& groups, float scale, float* out,
                             bool out_cr, int* err, cudaStream_t stream) {
  bool ok = true;
  const RankArgs a = grad_args(p, M, C, R, ld_small, groups, scale, out, out_cr, err, &ok);
  if (!ok) return cudaErrorInvalidValue;
  return launch_grad_any(R, maps, a, p.grid, maps, a, 0, p.split, p.smem, stream);
}

namespace {

// The side kernel has an SM to itself: a deeper ring than the cluster kernel's two CTAs per SM.
constexpr int kSideBudget = 220 * 1024;
constexpr int kSideMaxStages = 12;

RankArgs side_args(const RankPlan& p, int M, int C, int R, int ld_small, const RowGroups& groups,
                   float scale, float* out, bool out_cr, int* err, bool* ok, size_t* smem) {
  RankArgs a = grad_args(p, M, C, R, ld_small, groups, scale, out, out_cr, err, ok);
  const RankLayout L = rank_layout(p.small.bytes, R, kSideBudget, kSideMaxStages);
  a.stages = L.stages;
  a.stage_bytes = L.stage_bytes;
  a.small_bytes = L.small_bytes;
  a.ring_bytes = L.ring_bytes;
  *ok = *ok && L.small_bytes == p.small.bytes;
  *smem = L.smem;
  return a;
}

template <int NT>
cudaError_t launch_side_nt(const RankMaps& m1, const RankArgs& a1, int grid1, const RankMaps& m2,
                           const RankArgs& a2, int grid2, size_t smem, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(rank_grad_loop_kernel<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_kernel(rank_grad_loop_kernel<NT>, dim3(static_cast<unsigned>(grid1 + grid2)),
                       dim3(kRankThreads), smem, stream, false, 1, m1.big, m1.small, a1, m2.big,
                       m2.small, a2, grid1);
}

cudaError_t launch_side_any(int R, const RankMaps& m1, const RankArgs& a1, int grid1,
                            const RankMaps& m2, const RankArgs& a2, int grid2, size_t smem,
                            cudaStream_t stream) {
  switch (R / 8) {
#define QLORA_RANK_SIDE_CASE(NTV) \
  case NTV:                       \
    return launch_side_nt<NTV>(m1, a1, grid1, m2, a2, grid2, smem, stream);
    QLORA_RANK_SIDE_CASE(1)
    QLORA_RANK_SIDE_CASE(2)
    QLORA_RANK_SIDE_CASE(3)
    QLORA_RANK_SIDE_CASE(4)
    QLORA_RANK_SIDE_CASE(5)
    QLORA_RANK_SIDE_CASE(6)
    QLORA_RANK_SIDE_CASE(7)
    QLORA_RANK_SIDE_CASE(8)
    QLORA_RANK_SIDE_CASE(9)
    QLORA_RANK_SIDE_CASE(10)
    QLORA_RANK_SIDE_CASE(11)
    QLORA_RANK_SIDE_CASE(12)
    QLORA_RANK_SIDE_CASE(13)
    QLORA_RANK_SIDE_CASE(14)
    QLORA_RANK_SIDE_CASE(15)
    QLORA_RANK_SIDE_CASE(16)
#undef QLORA_RANK_SIDE_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_rank_grad_side(const RankMaps& m1, const RankPlan& p1, int M, int C1, int R1,
                                  int ld1, const RowGroups& g1, float* out1, bool cr1,
                                  const RankMaps* m2, const RankPlan* p2, int C2, int R2,
                                  int ld2, const RowGroups& g2, float* out2, bool cr2,
                                  float scale, int* err, int ctas, cudaStream_t stream) {
  bool ok = true;
  size_t smem1 = 0, smem2 = 0;
  const RankArgs a1 = side_args(p1, M, C1, R1, ld1, g1, scale, out1, cr1, err, &ok, &smem1);
  if (!ok) return cudaErrorInvalidValue;
  if (!m2) {
    if (ctas < 1) return cudaErrorInvalidValue;
    return launch_side_any(R1, m1, a1, ctas, m1, a1, 0, smem1, stream);
  }
  // Two problems in one launch need one instance (same rank); CTAs split by their bytes.
  if (!p2 || R2 != R1 || ctas < 2) return cudaErrorInvalidValue;
  const RankArgs a2 = side_args(*p2, M, C2, R2, ld2, g2, scale, out2, cr2, err, &ok, &smem2);
  if (!ok) return cudaErrorInvalidValue;
  int grid1 = static_cast<int>((static_cast<long long>(ctas) * C1 + (C1 + C2) / 2) / (C1 + C2));
  grid1 = grid1 < 1 ? 1 : (grid1 > ctas - 1 ? ctas - 1 : grid1);
  return launch_side_any(R1, m1, a1, grid1, *m2, a2, ctas - grid1,
                         smem1 > smem2 ? smem1 : smem2, stream);
}

bool rank_grad_pair_ok(const RankPlan& p1, int R1, const RankPlan& p2, int R2) {
  return R1 == R2 && p1.split == p2.split && p1.small.bytes == p2.small.bytes &&
         p1.small.pitch == p2.small.pitch && p1.small.blocks == p2.small.blocks;
}

cudaError_t launch_rank_grad_pair(const RankMaps& m1, const RankPlan& p1, int M, int C1, int R,
                                  int ld1, const RowGroups& g1, float* out1, bool cr1,
                                  const RankMaps& m2, const RankPlan& p2, int C2, int ld2,
                                  const RowGroups& g2, float* out2, bool cr2, float scale,
                                  int* err, cudaStream_t stream) {
  bool ok1 = true, ok2 = true;
  const RankArgs a1 = grad_args(p1, M, C1, R, ld1, g1, scale, out1, cr1, err, &ok1);
  const RankArgs a2 = grad_args(p2, M, C2, R, ld2, g2, scale, out2, cr2, err, &ok2);
  if (!ok1 || !ok2 || !rank_grad_pair_ok(p1, R, p2, R)) return cudaErrorInvalidValue;
  return launch_grad_any(R, m1, a1, p1.grid, m2, a2, p2.grid, p1.split,
                         p1.smem > p2.smem ? p1.smem : p2.smem, stream);
}

#undef QLORA_RANK_GRAD_CASE

}  // namespace qlora

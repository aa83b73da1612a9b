// sm_100a kernels of the attention output projection (DeepSeek-V3.2-Exp,
// model.py 607-608 as shown on the atlas page "Attention update"): the head
// outputs of a row are flattened (128 heads x 128 value dimensions = 16384)
// and projected back to the model width by wo:
//
//   delta[b, n] = bf16( sum_k x[b, k] * wo[n, k] ),   k < 16384, n < dim
//
// wo is the torch Linear weight [dim, 16384] (k contiguous); the pages show no
// bias.  The kernels take the input width as a runtime multiple of 64 and wo
// with a row stride, so a tensor-parallel shard projects its own heads'
// outputs through its column slice of wo (the row-parallel partial, summed
// over the shards afterwards).  At decode sizes the projection is a stream over wo (235 MB at
// dim = 7168) with a narrow batch, so it is written as a weight stream:
//
//   projection_kernel  persistent swap-AB tcgen05 GEMM.  An output tile is
//                      (batch tile y of n_tile <= 256 rows, wo tile m of 128
//                      rows); a work unit is (tile, k-block of 64): A = wo
//                      box [128 x 64], B = x box [n_tile x 64], both by TMA
//                      (128B swizzle) into a ring of stages; D[n, b] in TMEM.
//                      With fewer tiles than SMs, CTA c takes the contiguous
//                      unit range [c U / C, (c+1) U / C) of all U = tiles x
//                      256 units, so every SM streams the same number of
//                      weight bytes; a range covers at most two tiles
//                      (segments), and each segment's accumulator (two TMEM
//                      buffers, so the MMAs run on while the previous one
//                      drains) goes to an f32 partial slot.  With at least as
//                      many tiles as SMs, CTA c computes tile c whole and
//                      writes bf16 directly ("direct").
//   projection_reduce_kernel  sums the partial slots of each tile in a fixed
//                      order (deterministic) and rounds to bf16.
//
// Warp roles of projection_kernel (192 threads): warps 0-3 drain the
// accumulator (TMEM lane quarter = warp), warp 4 lane 0 issues TMA, warp 5
// allocates TMEM and its lane 0 issues the MMAs.
//
// A prepared wo (prepare_wo_kernel, once per weight) holds every 128 x 256
// block of wo as 64 contiguous KB laid out exactly as the kernel's shared
// memory wants it, so a work unit's weights arrive by one bulk copy: read in
// place, the same unit touches 512 bytes in each of 128 rows 32 KB apart, and
// the short runs cost DRAM bandwidth (each run opens a DRAM row for 512 bytes).
#pragma once

#include "kernels.cuh"
#include "projection_plan.h"

namespace mla {

constexpr int kProjK = kH * kDv;                   // 16384 inputs per row (all heads)
constexpr int kProjKBlock = 64;                    // k per unit: one 128-byte swizzle row
constexpr int kProjKBlocks = kProjK / kProjKBlock; // 256 k-blocks per row tile (all heads)
constexpr int kProjM = 128;                        // wo rows per tile (MMA M)
constexpr int kProjNMax = 256;                     // batch rows per tile (MMA N, TMA box)
constexpr int kProjStagesMax = 8;
constexpr int kProjStageBudget = 200 * 1024;       // shared memory for the ring
constexpr int kProjABytes = kProjM * kProjKBlock * 2;  // 16 KB
constexpr int kProjThreads = 192;
constexpr int kProjTileK = 4 * kProjKBlock;        // columns of one prepared block (64 KB)
constexpr int kProjReduceRows = 16;                // batch rows per reduce CTA

// A unit covers kgroup consecutive k-blocks: 1, or kProjKGroupWide when the
// batch tile is narrow enough for two such stages (then the wo box reads four
// consecutive 128-byte pieces of every row back to back).
constexpr int kProjKGroupWide = 4;
constexpr int kProjWideNMax = 64;  // widest batch tile that uses kProjKGroupWide
__host__ __device__ constexpr int proj_stage_bytes(int n_tile, int kgroup) {
  return kgroup * (kProjABytes + n_tile * kProjKBlock * 2);
}
__host__ __device__ constexpr int proj_stages(int n_tile, int kgroup) {
  return kProjStageBudget / proj_stage_bytes(n_tile, kgroup) < kProjStagesMax
             ? kProjStageBudget / proj_stage_bytes(n_tile, kgroup)
             : kProjStagesMax;
}
// shared memory of one CTA: the ring, barriers, alignment pad
__host__ __device__ constexpr int proj_smem_bytes(int n_tile, int kgroup) {
  return proj_stages(n_tile, kgroup) * proj_stage_bytes(n_tile, kgroup) + 256 + kSmemAlignPad;
}
// the largest of them, over the batch tiles and unit widths the host can choose
constexpr int proj_smem_max() {
  int m = 0;
  for (int n = 16; n <= kProjNMax; n += 16) {
    m = proj_smem_bytes(n, 1) > m ? proj_smem_bytes(n, 1) : m;
    if (n <= kProjWideNMax) m = proj_smem_bytes(n, kProjKGroupWide) > m ? proj_smem_bytes(n, kProjKGroupWide) : m;
  }
  return m;
}
static_assert(proj_smem_max() <= 232448, "shared memory");
static_assert(proj_stages(kProjNMax, 1) >= 2 && proj_stages(kProjWideNMax, kProjKGroupWide) >= 2, "ring depth");

// The prepared layout of wo [dim, k_in] (dim % 128 == 0, k_in % 256 == 0):
// block (m, g) = rows [128 m, 128 m + 128) x columns [256 g, 256 g + 256),
// at ((m * (k_in / 256)) + g) * 64 KB; inside it, 64-column k-block j at
// j * 16 KB, 8-row group r at r * 1 KB, row i of the group at i * 128 B and
// its 16-byte chunk q (columns 8q .. 8q + 7 of the k-block) at (q ^ i) * 16 B
// (the 128-byte swizzle of a K-major UMMA operand).  One thread per chunk.
__global__ void __launch_bounds__(256)
prepare_wo_kernel(const uint4* __restrict__ wo, long long ld_chunks, int dim, int k_in, uint4* __restrict__ out) {
  const long long row_chunks = k_in / 8;
  const long long n = (long long)dim * row_chunks;
  const long long blocks_per_row = k_in / kProjTileK;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < n; c += (long long)gridDim.x * blockDim.x) {
    const long long row = c / row_chunks;
    const int qa = (int)(c - row * row_chunks);  // chunk within the row
    const long long m = row / kProjM;
    const int rr = (int)(row - m * kProjM), r = rr >> 3, i = rr & 7;
    const int g = qa >> 5, j = (qa >> 3) & 3, q = qa & 7;
    const long long dst = (m * blocks_per_row + g) * 4096 + j * 1024 + r * 64 + i * 8 + (q ^ i);
    out[dst] = wo[row * ld_chunks + qa];
  }
}

__global__ void __launch_bounds__(kProjThreads, 1)
projection_kernel(const __grid_constant__ CUtensorMap tm_wo, const __grid_constant__ CUtensorMap tm_wo4,
                  const __grid_constant__ CUtensorMap tm_x, const __nv_bfloat16* __restrict__ wo_prepared,
                  float* __restrict__ partial, __nv_bfloat16* __restrict__ delta, int B, int dim, int n_tile,
                  int n_ctas, int direct, int kgroup, int k_blocks, int* d_status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int stages = proj_stages(n_tile, kgroup);
  const int stage_bytes = proj_stage_bytes(n_tile, kgroup);
  const int upt = k_blocks / kgroup;            // units per tile
  const int a_bytes = kgroup * kProjABytes;     // wo part of a stage; the x boxes follow
  const int m_tiles = dim / kProjM;
  const long long U = (long long)m_tiles * ((B + n_tile - 1) / n_tile) * upt;
  const long long u0 = proj_unit_begin<long long>(c, U, n_ctas);
  const int n_units = (int)(proj_unit_begin<long long>(c + 1, U, n_ctas) - u0);
  const long long t0 = u0 / upt;  // first tile of this CTA
  const int n_seg = n_units > 0 ? (int)((u0 + n_units - 1) / upt - t0) + 1 : 0;  // <= 2
  // unit u: tile u / upt = y * m_tiles + m, first k-block (u % upt) * kgroup
  auto unit_m = [&](long long u) { return (int)((u / upt) % m_tiles); };
  auto unit_row0 = [&](long long u) { return (int)((u / upt) / m_tiles) * n_tile; };
  auto unit_kb0 = [&](long long u) { return (int)(u % upt) * kgroup; };
  // wo part of a unit: one 2-D box [128 rows x 64], or with kgroup = 4 one
  // 4-D box over (64 k, 8 rows, 4 k-blocks, 16 row groups), which lands as
  // [group][k-block][row][128 B]: 8-row x 128-byte swizzle atoms, the groups
  // 4 KB apart, k-block j at j KB
  auto load_wo = [&](uint32_t dst, uint32_t bar, long long u) {
    if (wo_prepared != nullptr) {  // kgroup k-blocks of one prepared block, contiguous
      const int kb0 = unit_kb0(u);
      const __nv_bfloat16* src = wo_prepared +
                                 ((size_t)unit_m(u) * (k_blocks / 4) + kb0 / 4) * (size_t)(kProjM * kProjTileK) +
                                 (size_t)(kb0 % 4) * (kProjM * kProjKBlock);
      bulk_load(dst, src, (uint32_t)(kgroup * kProjABytes), bar);
    } else if (kgroup == 1)
      tma_load_2d(dst, &tm_wo, bar, unit_kb0(u) * kProjKBlock, unit_m(u) * kProjM);
    else
      tma_load_4d(dst, &tm_wo4, bar, 0, 0, unit_kb0(u), unit_m(u) * (kProjM / 8));
  };
  auto load_x = [&](uint32_t dst, uint32_t bar, long long u) {
    for (int j = 0; j < kgroup; ++j)
      tma_load_2d(dst + j * n_tile * kProjKBlock * 2, &tm_x, bar, (unit_kb0(u) + j) * kProjKBlock, unit_row0(u));
  };

  const uint32_t sRing = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  auto full = [&](int s) { return smem_u32(&bars[s]); };
  auto empty = [&](int s) { return smem_u32(&bars[kProjStagesMax + s]); };
  auto acc_full = [&](int a) { return smem_u32(&bars[2 * kProjStagesMax + a]); };
  auto acc_empty = [&](int a) { return smem_u32(&bars[2 * kProjStagesMax + 2 + a]); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[2 * kProjStagesMax + 4]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[2 * kProjStagesMax + 5]);
  const AbortState ab{abort_flag, d_status};
  // one accumulator buffer: n_tile f32 columns, rounded to a power of two
  const uint32_t acc_cols = n_tile <= 32 ? 32u : (n_tile <= 64 ? 64u : (n_tile <= 128 ? 128u : 256u));

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kProjStagesMax; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(acc_full(a), 1);
      mbar_init(acc_empty(a), 4);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 2 * acc_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA
    if (lane == 0 && n_units > 0) {
      if (wo_prepared == nullptr) tma_prefetch_desc(kgroup == 1 ? &tm_wo : &tm_wo4);
      tma_prefetch_desc(&tm_x);
      // The first stages' weights go out before the wait on the kernel that
      // writes x (programmatic dependent launch): wo does not depend on it.
      const int pre = n_units < stages ? n_units : stages;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(full(i), stage_bytes);
        load_wo(sRing + i * stage_bytes, full(i), u0 + i);
      }
      grid_dep_wait();
      for (int i = 0; i < pre; ++i) load_x(sRing + i * stage_bytes + a_bytes, full(i), u0 + i);
      for (int i = pre, st = pre % stages; i < n_units; ++i, st = (st + 1 == stages) ? 0 : st + 1) {
        const long long u = u0 + i;
        wait(empty(st), ((i / stages) - 1) & 1, ab);
        const uint32_t dst = sRing + st * stage_bytes;
        mbar_arrive_expect_tx(full(st), stage_bytes);
        load_wo(dst, full(st), u);
        load_x(dst + a_bytes, full(st), u);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA
    if (lane == 0 && n_units > 0) {
      const uint32_t idesc = idesc_bf16_f32(kProjM, n_tile, false, false);
      int seg = 0;
      for (int i = 0, st = 0; i < n_units; ++i, st = (st + 1 == stages) ? 0 : st + 1) {
        const long long u = u0 + i;
        const bool first = (i == 0) || (u % upt == 0);
        const bool last = (i == n_units - 1) || ((u + 1) % upt == 0);
        const int acc = seg & 1;
        if (first && seg >= 2) wait(acc_empty(acc), ((seg - 2) >> 1) & 1, ab);
        wait(full(st), (i / stages) & 1, ab);
        tc_fence_after();
        const uint32_t a0 = sRing + st * stage_bytes;
        const uint32_t b0 = a0 + a_bytes;
        // wo k-block j: the 2-D box (8-row groups 1 KB apart), block j of
        // the 4-D box (groups kgroup KB apart, block j at j KB), or k-block j
        // of a prepared block (groups 1 KB apart, block j at j * 16 KB)
        const uint32_t a_sbo = wo_prepared != nullptr ? 1024u : 1024u * (uint32_t)kgroup;
        const uint32_t a_jstride = wo_prepared != nullptr ? (uint32_t)kProjABytes : 1024u;
        // descriptors built once per unit; an operand at byte offset x is the
        // base plus x/16
        const uint64_t ad = smem_desc_sw128(a0, 16, a_sbo);
        const uint64_t bdd = smem_desc_sw128(b0, 16, 1024);
        for (int j = 0; j < kgroup; ++j) {
          const uint64_t aj = ad + (uint64_t)((j * a_jstride) >> 4);
          const uint64_t bj = bdd + (uint64_t)((j * n_tile * kProjKBlock * 2) >> 4);
#pragma unroll
          for (int k = 0; k < kProjKBlock / 16; ++k)  // 32 bytes of k per step inside the 128-byte rows
            mma_ss(tmem + acc * acc_cols, aj + (uint64_t)(k * 2), bj + (uint64_t)(k * 2), idesc,
                   (first && j == 0 && k == 0) ? 0u : 1u);
        }
        mma_commit(empty(st));
        if (last) {
          mma_commit(acc_full(acc));
          ++seg;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ drain
    // Thread (warp w, lane l) holds wo row 32w + l of the tile: one TMEM
    // column per batch row.  Partial slot 2c + seg is laid out [batch row of
    // the tile][128 wo rows]; a direct tile goes to delta in bf16.
    const int nl = warp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    for (int seg = 0; seg < n_seg; ++seg) {
      const int acc = seg & 1;
      const long long u_seg = (t0 + seg) * upt;
      const int row0 = unit_row0(u_seg);
      wait(acc_full(acc), (seg >> 1) & 1, ab);
      tc_fence_after();
      float* dst = partial + ((size_t)(2 * c + seg) * n_tile) * kProjM + nl;
      __nv_bfloat16* dd = delta + (size_t)row0 * dim + (size_t)unit_m(u_seg) * kProjM + nl;
      for (int j0 = 0; j0 < n_tile; j0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + acc * acc_cols + j0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (row0 + j0 + j >= B) continue;
          if (direct)
            dd[(size_t)(j0 + j) * dim] = __float2bfloat16_rn(__uint_as_float(v[j]));
          else
            dst[(size_t)(j0 + j) * kProjM] = __uint_as_float(v[j]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  // every CTA has issued its partial stores: the reduce kernel may launch
  // (it waits for this grid's completion before reading them)
  grid_dep_launch();
  if (warp == 5) tmem_dealloc(tmem, 2 * acc_cols);
}

// delta[b, 128 m + n] = bf16( sum over the CTAs c whose units cover the tile
// (y, m), in increasing c, of their partial for it ).  Grid (tiles, groups of
// kProjReduceRows rows of a tile); thread t sums row t / 32 of its group,
// wo rows 4 (t % 32) .. +3, with one independent 16-byte load per
// contributing CTA.  Only the split mode launches it: fewer tiles than SMs,
// so unit and CTA indices stay far below 2^31 and 32-bit arithmetic is exact.
constexpr int kProjReduceThreads = kProjReduceRows * 32;

__global__ void __launch_bounds__(kProjReduceThreads)
projection_reduce_kernel(const float* __restrict__ partial, __nv_bfloat16* __restrict__ delta, int B, int dim,
                         int n_tile, int n_ctas, int kgroup, int k_blocks) {
  const int t = blockIdx.x;
  const int m_tiles = dim / kProjM;
  const int m = t % m_tiles;
  const int row0 = (t / m_tiles) * n_tile;
  const int j = blockIdx.y * kProjReduceRows + (int)(threadIdx.x >> 5);  // row within the tile
  const int n4 = (int)(threadIdx.x & 31) * 4;
  const int upt = k_blocks / kgroup;  // units per tile
  const int U = m_tiles * ((B + n_tile - 1) / n_tile) * upt;
  int c_lo, c_hi;  // the CTAs holding the tile's units
  proj_tile_ctas<int>(t, upt, U, n_ctas, &c_lo, &c_hi);
  grid_dep_wait();  // the partials come from projection_kernel
  if (j >= n_tile || row0 + j >= B) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int cc = c_lo; cc <= c_hi; ++cc) {
    const int seg = proj_segment_of<int>(cc, t, upt, U, n_ctas);  // the tile is cc's first or second segment
    const float4 v = __ldg(reinterpret_cast<const float4*>(partial + ((size_t)(2 * cc + seg) * n_tile + j) * kProjM + n4));
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  uint2 packed;
  packed.x = pack_bf16x2(acc.x, acc.y);
  packed.y = pack_bf16x2(acc.z, acc.w);
  *reinterpret_cast<uint2*>(delta + (size_t)(row0 + j) * dim + (size_t)m * kProjM + n4) = packed;
}

}  // namespace mla

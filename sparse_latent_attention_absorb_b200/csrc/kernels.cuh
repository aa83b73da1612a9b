// sm_100a kernels of the sparse MLA decode step (DeepSeek-V3.2-Exp,
// model.py 590-606 as shown on the atlas pages "Query-key similarity",
// "Softmax" and "Apply value weights").
//
//   absorb_kernel            q_lat = q_nope . W_UK per head        (tcgen05)
//   sparse_attend_kernel     gathered scores, online softmax, mix  (tcgen05,
//                            2-CTA cluster, DSMEM score exchange)
//   combine_value_up_kernel  log-sum-exp merge of the key splits,
//                            then O~ . W_UV^T per head            (tcgen05)
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <cstring>

#include "ptx.cuh"

namespace mla {

constexpr int kH = MLA_HEADS;         // 128 heads
constexpr int kDn = MLA_D_NOPE;       // 128
constexpr int kDr = MLA_D_ROPE;       // 64
constexpr int kDl = MLA_D_LATENT;     // 512
constexpr int kDv = MLA_D_V;          // 128
constexpr int kHeadRows = kDn + kDv;  // rows of one head in wkv_b

// Dynamic shared memory is only guaranteed 16-byte alignment; 128B-swizzle
// atoms need 1024.  Every kernel requests kSmemAlignPad extra bytes and
// rounds its base up.
constexpr int kSmemAlignPad = 1024;
__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// =============================================================================
// absorb_kernel: q_lat[b,h,c] = sum_d q_nope[b,h,d] * W_UK[h,d,c]
//
// Swap-AB GEMM per (head h, 128-column chunk of c, tile of up to 128 rows b),
// over the n_heads heads of the call (128, or a tensor-parallel shard's):
//   D[c, b] = sum_d W_UK[h, d, c] * q_nope[b, h, d]
// M = 128 (c), N = batch tile (multiple of 16), K = 128 (d).
// A = W_UK[h][:, chunk] is M-major in memory (c contiguous): two TMA boxes of
// 64 c x 128 d, 128B-swizzled.  B = q_nope[:, h, :] is K-major: two 3-D TMA
// boxes of 64 d x N rows.  The accumulator lives in TMEM (lanes = c).
// =============================================================================
constexpr int kAbsorbNMax = 128;
constexpr int kAbsorbSmemA = 2 * 64 * 128 * 2;                      // 32 KB
// shared memory for a batch tile of n rows: W_UK chunk, q_nope tile, barriers
// (sized to the tile so that four CTAs fit on an SM when n <= 64)
__host__ __device__ constexpr int absorb_smem_bytes(int n) { return kAbsorbSmemA + 2 * n * 128 + 256 + kSmemAlignPad; }
constexpr int kAbsorbSmemBytes = absorb_smem_bytes(kAbsorbNMax);

// Whole-kernel stamps of the trace build (globaltimer ns; earliest start via
// atomicMin, latest end via atomicMax), reset by mla_trace_reset().
enum KernelEvent {
  kKeAbsorbStart = 0,  // min over CTAs
  kKeAbsorbEnd,        // max over CTAs
  kKeCombineStart,     // min over CTAs
  kKeCombineWaited,    // max over CTAs: past the wait on the attention kernel
  kKeCombineEnd,       // max over CTAs
  kKeCombineFirstWaited,  // min over CTAs: past the wait on the attention kernel
  kKeCombineIssued,    // max over CTAs: every k-block landed and its MMAs issued
  kKeCombineMmaDone,   // max over CTAs: accumulator complete
  kKeCombineWeights,   // max over CTAs: split weights ready (several splits)
  kKeCombineMerged,    // max over CTAs: merged operand in shared memory (several splits)
  kKernelEvents
};
#ifdef MLA_TRACE
__device__ unsigned long long g_mla_kernel_ns[kKernelEvents];
#define MLA_KERNEL_STAMP_MIN(ev) atomicMin(&g_mla_kernel_ns[(ev)], (unsigned long long)global_timer_ns())
#define MLA_KERNEL_STAMP_MAX(ev) atomicMax(&g_mla_kernel_ns[(ev)], (unsigned long long)global_timer_ns())
#else
#define MLA_KERNEL_STAMP_MIN(ev) \
  do {                           \
  } while (0)
#define MLA_KERNEL_STAMP_MAX(ev) \
  do {                           \
  } while (0)
#endif

__global__ void __launch_bounds__(128, 1)
absorb_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
              __nv_bfloat16* __restrict__ q_lat, int B, int n_tile, int n_heads, int* d_status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x;  // 128-wide chunk of the latent dimension
  const int h = blockIdx.y;
  const int b0 = blockIdx.z * kAbsorbNMax;

  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kAbsorbSmemA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAbsorbSmemA + 2 * n_tile * 128);
  const uint32_t bar_load = smem_u32(&bars[0]);
  const uint32_t bar_mma = smem_u32(&bars[1]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[2]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[3]);
  const AbortState ab{abort_flag, d_status};

  const uint32_t tmem_cols = n_tile <= 32 ? 32u : (n_tile <= 64 ? 64u : 128u);
  // The loads go out first (TMA needs no TMEM); TMEM is allocated meanwhile.
  if (tid == 0) {
    MLA_KERNEL_STAMP_MIN(kKeAbsorbStart);
    *abort_flag = 0;
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_arrive_expect_tx(bar_load, kAbsorbSmemA + 2 * n_tile * 128);
    const int wrow = h * kHeadRows;  // W_UK rows of head h
    tma_load_2d(sA, &tm_w, bar_load, chunk * 128, wrow);
    tma_load_2d(sA + 64 * 128 * 2, &tm_w, bar_load, chunk * 128 + 64, wrow);
    tma_load_3d(sB, &tm_q, bar_load, 0, h, b0);
    tma_load_3d(sB + n_tile * 128, &tm_q, bar_load, 64, h, b0);
    grid_dep_launch();  // the attention kernel may start gathering
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    wait(bar_load, 0, ab);
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, n_tile, /*a MN*/ true, /*b MN*/ false);
    // descriptors built once; an operand at byte offset x is the base plus x/16
    const uint64_t a0 = smem_desc_sw128(sA, 64 * 128 * 2, 1024);
    const uint64_t b0d = smem_desc_sw128(sB, 16, 1024);
#pragma unroll
    for (int k = 0; k < kDn / 16; ++k) {
      // A: 16 d-rows per step (two 8-row groups 1024 B apart); the two
      // 64-wide c blocks are 16 KB apart.  B: 32 bytes of d per step inside
      // the 128-byte row; the second 64-wide d block follows the first.
      mma_ss(tmem, a0 + (uint64_t)((k * 16 * 128) >> 4),
             b0d + (uint64_t)(((k >> 2) * n_tile * 128 + (k & 3) * 32) >> 4), idesc, k > 0 ? 1u : 0u);
    }
    mma_commit(bar_mma);
  }
  __syncwarp();

  // Epilogue: lane (32*warp + lane) holds column c of the chunk, one TMEM
  // column per batch row.
  wait(bar_mma, 0, ab);
  tc_fence_after();
  const int c = chunk * 128 + warp * 32 + lane;
  for (int n0 = 0; n0 < n_tile; n0 += 16) {
    uint32_t v[16];
    tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + n0, v);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int b = b0 + n0 + j;
      if (b < B) q_lat[((size_t)b * n_heads + h) * kDl + c] = __float2bfloat16_rn(__uint_as_float(v[j]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
  if (tid == 0) MLA_KERNEL_STAMP_MAX(kKeAbsorbEnd);
}

// =============================================================================
// sparse_attend_kernel
//
// One 2-CTA cluster per (batch row b, key split s).  CTA rank r owns latent
// columns [256r, 256r+256) and rotary columns [32r, 32r+32) of the score:
//   * its half of the absorbed query is the A operand of QK: the 256 latent
//     columns in TMEM (bf16 pairs; four tensor-map boxes staged in ring
//     stages 2-3, copied in by the softmax warps), the 32 rotary columns in
//     shared memory (one tensor-map box, already the K-major operand);
//   * for every selected position t of the split, a gather warp copies
//     kv[b,t,its 256] (128B-swizzled rows) and pe[b,t,its 32] (64B-swizzled
//     rows) into a ring of 64-position tiles (cp.async, 16 bytes per lane);
//     padding positions are zero-filled without a read;
//   * QK: S_r[h,t] = q_lat[h, its 256] . kv[t, its 256] + q_pe[h, its 32] .
//     pe[t, its 32]  -- a split-K half of the 576-wide score, M = 128 heads,
//     N = 64 positions, into a TMEM score buffer;
//   * two groups of four softmax warps take alternate tiles.  A thread owns
//     one head (TMEM lane) and all 64 positions of its group's tiles: it
//     reads its partial scores (which frees the one score buffer for the next
//     tile's QK), rounds them to fp16 in log2 units, pushes them into the peer
//     CTA's shared memory (st.async, completing on the peer's mbarrier),
//     adds the peer's half -- both CTAs add the same two fp16 values, so their
//     scores and everything after are bitwise identical -- masks, takes the
//     tile maximum, updates the running maximum lazily (O is rescaled only
//     when a row maximum grows by more than 2^8; the groups hand the running
//     maximum to each other tile by tile) and writes P (bf16) into its
//     group's TMEM buffer;
//   * PV: O_r[h, its 256] += P[h,t] . kv[t, its 256]  (A = P from TMEM,
//     B = the same gathered rows read M/N-major).
// The split's normalised O (bf16; with a single split per row, the final O~)
// and its log-sum-exp go to o_part / lse_part, O staged in the idle ring and
// written by one bulk copy per thread.
//
// Warp roles (448 threads): warps 0-3 softmax group 0 (even tiles), warps
// 4-7 softmax group 1 (odd tiles), warp w covering TMEM lanes 32(w%4)..;
// warp 10 TMEM allocation, the query's tensor-map loads and QK issue; warp 9
// PV issue; warps 8, 11, 12 and 13 gather (sixteen rows of every tile each).
// QK and PV are issued by different threads: their MMAs interleave in the
// tensor pipe, and a commit (which tracks the issuing thread's MMAs only)
// signals PV completion without waiting for a QK queued ahead of it.  Warp w
// runs on SM sub-partition w % 4, beside the two softmax warps of TMEM lane
// quarter w % 4.  The QK thread sits on sub-partition 2, beside no gather or
// PV warp: next to the quarter-0 softmax warps (as warp 8) it made them the
// last of their group to finish nearly every tile.
// =============================================================================
constexpr int kNt = 64;                            // positions per tile
constexpr int kStages = 4;                         // gathered tile ring
constexpr int kLatBlock = kNt * 128;               // one 64-column latent block of a tile (8 KB)
constexpr int kStageBytes = 4 * kLatBlock + kNt * 64;  // 4 latent blocks + the rotary block: 36 KB
constexpr int kQpeBytes = kH * 64;                 // rotary query columns of the half: 8 KB
constexpr int kQBoxBytes = kH * 128;               // one 64-column box of the latent query half: 16 KB
constexpr int kXHalves = (kNt / 8) * kH * 16;      // 16 KB: one exchanged score tile (fp16)
constexpr int kXBytes = kXHalves + kH * 4;         // + each row's fp32 offset
constexpr int kMslotBytes = 2 * kH * 4;            // running maximum published by each group
constexpr int kRedBytes = 4 * kH * 4;              // (row sum, maximum) of each group at the end
constexpr int kBarBytes = 512;
constexpr int kOffStage = 0;
constexpr int kOffX = kOffStage + kStages * kStageBytes;
constexpr int kOffQpe = kOffX + 2 * kXBytes;
constexpr int kOffMslot = kOffQpe + kQpeBytes;
constexpr int kOffRed = kOffMslot + kMslotBytes;
constexpr int kOffBar = kOffRed + kRedBytes;
constexpr int kAttendSmemBytes = kOffBar + kBarBytes + kSmemAlignPad;
constexpr int kSoftmaxWarps = 8;                   // two groups of four
constexpr int kMmaWarp = 10;    // TMEM allocation, QK issue (sub-partition 2)
constexpr int kPvWarp = 9;      // PV issue (sub-partition 1)
constexpr int kGatherWarps = 4;  // gather warp g fills rows 16g..16g+15 of every tile
// Gather warp index g of warp 8, 11, 12, 13 (sub-partitions 0, 3, 0, 1), or -1.
__device__ __forceinline__ int gather_index(int warp) {
  return warp == 8 ? 0 : (warp >= 11 && warp <= 13 ? warp - 10 : -1);
}
// PV(j) is issued after QK(j + kPvLag).  QK(j + kPvLag) needs the stage of
// tile j + kPvLag - kStages, freed by that tile's PV: it must come before
// PV(j), or PV(j) would wait for itself.  A lag of 3 keeps PV out of the QK
// it used to interleave with, but then the stage of tile j + 1 frees only
// after QK(j): the ring, not the score buffer, sets the pace.
constexpr int kPvLag = 2;
static_assert(kPvLag < kStages, "PV may not wait for a QK that needs its own stage");
// 14 warps: at most 128 registers a thread (the warps spread over the four
// SM sub-partitions, 16K registers each, two of which hold four warps).
constexpr int kAttendThreads = 32 * (kSoftmaxWarps + 2 + kGatherWarps);  // 448: warps 0..13
// TMEM columns
constexpr uint32_t kColS = 0;     // the score buffer (f32)
constexpr uint32_t kColP = 64;    // P buffer of group g at kColP + 32g (bf16 pairs)
constexpr uint32_t kColQ = 128;   // 128 columns: the latent query half (bf16 pairs)
constexpr uint32_t kColO = 256;   // 256 f32 columns of O
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kStageBytes % 1024 == 0 && kOffX % 1024 == 0 && kOffQpe % 1024 == 0 && kXBytes % 16 == 0,
              "swizzle atoms");
static_assert(kAttendSmemBytes <= 232448, "shared memory");
static_assert(kColS + kNt <= kColP && kColP + kNt <= kColQ && kColQ + 128 <= kColO, "TMEM map");
// Every gather warp copies its rows of every tile, in tile order: its wait
// on a stage's kv_empty before tile j is for PV(j - kStages), which cannot
// complete before this warp's own arrival for tile j - kStages, so successive
// waits on one barrier are exactly one phase apart (a parity test cannot tell
// phases two apart).  For the same reason a warp never arrives twice on one
// phase of kv_full.
static_assert(kGatherWarps * 16 == kNt, "sixteen rows of a tile per gather warp");
static_assert(kAttendThreads == 14 * 32 && kMmaWarp == 10 && kPvWarp == 9, "warp roles: 0-7 softmax, 9 PV, 10 QK, the rest gather");

struct AttendBars {
  uint64_t q_tma;               // the query boxes (TMA, transaction bytes) landed
  uint64_t q_full;              // softmax warps (8 arrivals) after storing Q
  uint64_t kv_full[kStages];    // every gather warp (4 arrivals) once its copies of the tile landed
  uint64_t kv_empty[kStages];   // MMA commit after PV of the tile
  uint64_t s_full[2];           // MMA commit after QK of a tile of group g: partial scores ready
  uint64_t s_empty;             // the tile's group (4 arrivals) after reading the partial scores
  uint64_t p_full[2];           // group g (4 arrivals) after writing P
  uint64_t p_free[2];           // MMA commit after PV of the tile: P buffer free, O stable
  uint64_t x_full[2];           // 1 local arrival + kXBytes of the peer group's st.async
  uint64_t x_free[2];           // 4 arrivals of the peer's group g once it has read our push
  uint64_t m_ready[2][4];       // group g, lane quarter q (1 arrival): running maximum published
  uint16_t vmask[kStages][4];   // valid positions of the tile in each stage (bit n%16 of part n/16)
  uint32_t tmem_addr;
  int abort_flag;
  int qk_issued;                // QK steps issued so far (written by the MMA thread)
};
static_assert(sizeof(AttendBars) <= kBarBytes, "barrier block");

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two floats to a pair of fp16 (round to nearest, saturated to +-65504 so a
// huge score cannot turn into inf - inf = NaN); `lo` goes to the low half.
__device__ __forceinline__ uint32_t pack_f16x2_sat(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t u) {
  __half2 h;
  memcpy(&h, &u, 4);
  return __half22float2(h);
}

// Optional pipeline trace (compile with -DMLA_TRACE): per-tile clock64()
// stamps of each pipeline event for the first cluster of a launch, read back
// with mla_trace_fetch().  Compiled out by default.
enum TraceEvent {
  kTrGatherIssue = 0,  // gather warp: copies of the tile issued
  kTrGatherLanded,     // gather warp: copies landed, tile published
  kTrQkStart,          // MMA thread: QK of the tile starts issuing
  kTrQkIssued,         // MMA thread: QK of the tile issued and committed
  kTrPvStart,          // MMA thread: PV of the tile starts issuing
  kTrPvIssued,         // MMA thread: PV of the tile issued and committed
  kTrSmStart,          // softmax (lane 0 of the group's first warp): partial scores available
  kTrSmPushed,         //   own half pushed to the peer
  kTrSmArrived,        //   peer's half observed
  kTrSmMax,            //   running maximum of the tile published
  kTrPWritten,         //   P written, p_full arrived
  kTrSmConverted,      //   own half read, reduced and rounded
  kTrSmFreeOk,         //   peer buffer free
  kTrSmSummed,         //   full scores and tile maximum formed
  kTrSmReleased,       //   peer told that its push has been read
  kTrSmMaxIn,          //   other group's running maximum received
  kTrGatherWoke,       // gather warp: its stage's previous tile released (wait returned)
  kTrSRead0,           // softmax warp of lane quarter q (kTrSRead0 + q): scores read, s_empty arrived
  kTrSRead1,
  kTrSRead2,
  kTrSRead3,
  kTrPFull0,           // softmax warp of lane quarter q (kTrPFull0 + q): P written, p_full arrived
  kTrPFull1,
  kTrPFull2,
  kTrPFull3,
  kTrQkKv,             // MMA thread: the tile's rows have landed (wait returned)
  kTrQkWoke,           // MMA thread: score buffer free (wait returned)
  kTrEvents
};
constexpr int kTraceTiles = 512;
// Per-cluster milestones of the trace build (globaltimer ns, CTA rank 0 of
// every cluster), read back with mla_trace_cluster_fetch().
enum ClusterEvent {
  kCeStart = 0,    // barriers and TMEM ready (after the cluster barrier)
  kCeQuery,        // MMA thread: query half in TMEM
  kCeFirstTile,    // MMA thread: first tile's rows landed
  kCeLastQk,       // MMA thread: last QK issued
  kCeLastPv,       // PV thread: last PV issued
  kCePvDone,       // softmax: last PV complete (epilogue may read O)
  kCeEnd,          // every thread past the epilogue
  kCeClocks,       // SM clock cycles from kCeStart to kCeEnd (clock64)
  kCeDepWaited,    // softmax: past the wait on the absorption kernel
  kCeQueryLoaded,  // softmax: first part of the query half in registers
  kCeFirstIssued,  // gather warp 0: first tile's copies issued
  kCeEntry,        // thread 0 at kernel entry
  kCeEpLoaded,     // thread 0: end_pos of the row loaded
  kCeIdxLoaded,    // gather warp 0: its first index word loaded
  kClusterEvents
};
constexpr int kTraceClusters = 4096;
#ifdef MLA_TRACE
__device__ long long g_mla_trace[2 * kTrEvents * kTraceTiles];
__device__ unsigned long long g_mla_cluster_ns[kClusterEvents * kTraceClusters];
#define MLA_TRACE_STAMP(ev, tile)                                                               \
  do {                                                                                           \
    if ((blockIdx.x >> 1) == 0 && (tile) < kTraceTiles)                                          \
      g_mla_trace[(rank * kTrEvents + (ev)) * kTraceTiles + (tile)] = clock64();                 \
  } while (0)
#define MLA_CLUSTER_STAMP(ev)                                                                    \
  do {                                                                                           \
    if (rank == 0 && unit < kTraceClusters) g_mla_cluster_ns[unit * kClusterEvents + (ev)] = global_timer_ns(); \
  } while (0)
#else
#define MLA_TRACE_STAMP(ev, tile) \
  do {                            \
  } while (0)
#define MLA_CLUSTER_STAMP(ev) \
  do {                        \
  } while (0)
#endif

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttendThreads, 1)
sparse_attend_kernel(const __grid_constant__ CUtensorMap tm_qlat, const __grid_constant__ CUtensorMap tm_qpe,
                     const __nv_bfloat16* __restrict__ kv_cache, const __nv_bfloat16* __restrict__ pe_cache,
                     const int32_t* __restrict__ end_pos, const int32_t* __restrict__ topk_idx, float scale,
                     void* __restrict__ o_part, float* __restrict__ lse_part, int K, int S_max, int n_split,
                     int span, const __nv_bfloat16* __restrict__ w_next, const int32_t* __restrict__ cache_slot,
                     int n_slots, int n_heads, int* d_status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int unit = blockIdx.x >> 1;
  const int b = unit / n_split;
  const int split = unit % n_split;
  const int k_begin = split * span;
  const int k_end = min(K, k_begin + span);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + kNt - 1) / kNt : 0;
#ifdef MLA_TRACE
  if (tid == 0) MLA_CLUSTER_STAMP(kCeEntry);
#endif
  int ep = end_pos[b];
  ep = ep < 0 ? 0 : (ep > S_max ? S_max : ep);
#ifdef MLA_TRACE
  if (tid == 0 && ep >= 0) MLA_CLUSTER_STAMP(kCeEpLoaded);
#endif
  // Cache slot of row b: b itself (decode), or cache_slot[b] when rows are
  // query positions sharing a sequence's latents (prefill).  A slot outside
  // [0, n_slots) leaves the row with no valid position (nothing is read).
  int slot = b;
  if (cache_slot != nullptr) {
    slot = cache_slot[b];
    if (slot < 0 || slot >= n_slots) {
      slot = 0;
      ep = 0;
    }
  }
  const int32_t* idx_row = topk_idx + (size_t)b * K;

  const uint32_t sStage = smem_u32(smem + kOffStage);
  const uint32_t sX = smem_u32(smem + kOffX);
  const uint32_t sQpe = smem_u32(smem + kOffQpe);
  float* mslot = reinterpret_cast<float*>(smem + kOffMslot);  // [group][head]
  float* red = reinterpret_cast<float*>(smem + kOffRed);      // [l | m][group][head]
  AttendBars* bars = reinterpret_cast<AttendBars*>(smem + kOffBar);
  const AbortState ab{&bars->abort_flag, d_status};
  const float c2 = scale * 1.4426950408889634f;  // scores to log2 units

  if (tid == 0) {
    bars->abort_flag = 0;
    bars->qk_issued = 0;
    mbar_init(smem_u32(&bars->q_tma), 1);
    mbar_init(smem_u32(&bars->q_full), kSoftmaxWarps);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars->kv_full[i]), kGatherWarps);
      mbar_init(smem_u32(&bars->kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->p_full[i]), 4);
      mbar_init(smem_u32(&bars->p_free[i]), 1);
      mbar_init(smem_u32(&bars->x_full[i]), 1);
      mbar_arrive_expect_tx(smem_u32(&bars->x_full[i]), kXBytes);  // armed for the group's first tile
      mbar_init(smem_u32(&bars->x_free[i]), 4);
      for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&bars->m_ready[i][q]), 1);
    }
    mbar_init(smem_u32(&bars->s_empty), 4);
    fence_mbarrier_init_cluster();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&bars->tmem_addr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote access
  tc_fence_after();
  const uint32_t tmem = bars->tmem_addr;
  grid_dep_launch();  // the combine kernel may start loading its weights
#ifdef MLA_TRACE
  const long long clk_start = clock64();
  if (tid == 0) MLA_CLUSTER_STAMP(kCeStart);
#endif

  if (gather_index(warp) >= 0) {
    // ------------------------------------------------------------ gather
    // All four gather warps fill every tile: warp g copies rows
    // [16g, 16g + 16) of it (latent: one row per instruction, 32 lanes x 16
    // bytes = this CTA's 256 columns; rotary: eight rows per instruction, this
    // CTA's 32 columns), so a freed stage is refilled by four warps at once.
    // A tile is published (kv_full, one arrival per warp) once every warp's
    // copies have landed.  Each warp visits the stages in tile order, so its
    // successive waits on one stage's kv_empty are exactly one phase apart.
    const int g = gather_index(warp);
    const int row0 = 16 * g;
    const __nv_bfloat16* kv_row0 = kv_cache + (size_t)slot * S_max * kDl + rank * 256;
    const __nv_bfloat16* pe_row0 = pe_cache + (size_t)slot * S_max * kDr + rank * 32;
    // Index of row 16g + (lane % 16) of tile 2p + lane / 16 (a pair of tiles
    // per register), or -1 for a padding or out-of-range slot.
    auto load_pair = [&](int pr) -> int {
      const int t = 2 * pr + (lane >> 4);
      int v = -1;
      if (t < n_tiles) {
        const int k = k_begin + t * kNt + row0 + (lane & 15);
        if (k < k_end) v = __ldg(idx_row + k);
      }
      return (v >= 0 && v < ep) ? v : -1;
    };
    // tile j = 2p + h of the pair register `idx` (its rows in lanes 16h..16h+15)
    auto gather_tile = [&](int j, int idx, int h) {
      const int st = j % kStages;
      if (j >= kStages) wait(smem_u32(&bars->kv_empty[st]), ((j / kStages) - 1) & 1, ab);
      // stages 2 and 3 first hold the query's boxes, until it is in TMEM
      if (j == 2) wait(smem_u32(&bars->q_full), 0, ab);
      if (lane == 0) MLA_TRACE_STAMP(kTrGatherWoke, j);
      const uint32_t stage = sStage + st * kStageBytes;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const int pos = __shfl_sync(0xffffffffu, idx, 16 * h + n);
        const size_t p = pos >= 0 ? (size_t)pos : 0;
        const uint32_t dst = stage + (lane >> 3) * kLatBlock + sw128_offset(row0 + n, lane & 7);
        cp_async_16(dst, kv_row0 + p * kDl + lane * 8, pos >= 0 ? 16u : 0u);
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int n = q * 8 + (lane >> 2), c = lane & 3;
        const int pos = __shfl_sync(0xffffffffu, idx, 16 * h + n);
        const size_t p = pos >= 0 ? (size_t)pos : 0;
        const uint32_t dst = stage + 4 * kLatBlock + sw64_offset(row0 + n, c);
        cp_async_16(dst, pe_row0 + p * kDr + c * 8, pos >= 0 ? 16u : 0u);
      }
      cp_async_commit();
      if (lane == 0) MLA_TRACE_STAMP(kTrGatherIssue, j);
      if (j == 0 && g == 0 && lane == 0) MLA_CLUSTER_STAMP(kCeFirstIssued);
      const uint32_t valid = (__ballot_sync(0xffffffffu, idx >= 0) >> (16 * h)) & 0xffffu;
      cp_async_wait_all();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        bars->vmask[st][g] = (uint16_t)valid;  // published by the arrival below
        mbar_arrive(smem_u32(&bars->kv_full[st]));
        MLA_TRACE_STAMP(kTrGatherLanded, j);
      }
    };
    // This warp's rows of tile j are pulled into L2 four tiles ahead of their
    // copies (lanes 16h..16h+15 of the pair register hold them).
    auto prefetch_tile = [&](int idx, int h) {
      const int pos = __shfl_sync(0xffffffffu, idx, 16 * h + (lane & 15));
      if (pos >= 0) {
        const char* r = reinterpret_cast<const char*>(kv_row0 + (size_t)pos * kDl) + (lane >> 4) * 256;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(r));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(r + 128));
        if (lane < 16) asm volatile("prefetch.global.L2 [%0];" ::"l"(pe_row0 + (size_t)pos * kDr));
      }
    };
    // index registers: tiles (2p, 2p+1), (2p+2, 2p+3), (2p+4, 2p+5); each is
    // loaded a pair ahead of its first use (a register copy of a pending load
    // would wait for the load)
    int cur = load_pair(0), nxt = load_pair(1), pf = load_pair(2);
#ifdef MLA_TRACE
    if (g == 0 && lane == 0 && cur != -2) MLA_CLUSTER_STAMP(kCeIdxLoaded);
#endif
    for (int pr = 0; 2 * pr < n_tiles; ++pr) {
      gather_tile(2 * pr, cur, 0);
      prefetch_tile(pf, 0);
      if (2 * pr + 1 < n_tiles) {
        gather_tile(2 * pr + 1, cur, 1);
        prefetch_tile(pf, 1);
      }
      cur = nxt;
      nxt = pf;
      pf = load_pair(pr + 3);
    }
    // With its last tile gathered (a few tiles before this CTA ends), gather
    // warp 0 pulls W_UV of head blockIdx.x into L2 for the value-up kernel
    // that follows (w_next = wkv_b, or null to skip).  One head at most: with
    // fewer CTAs than heads the SMs left idle already run the value-up
    // kernel's CTAs, which load W_UV themselves, and more prefetches per CTA
    // only held up this CTA's exit (each bulk prefetch is issued in order).
    if (g == 0 && lane == 0 && w_next != nullptr && (int)blockIdx.x < n_heads) {
      const __nv_bfloat16* w = w_next + (size_t)(blockIdx.x * kHeadRows + kDn) * kDl;  // 128 rows x 512: 128 KB
#pragma unroll
      for (int part = 0; part < 4; ++part) prefetch_l2(w + part * 32 * kDl, 32 * kDl * 2);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ QK issue
    // First the query: this CTA's latent half (four 64-column boxes of all
    // 128 head rows, 128-byte swizzle) into ring stages 2 and 3, which the
    // softmax warps copy into TMEM, and its 32 rotary columns straight into
    // their K-major operand (64-byte swizzle).  Rows past the call's heads
    // lie outside the tensor maps and arrive as zeros.
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_qlat);
      tma_prefetch_desc(&tm_qpe);
      grid_dep_wait();  // q_lat comes from the absorption kernel
      if (tid == kMmaWarp * 32) MLA_CLUSTER_STAMP(kCeDepWaited);
      mbar_arrive_expect_tx(smem_u32(&bars->q_tma), 4 * kQBoxBytes + kQpeBytes);
#pragma unroll
      for (int bx = 0; bx < 4; ++bx)
        tma_load_3d(sStage + (2 + bx / 2) * kStageBytes + (bx % 2) * kQBoxBytes, &tm_qlat,
                    smem_u32(&bars->q_tma), (int)rank * 256 + bx * 64, 0, b);
      tma_load_3d(sQpe, &tm_qpe, smem_u32(&bars->q_tma), (int)rank * 32, 0, b);
    }
    // QK(j) as soon as its rows have landed and the previous tile's scores
    // have been read (one score buffer).
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kNt, false, false);
      // Descriptors are built once; an operand at byte offset x from a base
      // is the base descriptor plus x/16 (start-address field).
      const uint64_t d_lat = smem_desc_sw128(sStage, 16, 1024);            // QK B, latent, K-major
      const uint64_t d_pe = smem_desc_sw64(sStage + 4 * kLatBlock, 512);    // QK B, rotary, K-major
      const uint64_t d_qpe = smem_desc_sw64(sQpe, 512);                     // QK A, rotary, K-major
      wait(smem_u32(&bars->q_full), 0, ab);
      MLA_CLUSTER_STAMP(kCeQuery);
      for (int qk = 0, st = 0; qk < n_tiles; ++qk, st = (st + 1 == kStages) ? 0 : st + 1) {
        wait(smem_u32(&bars->kv_full[st]), (qk / kStages) & 1, ab);
        if (qk == 0) MLA_CLUSTER_STAMP(kCeFirstTile);
        MLA_TRACE_STAMP(kTrQkKv, qk);
        if (qk > 0) wait(smem_u32(&bars->s_empty), (qk - 1) & 1, ab);
        MLA_TRACE_STAMP(kTrQkWoke, qk);
        tc_fence_after();
        MLA_TRACE_STAMP(kTrQkStart, qk);
        const uint64_t dl = d_lat + (uint64_t)((st * kStageBytes) >> 4);
        const uint64_t dr = d_pe + (uint64_t)((st * kStageBytes) >> 4);
        const uint32_t dst = tmem + kColS;
#pragma unroll
        for (int k = 0; k < 16; ++k)  // latent: A from TMEM
          mma_ts(dst, tmem + kColQ + k * 8, dl + (uint64_t)(((k >> 2) * kLatBlock + (k & 3) * 32) >> 4), idesc_qk,
                 k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < 2; ++k)  // rotary: 32 bytes per step inside the 64-byte rows
          mma_ss(dst, d_qpe + (uint64_t)((k * 32) >> 4), dr + (uint64_t)((k * 32) >> 4), idesc_qk, 1u);
        mma_commit(smem_u32(&bars->s_full[qk & 1]));
        *reinterpret_cast<volatile int*>(&bars->qk_issued) = qk + 1;
        MLA_TRACE_STAMP(kTrQkIssued, qk);
      }
      MLA_CLUSTER_STAMP(kCeLastQk);
    }
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ PV issue
    // PV(j) as soon as its P is written; its commits free the stage and the
    // P buffer and mark O stable.
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
      const uint64_t d_v = smem_desc_sw128(sStage, kLatBlock, 1024);  // PV B, latent, N-major
      for (int pv = 0, st = 0; pv < n_tiles; ++pv, st = (st + 1 == kStages) ? 0 : st + 1) {
        wait(smem_u32(&bars->p_full[pv & 1]), (pv >> 1) & 1, ab);
        // The score buffer's loop (QK -> softmax reads S -> next QK) sets the
        // pace, and the tensor pipe runs MMAs in issue order: PV(pv) enters
        // it only once QK(pv + kPvLag) has been issued, behind that QK.
        wait_counter(&bars->qk_issued, min(pv + kPvLag + 1, n_tiles), ab);
        tc_fence_after();
        MLA_TRACE_STAMP(kTrPvStart, pv);
        const uint64_t dv = d_v + (uint64_t)((st * kStageBytes) >> 4);
        const uint32_t pa = tmem + kColP + (pv & 1) * (kNt / 2);
#pragma unroll
        for (int k = 0; k < kNt / 16; ++k)  // 16 positions per step
          mma_ts(tmem + kColO, pa + k * 8, dv + (uint64_t)((k * 16 * 128) >> 4), idesc_pv,
                 (pv > 0 || k > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bars->kv_empty[st]));
        mma_commit(smem_u32(&bars->p_free[pv & 1]));
        MLA_TRACE_STAMP(kTrPvIssued, pv);
      }
      MLA_CLUSTER_STAMP(kCeLastPv);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int grp = warp >> 2;      // tiles grp, grp+2, ...
    const int qd = warp & 3;        // TMEM lane quarter
    const int i = qd * 32 + lane;   // head (TMEM lane)
    const bool live = i < n_heads;  // lanes past the call's heads hold a zero query and write nothing
    const bool leader = (qd == 0 && lane == 0);
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;

    // This CTA's half of the query: latent columns 0..127 (group 0) and
    // 128..255 (group 1) from their staged boxes into TMEM (the rotary part
    // is already in place); with no tile to process nothing is needed.
    {
      if (n_tiles > 0) {
        wait(smem_u32(&bars->q_tma), 0, ab);
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // box 2 grp + part: 64 latent values = 32 columns
          const uint32_t row = sStage + (2 + grp) * kStageBytes + part * kQBoxBytes + (uint32_t)i * 128u;
          uint32_t r[32];
#pragma unroll
          for (int v = 0; v < 8; ++v)
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(r[4 * v]), "=r"(r[4 * v + 1]), "=r"(r[4 * v + 2]), "=r"(r[4 * v + 3])
                         : "r"(row + (uint32_t)((v ^ (i & 7)) << 4))
                         : "memory");
          tmem_st32(tmem + lane_base + kColQ + (2 * grp + part) * 32, r);
          if (part == 0 && leader && grp == 0) MLA_CLUSTER_STAMP(kCeQueryLoaded);
        }
        tmem_wait_st();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->q_full));
    }

    const uint32_t sbuf = tmem + lane_base + kColS;
    const uint32_t pbuf = tmem + lane_base + kColP + grp * (kNt / 2);
    const uint32_t x_mine = sX + grp * kXBytes;              // the peer's half arrives here
    const uint32_t x_peer = cluster_map(x_mine, peer);       // our half goes there
    const uint32_t xfull_peer = cluster_map(smem_u32(&bars->x_full[grp]), peer);
    const uint32_t xfree_peer = cluster_map(smem_u32(&bars->x_free[grp]), peer);
    float m_cur = -INFINITY;  // running maximum as of this group's last tile (log2 units)
    float l_part = 0.f;       // this group's share of the row sum, relative to m_cur

    int it = 0;  // this group's tile counter: tile j = 2 it + grp
    for (int j = grp; j < n_tiles; j += 2, ++it) {
      // partial scores of tile j: read, release the buffer
      wait(smem_u32(&bars->s_full[grp]), it & 1, ab);
      tc_fence_after();
      if (leader) MLA_TRACE_STAMP(kTrSmStart, j);
      // valid positions of tile j (the stage cannot be refilled before PV(j))
      const int st = j % kStages;
      wait(smem_u32(&bars->kv_full[st]), (j / kStages) & 1, ab);
      // parts 0,1 and 2,3 read as two words: bit n of word n/32
      const uint32_t vm0 = *reinterpret_cast<volatile uint32_t*>(&bars->vmask[st][0]);
      const uint32_t vm1 = *reinterpret_cast<volatile uint32_t*>(&bars->vmask[st][2]);
      // Our half in log2 units, as fp16 relative to its own maximum over the
      // tile (sent exactly, in fp32, beside it): the rounding then scales with
      // the spread of the scores inside the tile, not with their size.
      // Padding positions become -inf, which the peer's sum carries along.
      uint32_t hv[32];
      float off;
      {
        uint32_t sv[64];
        tmem_ld32(sbuf, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(sbuf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&bars->s_empty));
          MLA_TRACE_STAMP(kTrSRead0 + qd, j);
        }
        // eight independent partial maxima (a 64-deep chain would be latency)
        float om8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) om8[u] = __uint_as_float(sv[u]);
#pragma unroll
        for (int t = 8; t < 64; ++t) om8[t & 7] = fmaxf(om8[t & 7], __uint_as_float(sv[t]));
        const float om = fmaxf(fmaxf(fmaxf(om8[0], om8[1]), fmaxf(om8[2], om8[3])),
                               fmaxf(fmaxf(om8[4], om8[5]), fmaxf(om8[6], om8[7])));
        off = om * c2;  // c2 > 0: the maximum of the scaled values
#pragma unroll
        for (int t = 0; t < 32; ++t)
          hv[t] = pack_f16x2_sat(fmaf(__uint_as_float(sv[2 * t]), c2, -off),
                                 fmaf(__uint_as_float(sv[2 * t + 1]), c2, -off));
      }
      if ((vm0 & vm1) != 0xffffffffu) {  // a tile with padding (the tail of a split)
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const uint32_t w = (t < 16) ? vm0 : vm1;
          const uint32_t keep = (((w >> ((2 * t) & 31)) & 1u) ? 0x0000ffffu : 0u) |
                                (((w >> ((2 * t + 1) & 31)) & 1u) ? 0xffff0000u : 0u);
          hv[t] = (hv[t] & keep) | (0xfc00fc00u & ~keep);  // fp16 -inf where masked
        }
      }
      // push our half into the peer's buffer (free once the peer has read our
      // previous push from it)
      if (leader) MLA_TRACE_STAMP(kTrSmConverted, j);
      if (it > 0) wait_cluster(smem_u32(&bars->x_free[grp]), (it - 1) & 1, ab);
      if (leader) MLA_TRACE_STAMP(kTrSmFreeOk, j);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        st_async_v4(x_peer + (uint32_t)((q * kH + i) * 16), hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3],
                    xfull_peer);
      st_async_b32(x_peer + (uint32_t)(kXHalves + i * 4), __float_as_uint(off), xfull_peer);
      if (leader) MLA_TRACE_STAMP(kTrSmPushed, j);

      // The peer's half.  Scores relative to base = off + off_peer, summed
      // as fp16 pairs: both CTAs add the same two values (addition commutes),
      // so their scores and everything after them are bitwise identical.
      wait(smem_u32(&bars->x_full[grp]), it & 1, ab);
      if (qd == 0 && lane == 0) {
        MLA_TRACE_STAMP(kTrSmArrived, j);
        mbar_arrive_expect_tx(smem_u32(&bars->x_full[grp]), kXBytes);  // re-arm for tile j + 2
      }
      float off_peer;
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(off_peer) : "r"(x_mine + (uint32_t)(kXHalves + i * 4)) : "memory");
      const float base = off + off_peer;
      uint32_t sh[32];
      __half2 hmx4[4];  // four independent partial maxima
#pragma unroll
      for (int e = 0; e < 4; ++e) hmx4[e] = __halves2half2(__ushort_as_half(0xfc00u), __ushort_as_half(0xfc00u));
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t o[4];
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
                     : "r"(x_mine + (uint32_t)((q * kH + i) * 16))
                     : "memory");
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __half2 a, p2;
          memcpy(&a, &hv[4 * q + e], 4);
          memcpy(&p2, &o[e], 4);
          const __half2 sum = __hadd2(a, p2);
          hmx4[e] = __hmax2(hmx4[e], sum);
          memcpy(&sh[4 * q + e], &sum, 4);
        }
      }
      const float2 hm = __half22float2(__hmax2(__hmax2(hmx4[0], hmx4[1]), __hmax2(hmx4[2], hmx4[3])));
      const float mx = fmaxf(hm.x, hm.y) + base;  // the tile maximum (-inf if all masked)
      if (leader) MLA_TRACE_STAMP(kTrSmSummed, j);
      // Every lane has consumed its loads of the peer's push (the sums above
      // use them), so the peer may overwrite the buffer with tile j + 2.  A
      // relaxed arrival: a release here would wait for our own pushes in
      // flight to the peer.
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(xfree_peer);
      if (leader) MLA_TRACE_STAMP(kTrSmReleased, j);

      // Running maximum.  It moves only when a tile's maximum exceeds it by
      // more than 2^8 (so p <= 256 otherwise).  The other group hands over
      // its value after tile j-1; this group's row sum is brought to it.
      float m_prev = -INFINITY;
      if (j > 0) {
        wait(smem_u32(&bars->m_ready[grp ^ 1][qd]), ((j - 1) >> 1) & 1, ab);
        m_prev = mslot[(grp ^ 1) * kH + i];
      }
      if (leader) MLA_TRACE_STAMP(kTrSmMaxIn, j);
      if (m_prev != m_cur) {
        l_part = (m_cur == -INFINITY) ? 0.f : l_part * ex2_approx(m_cur - m_prev);
        m_cur = m_prev;
      }
      const bool grow = mx > m_cur + kRescaleThreshold;
      const float alpha = grow ? ((m_cur == -INFINITY) ? 0.f : ex2_approx(m_cur - mx)) : 1.f;
      if (grow) m_cur = mx;
      mslot[grp * kH + i] = m_cur;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->m_ready[grp][qd]));
      if (leader) MLA_TRACE_STAMP(kTrSmMax, j);

      // The TMEM accesses are warp-collective, so the whole warp rescales
      // when any of its rows must; rows that keep their maximum use alpha = 1.
      if (__any_sync(0xffffffffu, grow) && j > 0) {
        // PV(j-1) (and so every earlier MMA) must have finished before O is
        // rescaled in place; PV(j) waits for this group's P.
        wait(smem_u32(&bars->p_free[(j - 1) & 1]), ((j - 1) >> 1) & 1, ab);
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 16; ++cc) {
          const uint32_t col = kColO + cc * 16;
          uint32_t ov[16];
          tmem_ld16(tmem + lane_base + col, ov);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t) ov[t] = __float_as_uint(__uint_as_float(ov[t]) * alpha);
          tmem_st16(tmem + lane_base + col, ov);
        }
        tmem_wait_st();
      }
      l_part *= alpha;

      // Masked positions hold -inf and give exp2(-inf) = 0.  While a row has
      // seen no valid position its maximum is still -inf; subtracting 0 then
      // keeps every masked term at exactly 0 instead of exp2(NaN).
      const float m_sub = (m_cur == -INFINITY) ? 0.f : m_cur;
      const float csub = m_sub - base;  // s - m_sub = s_rel - csub
      // this group's P buffer was last read by PV(j-2)
      if (it > 0) wait(smem_u32(&bars->p_free[grp]), (it - 1) & 1, ab);
      tc_fence_after();
      float lt4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent partial sums
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float2 f = unpack_f16x2(sh[16 * hh + t]);
          const float p0 = ex2_approx(f.x - csub);
          const float p1 = ex2_approx(f.y - csub);
          pk[t] = pack_bf16x2(p0, p1);
          lt4[t & 3] += p0 + p1;
        }
        tmem_st16(pbuf + 16 * hh, pk);
      }
      l_part += (lt4[0] + lt4[1]) + (lt4[2] + lt4[3]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bars->p_full[grp]));
        MLA_TRACE_STAMP(kTrPFull0 + qd, j);
      }
      if (leader) MLA_TRACE_STAMP(kTrPWritten, j);
    }

    // epilogue: both groups' row sums brought to the final maximum (the
    // larger of the two: the maximum never decreases), normalised O half and
    // the split's log-sum-exp
    red[grp * kH + i] = l_part;
    red[(2 + grp) * kH + i] = m_cur;
    named_bar_sync(1 + qd, 64);  // warps qd and qd + 4
    const float l_o = red[(grp ^ 1) * kH + i];
    const float m_o = red[(2 + (grp ^ 1)) * kH + i];
    const float m_fin = fmaxf(m_cur, m_o);
    const float l_a = (m_cur == -INFINITY) ? 0.f : l_part * ex2_approx(m_cur - m_fin);
    const float l_b = (m_o == -INFINITY) ? 0.f : l_o * ex2_approx(m_o - m_fin);
    const float l_sum = l_a + l_b;  // the same sum in both groups (fp32 addition commutes)
    if (n_tiles > 0) {
      // the last PV done implies every MMA of the split is done
      wait(smem_u32(&bars->p_free[(n_tiles - 1) & 1]), ((n_tiles - 1) >> 1) & 1, ab);
      tc_fence_after();
      if (leader && grp == 0) MLA_CLUSTER_STAMP(kCePvDone);
    }
    const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
    // The split's normalised mix goes out in bf16: with one split per row it
    // is the mixed latent O~ itself (the value-up operand); with several the
    // value-up kernel merges the splits by their log-sum-exp weights.
    // The ring is idle once the last PV is done, so each thread stages its
    // 128-column half row there (rows padded by 16 bytes: the 32 rows of a
    // warp fall on distinct banks) and writes it out with one bulk copy.
    const size_t orow = (((size_t)b * n_split + split) * n_heads + (live ? i : 0)) * kDl + rank * 256 + 128 * grp;
    constexpr uint32_t row_bytes = 128u * 2u;
    const uint32_t stg = sStage + (uint32_t)(grp * kH + i) * (row_bytes + 16u);
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t ov[32];
      if (n_tiles > 0) {
        tmem_ld32(tmem + lane_base + kColO + 128 * grp + cc * 32, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) ov[t] = 0u;
      }
#pragma unroll
      for (int t = 0; t < 32; t += 8)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg + (uint32_t)(cc * 64 + t * 2)),
                     "r"(pack_bf16x2(__uint_as_float(ov[t]) * inv, __uint_as_float(ov[t + 1]) * inv)),
                     "r"(pack_bf16x2(__uint_as_float(ov[t + 2]) * inv, __uint_as_float(ov[t + 3]) * inv)),
                     "r"(pack_bf16x2(__uint_as_float(ov[t + 4]) * inv, __uint_as_float(ov[t + 5]) * inv)),
                     "r"(pack_bf16x2(__uint_as_float(ov[t + 6]) * inv, __uint_as_float(ov[t + 7]) * inv))
                     : "memory");
    }
    if (live) {
      fence_proxy_async_smem();  // the staged row, visible to the bulk copy
      uint8_t* dst = static_cast<uint8_t*>(o_part) + orow * 2;
      bulk_store(dst, stg, row_bytes);
      bulk_commit();
      bulk_wait_read();
    }
    if (rank == 0 && grp == 0 && live) {
      lse_part[((size_t)b * n_split + split) * n_heads + i] =
          l_sum > 0.f ? (m_fin + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
    }
  }

  // teardown: all TMEM traffic done, then release TMEM; keep both CTAs alive
  // until neither can touch the other's shared memory any more.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
#ifdef MLA_TRACE
  if (tid == 0) {
    MLA_CLUSTER_STAMP(kCeEnd);
    if (rank == 0 && unit < kTraceClusters)
      g_mla_cluster_ns[unit * kClusterEvents + kCeClocks] = (unsigned long long)(clock64() - clk_start);
  }
#endif
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
  cluster_sync();
}
// =============================================================================
// combine_value_up_kernel
//
// Per (head h, tile of up to 64 rows b):
//   with several splits: coefficients a_s = exp(lse_s - L) with
//   L = log sum_s exp(lse_s); O~[b, :] = sum_s a_s o_part[b, s, h, :] (bf16
//   partials, summed in f32), rounded
//   to bf16 into shared memory (K-major B operand, 128B-swizzled);
//   with one split: O~ is already bf16 in memory and comes in by TMA;
//   D[e, b] = sum_c W_UV[h, e, c] * O~[b, c]   (M = 128 value dims, K = 512)
//   with W_UV[h] (128 KB) brought in by eight TMA boxes.
// W_UV is requested before the wait on the attention kernel (programmatic
// dependent launch), so the weight read overlaps the end of that kernel.
// =============================================================================
constexpr int kCombineNMax = 64;
constexpr int kCombineMaxSplits = 128;
constexpr int kCombineSmemA = 8 * 128 * 128;             // 128 KB
constexpr int kCombineSmemB = 8 * kCombineNMax * 128;    // 64 KB
constexpr int kCombineSmemCoef = kCombineNMax * kCombineMaxSplits * 4;  // 32 KB
constexpr int kCombineSmemBytes = kCombineSmemA + kCombineSmemB + kCombineSmemCoef + 128 + kSmemAlignPad;
constexpr int kCombineThreads = 256;
static_assert(kCombineSmemBytes <= 232448, "shared memory");

__global__ void __launch_bounds__(kCombineThreads, 1)
combine_value_up_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_o,
                        const void* __restrict__ o_part, const float* __restrict__ lse_part,
                        __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out, int B, int n_split, int n_tile,
                        int n_heads, int* d_status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * kCombineNMax;
  const int rows = min(kCombineNMax, B - b0);

  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kCombineSmemA;
  float* coef = reinterpret_cast<float*>(smem + kCombineSmemA + kCombineSmemB);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kCombineSmemA + kCombineSmemB + kCombineSmemCoef);
  // bar_k[kb]: W_UV box kb (and, with one split, O~ box kb) landed
  auto bar_k = [&](int kb) { return smem_u32(&bars[kb]); };
  const uint32_t bar_mma = smem_u32(&bars[8]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[9]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[10]);
  const AbortState ab{abort_flag, d_status};
  const uint32_t tmem_cols = n_tile <= 32 ? 32u : 64u;

  if (tid == 0) {
    MLA_KERNEL_STAMP_MIN(kKeCombineStart);
    *abort_flag = 0;
    for (int kb = 0; kb < 8; ++kb) mbar_init(bar_k(kb), 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    tma_prefetch_desc(&tm_w);
    const int wrow = h * kHeadRows + kDn;  // W_UV rows of head h
    for (int kb = 0; kb < 8; ++kb) {
      mbar_arrive_expect_tx(bar_k(kb), 128 * 128 + (n_split == 1 ? n_tile * 128 : 0));
      tma_load_2d(sA + kb * 128 * 128, &tm_w, bar_k(kb), kb * 64, wrow);
    }
  }
  grid_dep_launch();  // a programmatically dependent successor (the output projection) may start
  grid_dep_wait();    // o_part / lse_part come from the attention kernel
  if (tid == 0) {
    MLA_KERNEL_STAMP_MAX(kKeCombineWaited);
    MLA_KERNEL_STAMP_MIN(kKeCombineFirstWaited);
  }

  if (n_split == 1) {
    // O~ rows b0.. of head h: eight boxes of 64 columns x n_tile rows (rows
    // past B read as zero), each completing its k-block's barrier
    if (tid == 0) {
      tma_prefetch_desc(&tm_o);
      for (int kb = 0; kb < 8; ++kb) tma_load_3d(sB + kb * n_tile * 128, &tm_o, bar_k(kb), kb * 64, h, b0);
    }
    if (tid < rows && lse_out)
      lse_out[(size_t)(b0 + tid) * n_heads + h] = lse_part[(size_t)(b0 + tid) * n_heads + h];
  } else {
    // split weights, one row per thread
    if (tid < rows) {
      const int b = b0 + tid;
      float mx = -INFINITY;
      for (int s = 0; s < n_split; ++s) mx = fmaxf(mx, lse_part[((size_t)b * n_split + s) * n_heads + h]);
      float total = 0.f;
      for (int s = 0; s < n_split; ++s) {
        const float l = lse_part[((size_t)b * n_split + s) * n_heads + h];
        const float w = (mx == -INFINITY) ? 0.f : __expf(l - mx);
        coef[tid * kCombineMaxSplits + s] = w;
        total += w;
      }
      const float inv = total > 0.f ? 1.f / total : 0.f;
      for (int s = 0; s < n_split; ++s) coef[tid * kCombineMaxSplits + s] *= inv;
      if (lse_out) lse_out[(size_t)b * n_heads + h] = total > 0.f ? mx + __logf(total) : -INFINITY;
    }
    __syncthreads();
    if (tid == 0) MLA_KERNEL_STAMP_MAX(kKeCombineWeights);

    // merged O~ rows -> bf16 K-major operand (row n = batch row, 512
    // columns): each split's 8 columns are one 16-byte load, up to sixteen
    // splits in flight together
    const __nv_bfloat16* o_bf = static_cast<const __nv_bfloat16*>(o_part);
    const size_t split_stride = (size_t)n_heads * kDl;
    for (int it = tid; it < n_tile * 64; it += kCombineThreads) {
      const int n = it >> 6, q = it & 63;  // q: 8-column chunk of the 512
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (n < rows) {
        const float* cf = coef + n * kCombineMaxSplits;
        const __nv_bfloat16* src = o_bf + ((size_t)(b0 + n) * n_split * n_heads + h) * kDl + q * 8;
        for (int s0 = 0; s0 < n_split; s0 += 16) {
          uint4 x[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (s0 + u < n_split) x[u] = __ldg(reinterpret_cast<const uint4*>(src + (size_t)(s0 + u) * split_stride));
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            if (s0 + u < n_split) {
              const float a = cf[s0 + u];
              const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {  // bf16 -> f32 is exact: the high half of the word
                acc[2 * e] += a * __uint_as_float(w[e] << 16);
                acc[2 * e + 1] += a * __uint_as_float(w[e] & 0xffff0000u);
              }
            }
          }
        }
      }
      const uint32_t dst = sB + (q >> 3) * (n_tile * 128) + sw128_offset(n, q & 7);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pack_bf16x2(acc[0], acc[1])),
                   "r"(pack_bf16x2(acc[2], acc[3])), "r"(pack_bf16x2(acc[4], acc[5])),
                   "r"(pack_bf16x2(acc[6], acc[7]))
                   : "memory");
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (tid == 0 && n_split > 1) MLA_KERNEL_STAMP_MAX(kKeCombineMerged);

  if (tid == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, n_tile, false, false);
    // descriptors built once; an operand at byte offset x is the base plus x/16
    const uint64_t a0 = smem_desc_sw128(sA, 16, 1024);
    const uint64_t b0d = smem_desc_sw128(sB, 16, 1024);
    for (int kb = 0; kb < 8; ++kb) {  // each 64-column k-block as soon as it has landed
      wait(bar_k(kb), 0, ab);
      tc_fence_after();
      const uint64_t ak = a0 + (uint64_t)((kb * (128 * 128)) >> 4);
      const uint64_t bk = b0d + (uint64_t)((kb * (n_tile * 128)) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem, ak + (uint64_t)(kk * 2), bk + (uint64_t)(kk * 2), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
    }
    mma_commit(bar_mma);
    MLA_KERNEL_STAMP_MAX(kKeCombineIssued);
  }
  __syncwarp();

  if (warp < 4) {
    wait(bar_mma, 0, ab);
    tc_fence_after();
    if (tid == 0) MLA_KERNEL_STAMP_MAX(kKeCombineMmaDone);
    const int e = warp * 32 + lane;  // value dimension
    for (int n0 = 0; n0 < n_tile; n0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + n0, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n = n0 + j;
        if (n < rows) out[((size_t)(b0 + n) * n_heads + h) * kDv + e] = __float2bfloat16_rn(__uint_as_float(v[j]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
  if (tid == 0) MLA_KERNEL_STAMP_MAX(kKeCombineEnd);
}

}  // namespace mla

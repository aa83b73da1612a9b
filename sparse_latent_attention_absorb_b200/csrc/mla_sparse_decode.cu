// Host side of the sparse MLA decode C ABI (see include/mla_sparse_decode.h):
// argument validation, key-split planning, TMA tensor-map encoding and the
// launches of the three sm_100a kernels on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "dequant.cuh"
#include "index_check.cuh"
#include "kernels.cuh"
#include "mla_sparse_decode.h"
#include "projection.cuh"

namespace {

using namespace mla;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ceil_div(int a, int b) { return (a + b - 1) / b; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- device info

struct DeviceInfo {
  int sm_count = 0;
  bool sm100 = false;
  bool configured = false;
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];

int current_device(DeviceInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.configured) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MLA_ERR_CUDA;
    d.sm100 = (major == 10 && minor == 0);
    d.sm_count = sms;
    if (d.sm100) {
      if (cudaFuncSetAttribute(absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAbsorbSmemBytes) != cudaSuccess ||
          cudaFuncSetAttribute(sparse_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttendSmemBytes) != cudaSuccess ||
          cudaFuncSetAttribute(combine_value_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCombineSmemBytes) != cudaSuccess ||
          cudaFuncSetAttribute(projection_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, proj_smem_max()) != cudaSuccess ||
          cudaFuncSetAttribute(check_indices_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kCheckMaxWords * 4) != cudaSuccess)
        return MLA_ERR_CUDA;
    }
    d.configured = true;
  }
  *info = &d;
  return d.sm100 ? MLA_OK : MLA_ERR_UNSUPPORTED;
}

// SM count used for split planning; 148 (B200) when no device is visible, so
// that sizing queries also work on a host without a GPU.
int planning_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
    return sms;
  cudaGetLastError();
  return 148;
}

// ---------------------------------------------------------------- tensor maps

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encoder() {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_encode) return MLA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return MLA_ERR_CUDA;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return MLA_OK;
}

// wkv_b (or a shard of n_heads heads) as a 2-D bf16 tensor
// [n_heads*256 rows, 512 columns], boxes of 64 columns x 128 rows, 128-byte
// swizzle.
int encode_wkv_b(CUtensorMap* m, const void* wkv_b, int n_heads) {
  cuuint64_t dims[2] = {(cuuint64_t)kDl, (cuuint64_t)n_heads * kHeadRows};
  cuuint64_t strides[1] = {(cuuint64_t)kDl * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(wkv_b), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// q_nope as a 3-D bf16 tensor {d: 128, h: n_heads, b: B}, boxes of
// 64 d x 1 head x n_tile rows, 128-byte swizzle (rows past B read as zero).
int encode_q_nope(CUtensorMap* m, const void* q_nope, int B, int n_tile, int n_heads) {
  cuuint64_t dims[3] = {(cuuint64_t)kDn, (cuuint64_t)n_heads, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)kDn * 2, (cuuint64_t)n_heads * kDn * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)n_tile};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q_nope), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// A per-head query tensor (q_lat: width 512, or q_pe: width 64) as a 3-D bf16
// tensor {c: width, h: n_heads, b: B}, boxes of `box_c` columns x 128 heads x
// 1 row: one box is a column block of all heads of a row (heads past n_heads
// lie outside the tensor and read as zero).
int encode_q_half(CUtensorMap* m, const void* q, int B, int n_heads, int width, int box_c,
                  CUtensorMapSwizzle swizzle) {
  cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)n_heads, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)n_heads * width * 2};
  cuuint32_t box[3] = {(cuuint32_t)box_c, (cuuint32_t)kH, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// The mixed latent O~ (single-split rows) as a 3-D bf16 tensor
// {c: 512, h: n_heads, b: B}, boxes of 64 c x 1 head x n_tile rows, 128-byte
// swizzle (rows past B read as zero).
int encode_o_lat(CUtensorMap* m, const void* o_lat, int B, int n_tile, int n_heads) {
  cuuint64_t dims[3] = {(cuuint64_t)kDl, (cuuint64_t)n_heads, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)kDl * 2, (cuuint64_t)n_heads * kDl * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)n_tile};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(o_lat), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// wo (its first k_in columns) as a 2-D bf16 tensor [dim rows, k_in columns]
// with rows ld elements apart, boxes of 64 columns x 128 rows, 128-byte
// swizzle.
int encode_wo(CUtensorMap* m, const void* wo, int dim, int k_in, long long ld) {
  cuuint64_t dims[2] = {(cuuint64_t)k_in, (cuuint64_t)dim};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)kProjKBlock, (cuuint32_t)kProjM};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(wo), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// wo viewed as a 4-D bf16 tensor (64 k, 8 rows of a group, k_in/64 k-blocks,
// dim/8 groups) with strides (2 B, 2 ld B, 128 B, 16 ld B) (32 KB and 256 KB
// for the full wo): one box {64, 8, 4, 16} is 128 rows x 4 consecutive
// k-blocks, each row's four 128-byte pieces read back to back, landing as
// [group][k-block][row][128 B] (128-byte swizzle).
int encode_wo4(CUtensorMap* m, const void* wo, int dim, int k_in, long long ld) {
  cuuint64_t dims[4] = {(cuuint64_t)kProjKBlock, 8, (cuuint64_t)(k_in / kProjKBlock), (cuuint64_t)dim / 8};
  cuuint64_t strides[3] = {(cuuint64_t)ld * 2, (cuuint64_t)kProjKBlock * 2, (cuuint64_t)ld * 2 * 8};
  cuuint32_t box[4] = {(cuuint32_t)kProjKBlock, 8, (cuuint32_t)kProjKGroupWide, (cuuint32_t)(kProjM / 8)};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(wo), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// The projection input x as a 2-D bf16 tensor [B rows, k_in columns], boxes
// of 64 columns x n_tile rows, 128-byte swizzle (rows past B read as zero).
int encode_proj_x(CUtensorMap* m, const void* x, int B, int n_tile, int k_in) {
  cuuint64_t dims[2] = {(cuuint64_t)k_in, (cuuint64_t)B};
  cuuint64_t strides[1] = {(cuuint64_t)k_in * 2};
  cuuint32_t box[2] = {(cuuint32_t)kProjKBlock, (cuuint32_t)n_tile};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// ---------------------------------------------------------------- planning

constexpr int kMaxB = 1 << 20;
constexpr int kMaxK = 1 << 24;

bool sizes_ok(int B, int K, int S_max) { return B >= 1 && B <= kMaxB && K >= 1 && K <= kMaxK && S_max >= 1; }

// Splits of the K index slots of a row: enough (row, split) pairs to give
// every 2-SM cluster work, never more splits than 32-slot tiles, each split a
// whole number of tiles.
void plan_splits(int B, int K, int sm_count, int* n_split, int* span) {
  const int clusters = sm_count / 2 > 0 ? sm_count / 2 : 1;
  const int tiles = ceil_div(K, kNt);
  int want = clusters / B;
  if (want < 1) want = 1;
  if (want > tiles) want = tiles;
  if (want > kCombineMaxSplits) want = kCombineMaxSplits;
  const int sp = ceil_div(ceil_div(K, want), kNt) * kNt;
  *span = sp;
  *n_split = ceil_div(K, sp);
}

constexpr int kProjMaxDim = 1 << 16;

bool proj_sizes_ok(int B, int dim) {
  return B >= 1 && B <= kMaxB && dim >= kProjM && dim <= kProjMaxDim && dim % kProjM == 0;
}

// Output projection: batch tiles of at most 256 rows (equal, multiples of 16);
// with fewer output tiles than SMs one CTA per SM shares the work unit by unit
// (f32 partials, then the reduce kernel), otherwise one CTA per tile writes
// bf16 directly.
struct ProjPlan {
  int n_tile = 0, tiles = 0, n_ctas = 0, kgroup = 1, k_blocks = kProjKBlocks;
  bool direct = false;
  size_t partial_bytes = 0;
};

ProjPlan plan_projection(int B, int dim, int sm_count, int k_in = kProjK) {
  ProjPlan p;
  p.k_blocks = k_in / kProjKBlock;
  const int y_tiles = ceil_div(B, kProjNMax);
  p.n_tile = ceil_div(ceil_div(B, y_tiles), 16) * 16;
  p.tiles = y_tiles * (dim / kProjM);
  p.direct = p.tiles >= sm_count;
  // four k-blocks per unit where two such stages fit (split mode only: a
  // direct CTA's tile is 256 units of one k-block)
  p.kgroup = (!p.direct && p.n_tile <= kProjWideNMax && p.k_blocks % kProjKGroupWide == 0) ? kProjKGroupWide : 1;
  // split mode: at most one CTA per unit (every CTA owns at least one unit, so
  // the reduce's contributors are exactly the CTAs between a tile's first and
  // last unit) and more CTAs than tiles (a range spans at most two tiles)
  const long long units = (long long)p.tiles * (p.k_blocks / p.kgroup);
  p.n_ctas = p.direct ? p.tiles : (int)(units < sm_count ? units : sm_count);
  p.partial_bytes = p.direct ? 0 : (size_t)2 * p.n_ctas * p.n_tile * kProjM * sizeof(float);
  return p;
}

struct WorkspaceLayout {
  size_t q_lat = 0, o_part = 0, lse_part = 0, total = 0;
};

WorkspaceLayout workspace_layout(int B, int n_split, int n_heads = kH) {
  WorkspaceLayout w;
  size_t off = 0;
  w.q_lat = off;
  off = round_up(off + (size_t)B * n_heads * kDl * 2, 256);
  w.o_part = off;  // bf16: each split's normalised mix (O~ itself when a row is one split)
  off = round_up(off + (size_t)B * n_split * n_heads * kDl * 2, 256);
  w.lse_part = off;
  off = round_up(off + (size_t)B * n_split * n_heads * 4, 256);
  w.total = off;
  return w;
}

int launch_check() { return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// Launch with or without a programmatic dependency on the previous kernel in
// the stream.  With one, the kernel may start before that kernel has finished
// and must call grid_dep_wait() before it reads anything the other writes; the
// decode step uses it only between its own kernels.
template <typename... KArgs, typename... Args>
int launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return launch_check();
}

int launch_absorb(const void* q_nope, const void* wkv_b, void* q_lat, int B, int* d_status, cudaStream_t stream,
                  int n_heads = kH) {
  const int n_tile = B >= kAbsorbNMax ? kAbsorbNMax : ceil_div(B, 16) * 16;
  CUtensorMap tm_w, tm_q;
  int rc;
  if ((rc = encode_wkv_b(&tm_w, wkv_b, n_heads)) != MLA_OK) return rc;
  if ((rc = encode_q_nope(&tm_q, q_nope, B, n_tile, n_heads)) != MLA_OK) return rc;
  dim3 grid(kDl / 128, n_heads, ceil_div(B, kAbsorbNMax));
  return launch_ex(absorb_kernel, grid, dim3(128), absorb_smem_bytes(n_tile), stream, false, tm_w, tm_q,
                   static_cast<__nv_bfloat16*>(q_lat), B, n_tile, n_heads, d_status);
}

int launch_attend(const void* q_lat, const void* q_pe, const void* kv_cache, const void* pe_cache,
                  const int32_t* end_pos, const int32_t* topk_idx, float scale, void* o_part, float* lse_part, int B,
                  int K, int S_max, int n_split, int span, const void* w_next, int* d_status, cudaStream_t stream,
                  bool pdl, const int32_t* cache_slot = nullptr, int n_slots = 0, int n_heads = kH) {
  const long long ctas = 2LL * B * n_split;
  if (ctas > 0x7fffffffLL) return MLA_ERR_INVALID_ARG;
  CUtensorMap tm_qlat, tm_qpe;
  int rc;
  if ((rc = encode_q_half(&tm_qlat, q_lat, B, n_heads, kDl, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK) return rc;
  if ((rc = encode_q_half(&tm_qpe, q_pe, B, n_heads, kDr, 32, CU_TENSOR_MAP_SWIZZLE_64B)) != MLA_OK) return rc;
  return launch_ex(sparse_attend_kernel, dim3((unsigned)ctas), dim3(kAttendThreads), kAttendSmemBytes, stream, pdl,
                   tm_qlat, tm_qpe,
                   static_cast<const __nv_bfloat16*>(kv_cache), static_cast<const __nv_bfloat16*>(pe_cache), end_pos,
                   topk_idx, scale, o_part, lse_part, K, S_max, n_split, span,
                   static_cast<const __nv_bfloat16*>(w_next), cache_slot, n_slots, n_heads, d_status);
}

int launch_combine(const void* o_part, const float* lse_part, const void* wkv_b, void* out, float* lse_out, int B,
                   int n_split, int* d_status, cudaStream_t stream, bool pdl, int n_heads = kH) {
  const int n_tile = B >= kCombineNMax ? kCombineNMax : ceil_div(B, 16) * 16;
  CUtensorMap tm_w, tm_o;
  int rc;
  if ((rc = encode_wkv_b(&tm_w, wkv_b, n_heads)) != MLA_OK) return rc;
  if (n_split == 1) {
    if ((rc = encode_o_lat(&tm_o, o_part, B, n_tile, n_heads)) != MLA_OK) return rc;
  } else {
    tm_o = tm_w;  // unused
  }
  dim3 grid(n_heads, ceil_div(B, kCombineNMax));
  return launch_ex(combine_value_up_kernel, grid, dim3(kCombineThreads), kCombineSmemBytes, stream, pdl, tm_w, tm_o,
                   o_part, lse_part, static_cast<__nv_bfloat16*>(out), lse_out, B, n_split, n_tile, n_heads, d_status);
}

// projection_kernel, then (unless every CTA wrote its tile directly) the
// reduce kernel with a programmatic dependency on it.  With pdl, the
// projection kernel itself depends programmatically on the kernel before it:
// it requests its first weight stages before waiting for that kernel.
// With `prepared`, wo is in the prepared layout (mla_prepare_wo) and is read
// by bulk copies; its tensor maps are not used.
int launch_projection(const void* x, const void* wo, void* delta, int B, int dim, const ProjPlan& p, void* partial,
                      int* d_status, cudaStream_t stream, bool pdl, long long ld_wo = kProjK, bool prepared = false) {
  const int k_in = p.k_blocks * kProjKBlock;
  CUtensorMap tm_wo, tm_wo4, tm_x;
  int rc;
  if (prepared) {
    std::memset(&tm_wo, 0, sizeof(tm_wo));  // unused
    tm_wo4 = tm_wo;
  } else {
    if ((rc = encode_wo(&tm_wo, wo, dim, k_in, ld_wo)) != MLA_OK) return rc;
    if (p.kgroup == 1)
      tm_wo4 = tm_wo;  // unused
    else if ((rc = encode_wo4(&tm_wo4, wo, dim, k_in, ld_wo)) != MLA_OK)
      return rc;
  }
  if ((rc = encode_proj_x(&tm_x, x, B, p.n_tile, k_in)) != MLA_OK) return rc;
  if ((rc = launch_ex(projection_kernel, dim3((unsigned)p.n_ctas), dim3(kProjThreads),
                      proj_smem_bytes(p.n_tile, p.kgroup), stream, pdl, tm_wo, tm_wo4, tm_x,
                      static_cast<const __nv_bfloat16*>(prepared ? wo : nullptr), static_cast<float*>(partial),
                      static_cast<__nv_bfloat16*>(delta), B, dim, p.n_tile, p.n_ctas, p.direct ? 1 : 0, p.kgroup,
                      p.k_blocks, d_status)) != MLA_OK)
    return rc;
  if (p.direct) return MLA_OK;
  dim3 grid((unsigned)p.tiles, ceil_div(p.n_tile, kProjReduceRows));
  return launch_ex(projection_reduce_kernel, grid, dim3(kProjReduceThreads), 0, stream, true,
                   static_cast<const float*>(partial), static_cast<__nv_bfloat16*>(delta), B, dim, p.n_tile,
                   p.n_ctas, p.kgroup, p.k_blocks);
}

int prepare(DeviceInfo** info) {
  int rc = current_device(info);
  if (rc != MLA_OK) return rc;
  return get_encoder();
}

// Fixed device scratch for mla_sparse_decode_noalloc: one array per device
// that loads the library, alive until the process exits.  Host code only sees
// a stand-in for it, so its device address is looked up once per device.
__device__ __align__(256) uint8_t g_mla_static_scratch[MLA_STATIC_SCRATCH_BYTES];
void* g_static_scratch_addr[kMaxDevices] = {};

// Device address of g_mla_static_scratch on the current device (resolved on
// the first call made with that device current).
int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_static_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_static_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return MLA_OK;
}

}  // namespace

// =============================================================================
// C ABI
// =============================================================================

extern "C" const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
    case MLA_ERR_BAD_INDEX: return "MLA_ERR_BAD_INDEX";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    default: return "MLA_ERR_UNKNOWN";
  }
}

extern "C" int mla_num_splits(int B, int K) {
  if (!sizes_ok(B, K, 1)) return 0;
  int n_split = 0, span = 0;
  plan_splits(B, K, planning_sm_count(), &n_split, &span);
  return n_split;
}

extern "C" size_t mla_sparse_decode_workspace_size(int B, int K, int S_max) {
  if (!sizes_ok(B, K, S_max)) return 0;
  int n_split = 0, span = 0;
  plan_splits(B, K, planning_sm_count(), &n_split, &span);
  return workspace_layout(B, n_split).total;
}

extern "C" int mla_absorb_q(const void* q_nope, const void* wkv_b, void* q_lat, int B, cudaStream_t stream) {
  if (!q_nope || !wkv_b || !q_lat || !aligned16(q_nope) || !aligned16(wkv_b) || !aligned16(q_lat)) return MLA_ERR_INVALID_ARG;
  if (B < 1 || B > kMaxB) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  return launch_absorb(q_nope, wkv_b, q_lat, B, nullptr, stream);
}

extern "C" int mla_sparse_attend(const void* q_lat, const void* q_pe, const void* kv_cache, const void* pe_cache,
                                 const int32_t* end_pos, const int32_t* topk_idx, float scale, void* o_part,
                                 float* lse_part, int B, int K, int S_max, int n_split, int* d_status,
                                 cudaStream_t stream) {
  const void* ptrs[] = {q_lat, q_pe, kv_cache, pe_cache, end_pos, topk_idx, o_part, lse_part};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (!sizes_ok(B, K, S_max) || !std::isfinite(scale)) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  int want = 0, span = 0;
  plan_splits(B, K, info->sm_count, &want, &span);
  if (n_split != want) return MLA_ERR_INVALID_ARG;
  return launch_attend(q_lat, q_pe, kv_cache, pe_cache, end_pos, topk_idx, scale, o_part, lse_part, B, K, S_max,
                       n_split, span, nullptr, d_status, stream, false);
}

extern "C" int mla_combine_value_up(const void* o_part, const float* lse_part, const void* wkv_b, void* out,
                                    float* lse_out, int B, int n_split, cudaStream_t stream) {
  if (!o_part || !lse_part || !wkv_b || !out) return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_part) || !aligned16(lse_part) || !aligned16(wkv_b) || !aligned16(out)) return MLA_ERR_INVALID_ARG;
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return MLA_ERR_INVALID_ARG;
  if (B < 1 || B > kMaxB || n_split < 1 || n_split > kCombineMaxSplits) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  return launch_combine(o_part, lse_part, wkv_b, out, lse_out, B, n_split, nullptr, stream, false);
}

namespace {
// Opt-in index validation before every decode / prefill call (see
// mla_set_index_checks); off by default.
std::atomic<int> g_index_checks{0};

int launch_check_indices(const int32_t* end_pos, const int32_t* topk_idx, int B, int K, int S_max, int* d_status,
                         int* d_dup, cudaStream_t stream) {
  const size_t smem = (size_t)check_bitmap_words(S_max) * 4;
  return launch_ex(check_indices_kernel, dim3((unsigned)B), dim3(kCheckThreads), smem, stream, false, end_pos,
                   topk_idx, K, S_max, d_status, d_dup);
}
}  // namespace

namespace {
// The three kernels over B rows: row b is one query (its q_nope, q_pe, index
// row and end position) and reads cache slot cache_slot[b], or b when
// cache_slot is null.  Shared by the decode step (a row per batch row) and
// the prefill (a row per query position of a sequence).
int run_rows(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
             const int32_t* end_pos, const int32_t* topk_idx, const void* wkv_b, float scale, void* out, int B, int K,
             int S_max, const int32_t* cache_slot, int n_slots, void* workspace, size_t workspace_bytes,
             float* lse_out, int* d_status, cudaStream_t stream, int n_heads = kH) {
  const void* ptrs[] = {q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return MLA_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MLA_ERR_INVALID_ARG;
  if (!sizes_ok(B, K, S_max) || !std::isfinite(scale)) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  int n_split = 0, span = 0;
  plan_splits(B, K, info->sm_count, &n_split, &span);
  const WorkspaceLayout wl = workspace_layout(B, n_split, n_heads);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < wl.total)
    return MLA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* q_lat = ws + wl.q_lat;
  void* o_part = ws + wl.o_part;
  float* lse_part = reinterpret_cast<float*>(ws + wl.lse_part);

  if (d_status && g_index_checks.load(std::memory_order_relaxed) &&
      (rc = launch_check_indices(end_pos, topk_idx, B, K, S_max, d_status, nullptr, stream)) != MLA_OK)
    return rc;
  // The attention and combine kernels depend programmatically on the kernel
  // before them: each starts while its predecessor drains and waits for it
  // only where it reads that kernel's output.  The absorption kernel is an
  // ordinary launch, so all earlier work in the stream (whatever wrote the
  // caches and indices) has finished before any of the three starts.
  if ((rc = launch_absorb(q_nope, wkv_b, q_lat, B, d_status, stream, n_heads)) != MLA_OK) return rc;
  // The attention kernel also pulls W_UV into L2 near its end, for the
  // value-up kernel.
  if ((rc = launch_attend(q_lat, q_pe, kv_cache, pe_cache, end_pos, topk_idx, scale, o_part, lse_part, B, K, S_max,
                          n_split, span, wkv_b, d_status, stream, true, cache_slot, n_slots, n_heads)) != MLA_OK)
    return rc;
  return launch_combine(o_part, lse_part, wkv_b, out, lse_out, B, n_split, d_status, stream, true, n_heads);
}
}  // namespace

extern "C" int mla_sparse_decode(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                                 const int32_t* end_pos, const int32_t* topk_idx, const void* wkv_b, float scale,
                                 void* out, int B, int K, int S_max, void* workspace, size_t workspace_bytes,
                                 float* lse_out, int* d_status, cudaStream_t stream) {
  return run_rows(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, scale, out, B, K, S_max, nullptr, B,
                  workspace, workspace_bytes, lse_out, d_status, stream);
}

// The sparse prefill (see the header): R query rows over n_slots sequences'
// latents, row r reading slot cache_slot[r] with its own causal end position.
extern "C" int mla_sparse_prefill(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                                  const int32_t* cache_slot, const int32_t* end_pos, const int32_t* topk_idx,
                                  const void* wkv_b, float scale, void* out, int R, int K, int S_max, int n_slots,
                                  void* workspace, size_t workspace_bytes, float* lse_out, int* d_status,
                                  cudaStream_t stream) {
  if (!cache_slot || !aligned16(cache_slot) || n_slots < 1) return MLA_ERR_INVALID_ARG;
  return run_rows(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, scale, out, R, K, S_max, cache_slot,
                  n_slots, workspace, workspace_bytes, lse_out, d_status, stream);
}

// One tensor-parallel shard of the decode (see the header): the same three
// kernels over n_heads consecutive heads.
extern "C" size_t mla_sparse_decode_heads_workspace_size(int B, int K, int S_max, int n_heads) {
  if (!sizes_ok(B, K, S_max) || n_heads < 1 || n_heads > kH) return 0;
  int n_split = 0, span = 0;
  plan_splits(B, K, planning_sm_count(), &n_split, &span);
  return workspace_layout(B, n_split, n_heads).total;
}

extern "C" int mla_sparse_decode_heads(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                                       const int32_t* end_pos, const int32_t* topk_idx, const void* wkv_b,
                                       float scale, void* out, int B, int K, int S_max, int n_heads, void* workspace,
                                       size_t workspace_bytes, float* lse_out, int* d_status, cudaStream_t stream) {
  if (n_heads < 1 || n_heads > kH) return MLA_ERR_INVALID_ARG;
  return run_rows(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, scale, out, B, K, S_max, nullptr, B,
                  workspace, workspace_bytes, lse_out, d_status, stream, n_heads);
}

// fp8 block dequantisation (see the header).
extern "C" int mla_dequant_fp8_blocks(const void* w_fp8, const float* scale, void* w_bf16, int rows, int cols,
                                      cudaStream_t stream) {
  if (!w_fp8 || !scale || !w_bf16 || !aligned16(w_fp8) || !aligned16(w_bf16)) return MLA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(scale) & 3u) return MLA_ERR_INVALID_ARG;
  if (rows < 1 || cols < 16 || cols % 16 || (long long)rows * cols > (1LL << 40)) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  const long long n_vec = (long long)rows * (cols / 16);
  long long blocks = (n_vec + kDequantThreads - 1) / kDequantThreads;
  if (blocks > 8LL * info->sm_count) blocks = 8LL * info->sm_count;
  return launch_ex(dequant_fp8_blocks_kernel, dim3((unsigned)blocks), dim3(kDequantThreads), 0, stream, false,
                   static_cast<const uint8_t*>(w_fp8), scale, static_cast<__nv_bfloat16*>(w_bf16), rows, cols);
}

// Index validation (see the header): repeated valid entries of a row.
extern "C" int mla_check_topk_indices(const int32_t* end_pos, const int32_t* topk_idx, int B, int K, int S_max,
                                      int* d_status, int* d_row_flags, cudaStream_t stream) {
  if (!end_pos || !topk_idx || !aligned16(end_pos) || !aligned16(topk_idx)) return MLA_ERR_INVALID_ARG;
  if (!d_status && !d_row_flags) return MLA_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MLA_ERR_INVALID_ARG;
  if (d_row_flags && (reinterpret_cast<uintptr_t>(d_row_flags) & 3u)) return MLA_ERR_INVALID_ARG;
  if (!sizes_ok(B, K, S_max)) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  return launch_check_indices(end_pos, topk_idx, B, K, S_max, d_status, d_row_flags, stream);
}

extern "C" int mla_set_index_checks(int enable) {
  return g_index_checks.exchange(enable ? 1 : 0);
}

#ifdef MLA_TRACE
// Trace builds only: copies the pipeline trace of the last traced launch
// (2 CTAs x kTrEvents x kTraceTiles clock64 stamps) to host memory.
extern "C" int mla_trace_fetch(long long* host, int n) {
  const int total = 2 * kTrEvents * kTraceTiles;
  if (!host || n < total) return MLA_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(host, g_mla_trace, sizeof(long long) * total) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// Trace builds only: clears the whole-kernel stamps (earliest-start slots to
// the largest value, latest-end slots to zero).
extern "C" int mla_trace_reset() {
  unsigned long long v[kKernelEvents];
  for (int e = 0; e < kKernelEvents; ++e)
    v[e] = (e == kKeAbsorbStart || e == kKeCombineStart || e == kKeCombineFirstWaited) ? ~0ull : 0ull;
  return cudaMemcpyToSymbol(g_mla_kernel_ns, v, sizeof(v)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// Trace builds only: the whole-kernel stamps (kKernelEvents values).
extern "C" int mla_trace_kernel_fetch(unsigned long long* host, int n) {
  if (!host || n < kKernelEvents) return MLA_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(host, g_mla_kernel_ns, sizeof(unsigned long long) * kKernelEvents) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

// Trace builds only: the milestones of every cluster of the last traced
// launch (kClusterEvents values per cluster, 4096 clusters).
extern "C" int mla_trace_cluster_fetch(unsigned long long* host, int n) {
  const int total = kClusterEvents * kTraceClusters;
  if (!host || n < total) return MLA_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(host, g_mla_cluster_ns, sizeof(unsigned long long) * total) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}
#endif

// The decode step without a caller-provided workspace: the scratch lives in
// the library's fixed device array (see the header for who needs this).
// Everything it holds is written before it is read, so nothing is cleared.
extern "C" int mla_sparse_decode_noalloc(const void* q_nope, const void* q_pe, const void* kv_cache,
                                         const void* pe_cache, const int32_t* end_pos, const int32_t* topk_idx,
                                         const void* wkv_b, float scale, void* out, int B, int K, int S_max,
                                         float* lse_out, int* d_status, cudaStream_t stream) {
  const void* ptrs[] = {q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return MLA_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MLA_ERR_INVALID_ARG;
  if (!sizes_ok(B, K, S_max) || !std::isfinite(scale)) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  int n_split = 0, span = 0;
  plan_splits(B, K, info->sm_count, &n_split, &span);
  if (workspace_layout(B, n_split).total > (size_t)MLA_STATIC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((rc = static_scratch_address(&scratch)) != MLA_OK) return rc;
  return mla_sparse_decode(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, scale, out, B, K, S_max,
                           scratch, (size_t)MLA_STATIC_SCRATCH_BYTES, lse_out, d_status, stream);
}

// ---------------------------------------------------------------- host-buffer entry
// The decode step with the per-call tensors in host memory (see the header):
// the workspace holds the decode scratch, then device staging copies of the
// four inputs and the output.
namespace {
struct HostStaging {
  size_t decode = 0, q_nope = 0, q_pe = 0, end_pos = 0, topk_idx = 0, out = 0, total = 0;
};

HostStaging host_staging(int B, int K, int n_split) {
  HostStaging h;
  size_t off = workspace_layout(B, n_split).total;
  h.decode = 0;
  h.q_nope = off;
  off = round_up(off + (size_t)B * kH * kDn * 2, 256);
  h.q_pe = off;
  off = round_up(off + (size_t)B * kH * kDr * 2, 256);
  h.end_pos = off;
  off = round_up(off + (size_t)B * 4, 256);
  h.topk_idx = off;
  off = round_up(off + (size_t)B * K * 4, 256);
  h.out = off;
  off = round_up(off + (size_t)B * kH * kDv * 2, 256);
  h.total = off;
  return h;
}
}  // namespace

extern "C" size_t mla_sparse_decode_host_input_layout(int B, int K, int S_max, size_t* offsets) {
  if (!sizes_ok(B, K, S_max)) return 0;
  int n_split = 0, span = 0;
  plan_splits(B, K, planning_sm_count(), &n_split, &span);
  const HostStaging hs = host_staging(B, K, n_split);
  if (offsets) {
    offsets[0] = 0;
    offsets[1] = hs.q_pe - hs.q_nope;
    offsets[2] = hs.end_pos - hs.q_nope;
    offsets[3] = hs.topk_idx - hs.q_nope;
  }
  return hs.topk_idx + (size_t)B * K * 4 - hs.q_nope;
}

extern "C" size_t mla_sparse_decode_host_workspace_size(int B, int K, int S_max) {
  if (!sizes_ok(B, K, S_max)) return 0;
  int n_split = 0, span = 0;
  plan_splits(B, K, planning_sm_count(), &n_split, &span);
  return host_staging(B, K, n_split).total;
}

extern "C" int mla_sparse_decode_host(const void* h_q_nope, const void* h_q_pe, const int32_t* h_end_pos,
                                      const int32_t* h_topk_idx, const void* kv_cache, const void* pe_cache,
                                      const void* wkv_b, float scale, void* h_out, int B, int K, int S_max,
                                      void* workspace, size_t workspace_bytes, float* lse_out, int* d_status,
                                      cudaStream_t stream) {
  const void* ptrs[] = {h_q_nope, h_q_pe, h_end_pos, h_topk_idx, kv_cache, pe_cache, wkv_b, h_out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return MLA_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MLA_ERR_INVALID_ARG;
  if (!sizes_ok(B, K, S_max) || !std::isfinite(scale)) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  int n_split = 0, span = 0;
  plan_splits(B, K, info->sm_count, &n_split, &span);
  const HostStaging hs = host_staging(B, K, n_split);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < hs.total)
    return MLA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* d_q_nope = ws + hs.q_nope;
  void* d_q_pe = ws + hs.q_pe;
  int32_t* d_end_pos = reinterpret_cast<int32_t*>(ws + hs.end_pos);
  int32_t* d_topk_idx = reinterpret_cast<int32_t*>(ws + hs.topk_idx);
  void* d_out = ws + hs.out;
  // Host inputs laid out like the staging area (one buffer, the offsets of
  // mla_sparse_decode_host_input_layout) go up in a single copy; otherwise one
  // plain asynchronous copy per tensor.  Pinned host memory makes them truly
  // asynchronous; pageable memory works but stages through the driver.
  const char* h0 = static_cast<const char*>(h_q_nope);
  const bool packed = static_cast<const char*>(h_q_pe) == h0 + (hs.q_pe - hs.q_nope) &&
                      reinterpret_cast<const char*>(h_end_pos) == h0 + (hs.end_pos - hs.q_nope) &&
                      reinterpret_cast<const char*>(h_topk_idx) == h0 + (hs.topk_idx - hs.q_nope);
  if (packed) {
    if (cudaMemcpyAsync(d_q_nope, h_q_nope, hs.topk_idx + (size_t)B * K * 4 - hs.q_nope, cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
      return MLA_ERR_CUDA;
  } else if (cudaMemcpyAsync(d_q_nope, h_q_nope, (size_t)B * kH * kDn * 2, cudaMemcpyHostToDevice, stream) !=
                 cudaSuccess ||
             cudaMemcpyAsync(d_q_pe, h_q_pe, (size_t)B * kH * kDr * 2, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
             cudaMemcpyAsync(d_end_pos, h_end_pos, (size_t)B * 4, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
             cudaMemcpyAsync(d_topk_idx, h_topk_idx, (size_t)B * K * 4, cudaMemcpyHostToDevice, stream) != cudaSuccess) {
    return MLA_ERR_CUDA;
  }
  rc = mla_sparse_decode(d_q_nope, d_q_pe, kv_cache, pe_cache, d_end_pos, d_topk_idx, wkv_b, scale, d_out, B, K,
                         S_max, ws, hs.q_nope, lse_out, d_status, stream);
  if (rc != MLA_OK) return rc;
  if (cudaMemcpyAsync(h_out, d_out, (size_t)B * kH * kDv * 2, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

// ---------------------------------------------------------------- output projection
// delta = x . wo^T (see the header).

extern "C" size_t mla_output_projection_workspace_size(int B, int dim) {
  if (!proj_sizes_ok(B, dim)) return 0;
  const ProjPlan p = plan_projection(B, dim, planning_sm_count());
  return p.partial_bytes > 0 ? p.partial_bytes : 256;  // never 0 for valid sizes
}

extern "C" int mla_output_projection(const void* x, const void* wo, void* delta, int B, int dim, void* workspace,
                                     size_t workspace_bytes, int* d_status, cudaStream_t stream) {
  const void* ptrs[] = {x, wo, delta};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MLA_ERR_INVALID_ARG;
  if (!proj_sizes_ok(B, dim)) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  const ProjPlan p = plan_projection(B, dim, info->sm_count);
  const size_t need = p.partial_bytes > 0 ? p.partial_bytes : 256;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
    return MLA_ERR_WORKSPACE;
  return launch_projection(x, wo, delta, B, dim, p, workspace, d_status, stream, false);
}

// The projection of a tensor-parallel shard (see the header): x [B, k_in],
// wo's rows ld_wo elements apart, its first k_in columns used.
extern "C" size_t mla_output_projection_shard_workspace_size(int B, int dim, int k_in) {
  if (!proj_sizes_ok(B, dim) || k_in < kProjKBlock || k_in > kProjK || k_in % kProjKBlock) return 0;
  const ProjPlan p = plan_projection(B, dim, planning_sm_count(), k_in);
  return p.partial_bytes > 0 ? p.partial_bytes : 256;
}

extern "C" int mla_output_projection_shard(const void* x, const void* wo, long long ld_wo, void* delta, int B,
                                           int dim, int k_in, void* workspace, size_t workspace_bytes, int* d_status,
                                           cudaStream_t stream) {
  const void* ptrs[] = {x, wo, delta};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MLA_ERR_INVALID_ARG;
  if (!proj_sizes_ok(B, dim) || k_in < kProjKBlock || k_in > kProjK || k_in % kProjKBlock) return MLA_ERR_INVALID_ARG;
  if (ld_wo < k_in || ld_wo % 8 || ld_wo > (1LL << 31)) return MLA_ERR_INVALID_ARG;  // rows 16-byte aligned
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  const ProjPlan p = plan_projection(B, dim, info->sm_count, k_in);
  const size_t need = p.partial_bytes > 0 ? p.partial_bytes : 256;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
    return MLA_ERR_WORKSPACE;
  return launch_projection(x, wo, delta, B, dim, p, workspace, d_status, stream, false, ld_wo);
}

// wo in the prepared layout (see projection.cuh): one pass over it, once per
// weight.
extern "C" int mla_prepare_wo(const void* wo, long long ld_wo, int dim, int k_in, void* wo_prepared,
                              cudaStream_t stream) {
  if (!wo || !wo_prepared || !aligned16(wo) || !aligned16(wo_prepared)) return MLA_ERR_INVALID_ARG;
  if (dim < kProjM || dim > kProjMaxDim || dim % kProjM) return MLA_ERR_INVALID_ARG;
  if (k_in < kProjTileK || k_in > kProjK || k_in % kProjTileK) return MLA_ERR_INVALID_ARG;
  if (ld_wo < k_in || ld_wo % 8 || ld_wo > (1LL << 31)) return MLA_ERR_INVALID_ARG;  // rows 16-byte aligned
  DeviceInfo* info = nullptr;
  int rc = current_device(&info);
  if (rc != MLA_OK) return rc;
  const long long chunks = (long long)dim * (k_in / 8);
  const long long want = (chunks + 255) / 256;
  const unsigned grid = (unsigned)(want < 8LL * info->sm_count ? want : 8LL * info->sm_count);
  return launch_ex(prepare_wo_kernel, dim3(grid), dim3(256), 0, stream, false, static_cast<const uint4*>(wo),
                   ld_wo / 8, dim, k_in, static_cast<uint4*>(wo_prepared));
}

extern "C" int mla_output_projection_prepared(const void* x, const void* wo_prepared, void* delta, int B, int dim,
                                              int k_in, void* workspace, size_t workspace_bytes, int* d_status,
                                              cudaStream_t stream) {
  const void* ptrs[] = {x, wo_prepared, delta};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MLA_ERR_INVALID_ARG;
  if (!proj_sizes_ok(B, dim) || k_in < kProjTileK || k_in > kProjK || k_in % kProjTileK) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  const ProjPlan p = plan_projection(B, dim, info->sm_count, k_in);
  const size_t need = p.partial_bytes > 0 ? p.partial_bytes : 256;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
    return MLA_ERR_WORKSPACE;
  return launch_projection(x, wo_prepared, delta, B, dim, p, workspace, d_status, stream, false, kProjK, true);
}

// The decode step followed by the output projection: the workspace holds the
// decode scratch, the per-head outputs (bf16 [B,16384]) and the projection's
// partials.
namespace {
struct ProjectLayout {
  size_t decode = 0, out = 0, partial = 0, total = 0;
};
ProjectLayout project_layout(int B, int K, int dim, int sm_count) {
  ProjectLayout l;
  int n_split = 0, span = 0;
  plan_splits(B, K, sm_count, &n_split, &span);
  size_t off = round_up(workspace_layout(B, n_split).total, 256);
  l.out = off;
  off = round_up(off + (size_t)B * kProjK * 2, 256);
  l.partial = off;
  off = round_up(off + plan_projection(B, dim, sm_count).partial_bytes, 256);
  l.total = off;
  l.decode = l.out;
  return l;
}
}  // namespace

extern "C" size_t mla_sparse_decode_project_workspace_size(int B, int K, int S_max, int dim) {
  if (!sizes_ok(B, K, S_max) || !proj_sizes_ok(B, dim)) return 0;
  return project_layout(B, K, dim, planning_sm_count()).total;
}

extern "C" int mla_sparse_decode_project(const void* q_nope, const void* q_pe, const void* kv_cache,
                                         const void* pe_cache, const int32_t* end_pos, const int32_t* topk_idx,
                                         const void* wkv_b, float scale, const void* wo, void* delta, int B, int K,
                                         int S_max, int dim, void* workspace, size_t workspace_bytes,
                                         float* lse_out, int* d_status, cudaStream_t stream) {
  const void* ptrs[] = {q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, wo, delta};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MLA_ERR_INVALID_ARG;
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return MLA_ERR_INVALID_ARG;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return MLA_ERR_INVALID_ARG;
  if (!sizes_ok(B, K, S_max) || !proj_sizes_ok(B, dim) || !std::isfinite(scale)) return MLA_ERR_INVALID_ARG;
  DeviceInfo* info = nullptr;
  int rc = prepare(&info);
  if (rc != MLA_OK) return rc;
  const ProjectLayout l = project_layout(B, K, dim, info->sm_count);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < l.total)
    return MLA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* out = ws + l.out;
  rc = mla_sparse_decode(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, scale, out, B, K, S_max, ws,
                         l.decode, lse_out, d_status, stream);
  if (rc != MLA_OK) return rc;
  // programmatic dependency on the value-up kernel: the first weight stages
  // of wo stream in while it finishes
  return launch_projection(out, wo, delta, B, dim, plan_projection(B, dim, info->sm_count), ws + l.partial,
                           d_status, stream, true);
}

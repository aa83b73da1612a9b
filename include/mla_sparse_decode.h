/*
 * mla_sparse_decode.h -- C ABI of the B200 (sm_100a) sparse MLA decode library.
 *
 * Also declared here, after the decode step: the sparse prefill over the same
 * kernels (mla_sparse_prefill, page "Queries"), the attention output
 * projection (mla_output_projection, mla_sparse_decode_project, page
 * "Attention update"), a tensor-parallel shard of both
 * (mla_sparse_decode_heads, mla_output_projection_shard), the fp8 weight
 * dequantisation (mla_dequant_fp8_blocks) and index validation
 * (mla_check_topk_indices).
 *
 * One decode step of DeepSeek-V3.2-Exp's absorbed multi-head latent attention
 * with the indexer's top-k mask, as the atlas pages of
 * deepseek-ai/DeepSeek-V3.2-Exp inference/model.py (rev 87e509a2e5a1) show it:
 *   - "Query-key similarity" (decode): MQA-decode excerpt, model.py 590-606:
 *       absorb   q_lat = einsum("bshd,hdc->bshc", q_nope, wkv_b[:, :128])   (595)
 *       scores   (einsum(q_lat, kv_cache) + einsum(q_pe, pe_cache)) * scale  (596-597)
 *       mask     -inf except at topk_indices, shared by all heads          (601-602)
 *       softmax  over key positions                                        (604)
 *       mix      x = einsum("bsht,btc->bshc", scores, kv_cache)            (605)
 *       value-up x = einsum("bshc,hdc->bshd", x, wkv_b[:, -128:])          (606)
 *   - "Softmax": A = exp(S~) / sum_u exp(S~), in the scores' own type;
 *   - "Apply value weights": O_i = O~_i W_UV,i, and A(c W_UV) = (A c) W_UV.
 *
 * Fixed dimensions (the pages' model): 128 heads, q_nope 128, q_pe 64,
 * latent 512, value 128; wkv_b is [128*256, 512] = view [128 heads, 256, 512],
 * rows 0..127 of a head are W_UK and rows 128..255 are W_UV.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE memory owned by the caller, row-major and
 *     contiguous, 16-byte aligned.  The library allocates nothing and keeps no
 *     state besides per-device cached launch attributes; it is reentrant.
 *   - "bf16" pointers hold IEEE bfloat16 values (passed as void*).
 *   - Work is enqueued on `stream` (0 = legacy default stream); no host
 *     synchronisation happens.  An argument error is returned BEFORE anything
 *     is launched.  A launch error returns MLA_ERR_CUDA.  Faults during
 *     execution appear at the caller's next synchronisation; a device wait
 *     that exceeds its time limit (2 s; a healthy wait lasts microseconds)
 *     writes MLA_ERR_DEVICE_TIMEOUT to *d_status (when d_status is not NULL)
 *     and the kernels return without hanging, leaving the output incomplete.
 *     With d_status NULL such a call cannot be told apart from a good one,
 *     so production callers should pass a status word and check it.
 *   - Index semantics: topk_idx[b, k] selects cache position t of batch row b
 *     when 0 <= t < min(end_pos[b], S_max); any other value (canonically -1)
 *     is padding and is skipped.  Valid indices of one row must be distinct
 *     (the indexer's top-k output is): the pages' mask scatters 0 into a -inf
 *     row, so a repeat selects a position once, but the kernels gather every
 *     listed entry and would count a repeat twice.  mla_check_topk_indices
 *     (or mla_set_index_checks) reports rows that break this.
 *     Index order is irrelevant.  A row with no valid index yields out = 0 and
 *     lse = -inf.
 *   - Batch row b reads cache slot b (the excerpt slices kv_cache[:bsz]);
 *     mla_sparse_prefill gives each row its slot explicitly.
 */
#ifndef MLA_SPARSE_DECODE_H
#define MLA_SPARSE_DECODE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_HEADS 128
#define MLA_D_NOPE 128
#define MLA_D_ROPE 64
#define MLA_D_LATENT 512
#define MLA_D_V 128

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, bad size        */
  MLA_ERR_WORKSPACE = 2,      /* workspace missing, misaligned or too small */
  MLA_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed       */
  MLA_ERR_DEVICE_TIMEOUT = 4, /* written to *d_status by a timed-out wait   */
  MLA_ERR_BAD_INDEX = 5,      /* written to *d_status: a repeated index     */
  MLA_ERR_UNSUPPORTED = 6     /* device is not sm_100                       */
} mla_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* mla_status_string(int status);

/* Number of key splits the decode uses for a batch of B rows with K index
 * slots per row on the current device (a pure function of B, K and the
 * device's SM count).  Returns 0 for invalid sizes. */
int mla_num_splits(int B, int K);

/* Bytes of scratch `mla_sparse_decode` needs for these sizes on the current
 * device: the absorbed queries (bf16 [B,128,512]), the per-split outputs of
 * mla_sparse_attend (see there: bf16 [B,splits,128,512]) and their
 * log-sum-exps (f32 [B,splits,128]).  Returns 0 for invalid sizes. */
size_t mla_sparse_decode_workspace_size(int B, int K, int S_max);

/*
 * The whole decode step (steps absorb .. value-up above).  Three kernels on
 * `stream`; the second and third are launched with a programmatic dependency
 * on the one before them (each starts early and waits for its predecessor
 * before reading that kernel's output), the first as an ordinary launch, so
 * work enqueued on `stream` before the call has finished before any of them
 * reads an input.
 *   q_nope   bf16 [B,128,128]   non-rotary queries
 *   q_pe     bf16 [B,128,64]    rotary queries, already rotated
 *   kv_cache bf16 [B,S_max,512] normalised latent cache c^KV
 *   pe_cache bf16 [B,S_max,64]  rotated shared rotary key k^R
 *   end_pos  int32 [B]          valid cache length of each row
 *   topk_idx int32 [B,K]        selected positions (see index semantics)
 *   wkv_b    bf16 [128*256,512]
 *   scale    softmax scale applied to the summed latent+rotary score
 *            (192^-0.5 for the pages' model, times mscale^2 when extended)
 *   out      bf16 [B,128,128]   per-head output before the output projection
 *   workspace / workspace_bytes  device scratch, 256-byte aligned, at least
 *            mla_sparse_decode_workspace_size(B, K, S_max) bytes
 *   lse_out  optional f32 [B,128]: natural-log sum of exp(scaled score) over
 *            the selected positions (NULL = not written)
 *   d_status optional device int: receives MLA_ERR_DEVICE_TIMEOUT if a device
 *            wait times out (NULL = not written; never cleared by the library)
 * Returns an mla_status.
 */
int mla_sparse_decode(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                      const int32_t* end_pos, const int32_t* topk_idx, const void* wkv_b, float scale, void* out,
                      int B, int K, int S_max, void* workspace, size_t workspace_bytes, float* lse_out,
                      int* d_status, cudaStream_t stream);

/*
 * Step "absorb" alone (model.py 595):
 *   q_lat[b,h,c] = bf16( sum_d q_nope[b,h,d] * wkv_b[h*256 + d, c] )
 *   q_nope bf16 [B,128,128], wkv_b bf16 [128*256,512], q_lat bf16 [B,128,512].
 */
int mla_absorb_q(const void* q_nope, const void* wkv_b, void* q_lat, int B, cudaStream_t stream);

/*
 * Steps "scores" .. "mix" for every (row, split) (model.py 596-605), the
 * key positions of row b being split into `n_split` contiguous ranges of index
 * slots:
 *   o_part           bf16 [B,n_split,128,512], o_part[b,s,h,:] = the
 *                    softmax-normalised mix of the cached latents over the
 *                    valid positions of split s, rounded to bf16; with
 *                    n_split == 1 ([B,128,512]) it is the mixed latent
 *                    O~[b,h,:] itself, the value-up operand
 *   lse_part[b,s,h]  f32 [B,n_split,128]      log-sum-exp of the split's
 *                    scaled scores (-inf when the split has no valid index)
 *   q_lat bf16 [B,128,512] (from mla_absorb_q), the other inputs as above.
 * n_split must equal mla_num_splits(B, K).
 */
int mla_sparse_attend(const void* q_lat, const void* q_pe, const void* kv_cache, const void* pe_cache,
                      const int32_t* end_pos, const int32_t* topk_idx, float scale, void* o_part,
                      float* lse_part, int B, int K, int S_max, int n_split, int* d_status, cudaStream_t stream);

/*
 * Steps "combine" and "value-up" (model.py 605-606), o_part and lse_part in
 * the layout mla_sparse_attend writes for this n_split:
 *   O~[b,h,:] = sum_s exp(lse_part[b,s,h] - L) o_part[b,s,h,:]   (in f32),
 *   L = log sum_s exp(lse_part[b,s,h])          (n_split > 1; with one split
 *                                                O~ = o_part, L = lse_part),
 *   out[b,h,e] = bf16( sum_c bf16(O~[b,h,c]) * wkv_b[h*256 + 128 + e, c] ),
 *   lse_out[b,h] = L (optional).
 */
int mla_combine_value_up(const void* o_part, const float* lse_part, const void* wkv_b, void* out,
                         float* lse_out, int B, int n_split, cudaStream_t stream);

/*
 * Index validation (the index mask of model.py 601-602 on the page "Query-key
 * similarity": a -inf row with 0 scattered at the selected positions, so each
 * position is selected at most once).  One CTA per row marks the row's valid
 * entries (0 <= t < min(end_pos[b], S_max); the rest is padding) in a bitmap
 * and finds any entry listed twice.
 *   end_pos, topk_idx  as in mla_sparse_decode (device, 16-byte aligned)
 *   d_status     optional device int: receives MLA_ERR_BAD_INDEX (if it still
 *                holds 0) when some row has a repeated valid entry
 *   d_row_flags  optional device int [B]: 1 for a row with a repeat, else 0
 * At least one of d_status, d_row_flags must be given.  Enqueued on `stream`;
 * reads B*K indices once per 1,048,576 positions of end_pos.  The decode
 * itself does not depend on the result.  Returns an mla_status.
 */
int mla_check_topk_indices(const int32_t* end_pos, const int32_t* topk_idx, int B, int K, int S_max,
                           int* d_status, int* d_row_flags, cudaStream_t stream);

/*
 * Opt-in debug mode for the whole process: with enable != 0, every call of
 * mla_sparse_decode, mla_sparse_prefill and the entry points built on them
 * (noalloc, host-buffer, decode + projection) that is given a d_status
 * first enqueues mla_check_topk_indices on its index rows, so a repeated
 * index ends up as MLA_ERR_BAD_INDEX in *d_status (the decode still runs).
 * Off by default; costs one extra kernel per call.  Returns the previous
 * setting.
 */
int mla_set_index_checks(int enable);

/*
 * Size of the library's fixed device scratch used by
 * mla_sparse_decode_noalloc (32 MiB, enough for B = 64 rows with K = 2048 on
 * a 148-SM device; mla_sparse_decode_workspace_size() tells the need).
 */
#define MLA_STATIC_SCRATCH_BYTES (32u << 20)

/*
 * The whole decode step without a workspace argument.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory when they call -- for example a plugin whose host framework
 * owns all device memory and offers it no allocation hook, or a serving loop
 * that must not call cudaMalloc, which can block and synchronise the device.
 * It allocates nothing: the scratch is a fixed device array of
 * MLA_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.
 *   - Arguments, layouts and results are those of mla_sparse_decode minus the
 *     workspace.
 *   - Sizes whose mla_sparse_decode_workspace_size() exceeds
 *     MLA_STATIC_SCRATCH_BYTES are rejected with MLA_ERR_WORKSPACE before
 *     anything is launched.
 *   - The first call on a device looks up the array's device address (a
 *     host-side CUDA runtime call, made with that device current); make that
 *     first call before any stream capture.
 *   - Every call shares the one array, and it keeps whatever the last call
 *     left there (nothing in it needs to start at zero): calls whose work
 *     overlaps on the GPU (different streams, or different host threads)
 *     race on it.  Serialise them, e.g. on one stream.
 */
int mla_sparse_decode_noalloc(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                              const int32_t* end_pos, const int32_t* topk_idx, const void* wkv_b, float scale,
                              void* out, int B, int K, int S_max, float* lse_out, int* d_status,
                              cudaStream_t stream);

/*
 * The whole decode step with the per-call tensors in HOST memory: the
 * queries, end positions and indices are read from, and the output written
 * to, host buffers; the caches and wkv_b (model state) stay in device memory.
 * The pages have no counterpart: this entry point exists for callers whose
 * per-token inputs live on the host (a serving process that has not placed
 * them on the device), so that one call covers upload, decode and read-back.
 *   h_q_nope, h_q_pe, h_end_pos, h_topk_idx, h_out: host memory, layouts as in
 *            mla_sparse_decode, 16-byte aligned; pinned (page-locked) memory
 *            makes the copies asynchronous, other host memory also works but
 *            the driver stages it
 *   kv_cache, pe_cache, wkv_b, lse_out, d_status: device memory, as in
 *            mla_sparse_decode
 *   workspace / workspace_bytes: device scratch, 256-byte aligned, at least
 *            mla_sparse_decode_host_workspace_size(B, K, S_max) bytes: the
 *            decode's scratch plus device copies of the four inputs and out
 * Enqueues on `stream`, in order: the uploads, the decode step, one
 * cudaMemcpyAsync of out to h_out.  The uploads are one cudaMemcpyAsync per
 * input, or a single one when the four inputs sit in one host buffer at the
 * offsets mla_sparse_decode_host_input_layout gives (the staging area's own
 * layout: fewer, larger copies run closer to the link's bandwidth).  h_out
 * is complete once `stream` has passed this point; the host buffers must stay
 * valid until then.  Consecutive calls overlap when they rotate between
 * streams, each with its own workspace.  Returns an mla_status.
 *
 * mla_sparse_decode_host_input_layout: byte offsets of h_q_nope, h_q_pe,
 * h_end_pos and h_topk_idx (offsets[0..3], offsets[0] = 0) in such a packed
 * host buffer, and its size as the return value (0 for invalid sizes);
 * offsets may be NULL.
 */
size_t mla_sparse_decode_host_input_layout(int B, int K, int S_max, size_t* offsets);
size_t mla_sparse_decode_host_workspace_size(int B, int K, int S_max);
int mla_sparse_decode_host(const void* h_q_nope, const void* h_q_pe, const int32_t* h_end_pos,
                           const int32_t* h_topk_idx, const void* kv_cache, const void* pe_cache, const void* wkv_b,
                           float scale, void* h_out, int B, int K, int S_max, void* workspace,
                           size_t workspace_bytes, float* lse_out, int* d_status, cudaStream_t stream);

/*
 * Sparse prefill (the "MHA prefill" branch, model.py 574-589, as shown on the
 * atlas page "Queries" in prefill mode): every query position s of a
 * sequence attends to the positions t of the same sequence that the indexer
 * selected for it and that the causal mask allows (t <= s):
 *   x[b,s,h,:] = sum_t softmax_t( scale * q[b,s,h] . k[b,t,h] ) v[b,t,h]
 * with k = [W_UK c_t ; k^R_t] and v = W_UV c_t.  The pages up-project every
 * latent into per-head keys and values; this entry point computes the same
 * result in the absorbed form of mla_sparse_decode (q . k = (q_nope W_UK) .
 * c_t + q_pe . k^R_t, and the mix of W_UV c_t is W_UV applied to the mix of
 * c_t), so a selected position costs one 1152-byte latent + rotary row
 * instead of 128 heads' keys and values.
 * Each of the R rows is one query position:
 *   q_nope, q_pe, out, lse_out, topk_idx  as in mla_sparse_decode with B = R
 *   kv_cache bf16 [n_slots,S_max,512], pe_cache bf16 [n_slots,S_max,64]: the
 *            latents of n_slots sequences (a prefill chunk: S_max = seqlen)
 *   cache_slot int32 [R]  the sequence of each row (16-byte aligned); a
 *            value outside [0, n_slots) gives the row no valid position
 *   end_pos  int32 [R]    the causal bound: s + 1 for the query at position s
 *            (positions t >= end_pos[r] are masked, as the causal mask does)
 *   workspace: mla_sparse_decode_workspace_size(R, K, S_max) bytes
 * For the pages' prefill of B sequences of seqlen positions:
 * R = B * seqlen, cache_slot[b*seqlen + s] = b, end_pos[b*seqlen + s] = s+1,
 * topk_idx[b*seqlen + s] = the indexer's selection for position s.
 * Returns an mla_status.
 */
int mla_sparse_prefill(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                       const int32_t* cache_slot, const int32_t* end_pos, const int32_t* topk_idx, const void* wkv_b,
                       float scale, void* out, int R, int K, int S_max, int n_slots, void* workspace,
                       size_t workspace_bytes, float* lse_out, int* d_status, cudaStream_t stream);

/*
 * Output projection (model.py 607-608 as shown on the atlas page "Attention
 * update": the head outputs of a row are flattened and projected back to the
 * model width by wo, a RowParallelLinear from 128*128 inputs to dim outputs;
 * the pages show no bias):
 *   delta[b, n] = bf16( sum_{k < 16384} x[b, k] * wo[n, k] )   (fp32 accumulate)
 *   x     bf16 [B, 16384]  the decode output [B,128,128] of mla_sparse_decode,
 *                          row-major (k = 128 h + e)
 *   wo    bf16 [dim, 16384] the torch Linear weight, k contiguous
 *   delta bf16 [B, dim]    Delta_attn of the pages ([B, 1, 7168] at dim 7168)
 *   dim   model width: a multiple of 128, 128 <= dim <= 65536 (7168 on the pages)
 *   workspace / workspace_bytes  device scratch, 256-byte aligned, at least
 *            mla_output_projection_workspace_size(B, dim) bytes (f32 partial
 *            sums; the result does not depend on its contents)
 *   d_status optional device int, as in mla_sparse_decode
 * Sizes: 1 <= B <= 2^20; wo is read once per 256 batch rows.  The sum over k
 * is split across SMs and added up in a fixed order, so results are
 * reproducible.  Enqueues two kernels on `stream` (an ordinary launch, then a
 * reduction with a programmatic dependency on it; with at least as many
 * 128 x 256 output tiles as SMs, one kernel).  Returns an mla_status.
 * mla_output_projection_workspace_size returns 0 only for invalid sizes.
 */
size_t mla_output_projection_workspace_size(int B, int dim);
int mla_output_projection(const void* x, const void* wo, void* delta, int B, int dim, void* workspace,
                          size_t workspace_bytes, int* d_status, cudaStream_t stream);

/*
 * The decode step followed by the output projection, in one call:
 * delta = mla_output_projection(mla_sparse_decode(...)).  Arguments as in the
 * two calls; the per-head outputs stay in the workspace, which must hold at
 * least mla_sparse_decode_project_workspace_size(B, K, S_max, dim) bytes
 * (256-byte aligned).  The projection kernel is launched with a programmatic
 * dependency on the value-up kernel, so its first wo stages are requested
 * while the decode finishes (wo must not be written by the decode's inputs'
 * producers in the meantime: it is model state).  Returns an mla_status.
 */
size_t mla_sparse_decode_project_workspace_size(int B, int K, int S_max, int dim);
int mla_sparse_decode_project(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                              const int32_t* end_pos, const int32_t* topk_idx, const void* wkv_b, float scale,
                              const void* wo, void* delta, int B, int K, int S_max, int dim, void* workspace,
                              size_t workspace_bytes, float* lse_out, int* d_status, cudaStream_t stream);

/*
 * fp8 weights (the decode excerpt on the page "Query-key similarity",
 * model.py 591-592: when wkv_b is stored in fp8 with a scale, the decode
 * first builds self.dequant_wkv_b = weight_dequant(wkv_b.weight, wkv_b.scale)
 * once and uses it in place of wkv_b from then on).  The pages do not print
 * the format; this entry point reads it as DeepSeek-V3's block format:
 *   w_fp8   OCP FP8 E4M3 codes [rows, cols] (1 byte each)
 *   scale   f32 [ceil(rows/128), ceil(cols/128)]: one scale per 128 x 128 block
 *   w_bf16  bf16 [rows, cols]:
 *           w_bf16[r,c] = bf16( e4m3(w_fp8[r,c]) * scale[r/128, c/128] ),
 *           the product exact and rounded once to nearest (ties to even)
 * For wkv_b: rows = 128*256 (n_heads*256 for a shard), cols = 512, scale
 * [256, 4].  The result is the bf16 wkv_b every decode entry point takes, so
 * a caller holding fp8 weights dequantises once, as the pages do, and keeps
 * the result.  cols must be a multiple of 16; w_fp8 and w_bf16 16-byte
 * aligned, scale 4-byte aligned.  Enqueued on `stream`.  Returns an
 * mla_status.
 */
int mla_dequant_fp8_blocks(const void* w_fp8, const float* scale, void* w_bf16, int rows, int cols,
                           cudaStream_t stream);

/*
 * Tensor parallelism, one shard (the MLA constructor excerpt on the page
 * "Queries", model.py 523-539: wkv_b is a ColumnParallelLinear, so a rank
 * holds n_local_heads = 128 / world_size heads and views its wkv_b rows as
 * [n_local_heads, 256, 512]; wo is a RowParallelLinear whose partial outputs
 * the ranks sum).  The decode step for n_heads consecutive heads:
 *   q_nope bf16 [B,n_heads,128], q_pe bf16 [B,n_heads,64]  the shard's heads
 *   wkv_b  bf16 [n_heads*256,512]  the shard's rows of wkv_b
 *   out    bf16 [B,n_heads,128],  lse_out f32 [B,n_heads] (optional)
 *   kv_cache, pe_cache, end_pos, topk_idx, scale: as in mla_sparse_decode
 *            (the latent cache and the index rows are shared by all heads,
 *            so every shard holds them whole)
 *   workspace: mla_sparse_decode_heads_workspace_size(B, K, S_max, n_heads)
 * 1 <= n_heads <= 128; with n_heads = 128 this is mla_sparse_decode.  The
 * attention kernel keeps the heads on the 128 lanes of its MMA tile: lanes
 * past n_heads carry a zero query and store nothing, so a shard's attention
 * costs as much as all 128 heads' (the weight-bound steps scale with
 * n_heads).  Returns an mla_status; the size function returns 0 for invalid
 * sizes.
 */
size_t mla_sparse_decode_heads_workspace_size(int B, int K, int S_max, int n_heads);
int mla_sparse_decode_heads(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                            const int32_t* end_pos, const int32_t* topk_idx, const void* wkv_b, float scale,
                            void* out, int B, int K, int S_max, int n_heads, void* workspace,
                            size_t workspace_bytes, float* lse_out, int* d_status, cudaStream_t stream);

/*
 * The row-parallel partial of the output projection (wo = RowParallelLinear
 * on the page "Queries"; the projection of the page "Attention update"):
 *   delta_r[b, n] = bf16( sum_{k < k_in} x[b, k] * wo[n, k] )   (fp32 accumulate)
 *   x      bf16 [B, k_in]    the shard's decode output [B,n_heads,128] flattened
 *   wo     bf16 rows of ld_wo elements (16-byte aligned, ld_wo a multiple of
 *          8 and >= k_in); columns [0, k_in) of each of the dim rows are used
 *   delta  bf16 [B, dim]
 *   k_in   a multiple of 64, 64 <= k_in <= 16384
 *   workspace: mla_output_projection_shard_workspace_size(B, dim, k_in)
 * For rank r of T ranks holding n_heads = 128 / T heads: x = its out,
 * wo = the full wo + r*n_heads*128 (ld_wo = 16384) or its own column slice
 * (ld_wo = k_in), k_in = n_heads*128.  Summing delta_r over the ranks (the
 * all-reduce after the RowParallelLinear) gives the projection of all heads;
 * with k_in = 16384 and ld_wo = 16384 this is mla_output_projection.
 * Returns an mla_status; the size function returns 0 for invalid sizes.
 */
size_t mla_output_projection_shard_workspace_size(int B, int dim, int k_in);
int mla_output_projection_shard(const void* x, const void* wo, long long ld_wo, void* delta, int B, int dim, int k_in,
                                void* workspace, size_t workspace_bytes, int* d_status, cudaStream_t stream);

/*
 * The output projection from a prepared copy of wo (the same projection as
 * mla_output_projection_shard, bit for bit).  Read in place, each work unit
 * of the projection touches 512 bytes in each of 128 rows of wo 32 KB apart;
 * the prepared copy holds every such unit's 64 KB contiguously, so the
 * weight stream runs closer to the HBM copy rate.  Prepare once per weight
 * (like the fp8 dequantisation of wkv_b), project every step:
 *   mla_prepare_wo(wo, ld_wo, dim, k_in, wo_prepared, stream)
 *     wo           bf16 rows of ld_wo elements (16-byte aligned, ld_wo a
 *                  multiple of 8 and >= k_in); columns [0, k_in) are used
 *     wo_prepared  device buffer of dim * k_in * 2 bytes, 16-byte aligned,
 *                  written in an internal layout (only the function below
 *                  reads it); enqueued on `stream`
 *     dim  a multiple of 128, 128 <= dim <= 65536
 *     k_in a multiple of 256, 256 <= k_in <= 16384
 *   mla_output_projection_prepared(x, wo_prepared, delta, B, dim, k_in, ...)
 *     x bf16 [B, k_in], delta bf16 [B, dim], workspace as
 *     mla_output_projection_shard_workspace_size(B, dim, k_in).
 * Both return an mla_status.
 */
int mla_prepare_wo(const void* wo, long long ld_wo, int dim, int k_in, void* wo_prepared, cudaStream_t stream);
int mla_output_projection_prepared(const void* x, const void* wo_prepared, void* delta, int B, int dim, int k_in,
                                   void* workspace, size_t workspace_bytes, int* d_status, cudaStream_t stream);

/*
 * Self-test of the bounded waits every kernel relies on (no counterpart on the
 * pages): launches one CTA whose thread waits, through the kernels' own wait,
 * on a barrier that nothing arrives on.  After the wait limit (2 s) it must
 * write MLA_ERR_DEVICE_TIMEOUT to *d_status (left unchanged if already
 * non-zero) and return; *d_result receives 4 when the wait gave up, set the
 * abort flag and a second wait returned at once (bit 0 / bit 1 set = a wait
 * wrongly reported completion).  d_status, d_result: device ints, 4-byte
 * aligned.  Takes about 2 s on the stream; the context stays usable.
 * Returns an mla_status (of the launch).
 */
int mla_selftest_wait_timeout(int* d_status, int* d_result, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_SPARSE_DECODE_H */

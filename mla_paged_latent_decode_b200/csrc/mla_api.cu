// mla_api.cu -- the extern "C" boundary declared in include/mla_decode.h.
//
// Host-side argument validation, TMA tensor-map construction (through the
// driver entry point, so the library links only the static CUDA runtime), and
// the launches of the scheduler, decode and combine kernels on the caller's
// stream.  Nothing here allocates device memory or synchronises.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <mutex>

#include "mla_kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
// Limit of each bounded wait inside the decode kernels (mla_set_wait_limit_ns).
std::atomic<uint64_t> g_wait_ns{mla::kWaitLimitNs};
// Test hook of the timeout path (mla_debug_set_stall_flag); normally null.
std::atomic<const int32_t*> g_stall_flag{nullptr};

int current_sm_count(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  int v = g_sm_count[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return MLA_ERR_CUDA;
    g_sm_count[dev].store(v, std::memory_order_relaxed);
  }
  *sms = v;
  return MLA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// A [rows, 576] bf16 row-major matrix read in (box_rows x 64) boxes with 128-byte swizzle.
bool make_row_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows = 64) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(mla::kDqk), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(mla::kDqk) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The fp32 partial outputs [slots, rows, 512] written in 32 x 32 boxes with
// 128-byte swizzle; the row extent clips boxes that run past a sequence's rows.
bool make_partial_map(CUtensorMap* map, float* base, uint64_t rows, uint64_t slots) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::kDv), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(slots)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kDv) * 4,
                           static_cast<cuuint64_t>(mla::kDv) * 4 * rows};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The bf16 output [batch, rows, 512] written in boxes of 32 rows x 64 columns
// (128 bytes per row) with 128-byte swizzle; the row extent clips boxes that run
// past a sequence's rows.
bool make_out_map(CUtensorMap* map, void* base, uint64_t rows, uint64_t batch) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::kDv), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kDv) * 2,
                           static_cast<cuuint64_t>(mla::kDv) * 2 * rows};
  cuuint32_t box[3] = {64, 32, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The cache viewed as 3-D {64 dims, rows, 9 chunks} (strides: a row is 1152
// bytes, a chunk 128): one box of box_rows rows x box_chunks 64-dim chunks lands
// in shared memory chunk after chunk, each chunk box_rows x 128 bytes with
// 128-byte swizzle, which is the layout the MMA descriptors read.  One TMA
// instruction then moves several chunks.
bool make_chunk_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows,
                    uint32_t box_chunks) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(mla::kDqk / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kDqk) * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_chunks};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The E4M3 cache as [rows, 576] bytes read in boxes of 128 bytes x 64 rows, no
// swizzle.  The decode starts the box for chunk c at x = 64 c - 64, so that
// chunk c lands in the upper 64 bytes of each 128-byte row slot (x < 0 is out
// of bounds and filled with zeros).
bool make_fp8_page_map(CUtensorMap* map, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(mla::kDqk), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(mla::kDqk)};
  cuuint32_t box[2] = {128, 64};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The E4M3 cache viewed as 3-D {128 bytes, rows, 9 chunks} with strides of 576
// bytes (a row) and 64 bytes (a chunk): element (x, r, c) is byte 64 c + x of
// row r.  A box of 128 x box_rows x box_chunks started at x = -64 lands, for
// each chunk, 64 zero bytes (x < 0 is out of bounds) and then the chunk's 64
// codes in each 128-byte row slot, chunk after chunk: the layout the pair
// kernel's converters widen, in one TMA instruction.  (x never reaches 64, so
// no element past a row is read.)
bool make_fp8_chunk_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows,
                        uint32_t box_chunks) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(mla::kDqk / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kDqk), 64};
  cuuint32_t box[3] = {128, box_rows, box_chunks};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Query rows up to 64 per sequence run on single CTAs (one 64-row block); more
// rows run on CTA pairs, one pair per 128-row block.
bool uses_pairs(int s_q, int h_q) { return static_cast<int64_t>(s_q) * h_q > mla::kRowsPerCta; }

int workers_for(int sms, int s_q, int h_q, int* out) {
  const int rows = s_q * h_q;
  if (!uses_pairs(s_q, h_q)) {
    *out = sms > 1 ? sms : 1;
    return MLA_OK;
  }
  const int blocks128 = (rows + 127) / 128;
  int clusters = 0;
  if (mla::pair_kernel_max_clusters(&clusters) != cudaSuccess) return MLA_ERR_CUDA;
  int w = sms / (2 * blocks128);
  const int w_fit = clusters / blocks128;  // every pair of the grid resident at once
  if (w_fit < w) w = w_fit;
  *out = w > 1 ? w : 1;
  return MLA_OK;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int launch_combine_for(const int32_t* num_splits, float* part_o, float* part_lse, void* out,
                       float* lse, int batch, int s_q, int h_q, int rows, cudaStream_t st);

// The decode after argument checks: scheduler metadata given, workspace large
// enough.  gather_rows != null: the rows of sequence s are cached rows
// gather_rows[s * gather_stride + k] (CTA pairs only; block_table unused).
int decode_impl(const void* q, const void* kcache, int64_t num_blocks, const int32_t* block_table,
                int bt_stride, const int32_t* cache_seqlens, int batch, int s_q, int h_q, int dv,
                float softmax_scale, int causal, const int32_t* tile_md, const int32_t* num_splits,
                int num_workers, void* workspace, void* out, float* lse, int32_t* device_status,
                void* stream, const int32_t* gather_rows, int64_t gather_stride) {
  const int rows = s_q * h_q;
  CUtensorMap tm_q;
  if (!make_row_map(&tm_q, q, static_cast<uint64_t>(batch) * rows)) return MLA_ERR_CUDA;
  const uint64_t cache_rows = static_cast<uint64_t>(num_blocks) * mla::kPage;

  const size_t slots = static_cast<size_t>(batch) + static_cast<size_t>(num_workers);
  float* part_o = static_cast<float*>(workspace);
  float* part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                             round_up(slots * rows * dv * sizeof(float), 256));

  mla::DecodeParams p{};
  p.block_table = block_table;
  p.seqlens = cache_seqlens;
  p.tile_md = tile_md;
  p.num_splits = num_splits;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.status = device_status;
  p.bt_stride = bt_stride;
  p.num_blocks = num_blocks;
  p.batch = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.rows = rows;
  p.causal = causal;
  p.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  p.stall_flag = g_stall_flag.load(std::memory_order_relaxed);
  p.gather_rows = gather_rows;
  p.gather_cache = kcache;
  p.gather_stride = gather_stride;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (uses_pairs(s_q, h_q)) {
    // K part: 32 token rows x all 9 chunks per box; peer-token values: 32 rows x 4
    // chunks (gathered rows are copied without these maps)
    CUtensorMap tm_kpart = tm_q, tm_vx = tm_q;
    if (gather_rows == nullptr) {
      if (!make_chunk_map(&tm_kpart, kcache, cache_rows, 32, mla::kDqk / 64)) return MLA_ERR_CUDA;
      if (!make_chunk_map(&tm_vx, kcache, cache_rows, 32, 4)) return MLA_ERR_CUDA;
    }
    CUtensorMap tm_po, tm_out;
    if (!make_partial_map(&tm_po, part_o, static_cast<uint64_t>(rows), slots)) return MLA_ERR_CUDA;
    if (!make_out_map(&tm_out, out, static_cast<uint64_t>(rows), static_cast<uint64_t>(batch)))
      return MLA_ERR_CUDA;
    if (mla::launch_decode_pair(tm_q, tm_kpart, tm_vx, tm_po, tm_out, p, num_workers, st) !=
        cudaSuccess)
      return MLA_ERR_CUDA;
  } else {
    // a whole page (64 rows x 9 chunks) per box (gathered rows are copied without it)
    CUtensorMap tm_page = tm_q;
    if (gather_rows == nullptr &&
        !make_chunk_map(&tm_page, kcache, cache_rows, 64, mla::kDqk / 64))
      return MLA_ERR_CUDA;
    if (mla::launch_decode(tm_q, tm_page, p, num_workers, st) != cudaSuccess) return MLA_ERR_CUDA;
  }

  return launch_combine_for(num_splits, part_o, part_lse, out, lse, batch, s_q, h_q, rows, st);
}

}  // namespace

extern "C" {

const char* mla_error_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK: success";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: invalid argument (null, size or alignment)";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: unsupported dimension";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA runtime call failed";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT: a device-side wait timed out";
    case MLA_ERR_DEVICE_CHECK: return "MLA_ERR_DEVICE_CHECK: a device-side bounds check failed";
    case MLA_ERR_SCRATCH_LIMIT:
      return "MLA_ERR_SCRATCH_LIMIT: workspace needed exceeds the library's static scratch "
             "(MLA_STATIC_SCRATCH_BYTES)";
    case MLA_ERR_NO_FREE_PAGES:
      return "MLA_ERR_NO_FREE_PAGES: too few free pages for an append, or no room on the free "
             "list for a release";
    default: return "unknown mla status";
  }
}

int mla_merge_partials(const void* outs, const float* lses, int num_parts, int batch, int s_q,
                       int h_q, void* out, float* lse, void* stream) {
  if (outs == nullptr || lses == nullptr || out == nullptr || lse == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (num_parts < 1 || num_parts > 4096 || batch < 1 || s_q < 1 || h_q < 1)
    return MLA_ERR_INVALID_ARG;
  const int64_t nrows = static_cast<int64_t>(batch) * s_q * h_q;
  if (static_cast<int64_t>(s_q) * h_q > 65536 || nrows * num_parts >= (int64_t(1) << 31))
    return MLA_ERR_INVALID_ARG;
  if (!aligned(outs, 16) || !aligned(out, 16) || !aligned(lses, 4) || !aligned(lse, 4))
    return MLA_ERR_INVALID_ARG;
  cudaError_t e = mla::launch_merge(outs, lses, num_parts, nrows, s_q, h_q, out, lse,
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

uint64_t mla_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) ns = mla::kWaitLimitNs;
  if (ns < 1000) ns = 1000;
  if (ns > mla::kWaitLimitNs) ns = mla::kWaitLimitNs;
  return g_wait_ns.exchange(ns);
}

const int32_t* mla_debug_set_stall_flag(const int32_t* device_flag) {
  return g_stall_flag.exchange(device_flag);
}

const char* mla_version(void) {
  return "mla_paged_latent_decode_b200 sm_100a (tcgen05 pair decode for >64 query rows, M=64 decode otherwise)";
}

int mla_metadata_shape(int batch, int h_q, int s_q, int* num_workers, int* md_stride) {
  if (batch < 1 || h_q < 1 || s_q < 1 || num_workers == nullptr || md_stride == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s_q) * h_q > 65536) return MLA_ERR_UNSUPPORTED;
  int sms = 0;
  int rc = current_sm_count(&sms);
  if (rc != MLA_OK) return rc;
  rc = workers_for(sms, s_q, h_q, num_workers);
  if (rc != MLA_OK) return rc;
  *md_stride = MLA_MD_STRIDE;
  return MLA_OK;
}

int mla_get_metadata(const int32_t* cache_seqlens, int batch, int h_q, int s_q,
                     int32_t* tile_md, int32_t* num_splits, int num_workers, void* stream) {
  if (cache_seqlens == nullptr || tile_md == nullptr || num_splits == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65536 || h_q < 1 || s_q < 1 || num_workers < 1 ||
      num_workers > (1 << 20))
    return MLA_ERR_INVALID_ARG;
  const int piece_cost = uses_pairs(s_q, h_q) ? MLA_SPLIT_PIECE_COST_PAIR : MLA_SPLIT_PIECE_COST_CTA;
  cudaError_t e = mla::launch_metadata(cache_seqlens, batch, num_workers, piece_cost, tile_md,
                                       num_splits, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

size_t mla_workspace_size(int batch, int s_q, int h_q, int dv, int num_workers) {
  if (batch < 1 || s_q < 1 || h_q < 1 || dv != mla::kDv || num_workers < 1) return 0;
  const size_t slots = static_cast<size_t>(batch) + static_cast<size_t>(num_workers);
  const size_t rows = static_cast<size_t>(s_q) * static_cast<size_t>(h_q);
  return round_up(slots * rows * dv * sizeof(float), 256) + round_up(slots * rows * sizeof(float), 256);
}

int mla_decode_kvcache(const void* q, const void* kcache, int64_t num_blocks,
                       const int32_t* block_table, int bt_stride,
                       const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                       int d, int dv, float softmax_scale, int causal,
                       const int32_t* tile_md, const int32_t* num_splits, int num_workers,
                       void* workspace, size_t workspace_bytes,
                       void* out, float* lse, int32_t* device_status, void* stream) {
  if (q == nullptr || kcache == nullptr || block_table == nullptr || cache_seqlens == nullptr ||
      tile_md == nullptr || num_splits == nullptr || out == nullptr || lse == nullptr ||
      workspace == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (d != mla::kDqk || dv != mla::kDv) return MLA_ERR_UNSUPPORTED;
  if (batch < 1 || s_q < 1 || h_q < 1 || bt_stride < 1 || num_workers < 1 ||
      num_workers > (1 << 20) || (causal != 0 && causal != 1))
    return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s_q) * h_q > 65536) return MLA_ERR_UNSUPPORTED;
  if (num_blocks < 1 || num_blocks * mla::kPage >= (int64_t(1) << 31)) return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch) * s_q * h_q >= (int64_t(1) << 31)) return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(out, 16) || !aligned(workspace, 256) ||
      !aligned(lse, 4))
    return MLA_ERR_INVALID_ARG;
  const size_t need = mla_workspace_size(batch, s_q, h_q, dv, num_workers);
  if (need == 0 || workspace_bytes < need) return MLA_ERR_INVALID_ARG;

  return decode_impl(q, kcache, num_blocks, block_table, bt_stride, cache_seqlens, batch, s_q,
                     h_q, dv, softmax_scale, causal, tile_md, num_splits, num_workers, workspace,
                     out, lse, device_status, stream, nullptr, 0);
}

int mla_decode_kvcache_fp8(const void* q, const void* kcache, const float* kscale,
                           int64_t num_blocks, const int32_t* block_table, int bt_stride,
                           const int32_t* cache_seqlens, int batch, int s_q, int h_q, int d,
                           int dv, float softmax_scale, int causal, const int32_t* tile_md,
                           const int32_t* num_splits, int num_workers, void* workspace,
                           size_t workspace_bytes, void* out, float* lse,
                           int32_t* device_status, void* stream) {
  if (q == nullptr || kcache == nullptr || kscale == nullptr || block_table == nullptr ||
      cache_seqlens == nullptr || tile_md == nullptr || num_splits == nullptr || out == nullptr ||
      lse == nullptr || workspace == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (d != mla::kDqk || dv != mla::kDv) return MLA_ERR_UNSUPPORTED;
  if (batch < 1 || s_q < 1 || h_q < 1 || bt_stride < 1 || num_workers < 1 ||
      num_workers > (1 << 20) || (causal != 0 && causal != 1))
    return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s_q) * h_q > 65536) return MLA_ERR_UNSUPPORTED;
  if (num_blocks < 1 || num_blocks * mla::kPage >= (int64_t(1) << 31)) return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch) * s_q * h_q >= (int64_t(1) << 31)) return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(kscale, 16) || !aligned(out, 16) ||
      !aligned(workspace, 256) || !aligned(lse, 4))
    return MLA_ERR_INVALID_ARG;
  const size_t need = mla_workspace_size(batch, s_q, h_q, dv, num_workers);
  if (need == 0 || workspace_bytes < need) return MLA_ERR_INVALID_ARG;

  const int rows = s_q * h_q;
  const bool pairs = uses_pairs(s_q, h_q);
  const uint64_t cache_rows = static_cast<uint64_t>(num_blocks) * mla::kPage;
  CUtensorMap tm_q, tm_page8 = {}, tm_k8 = {}, tm_v8 = {};
  if (!make_row_map(&tm_q, q, static_cast<uint64_t>(batch) * rows)) return MLA_ERR_CUDA;
  if (pairs) {
    // a CTA of a pair: its 32 tokens x 9 chunks, or 32 tokens x 4 chunks of values
    if (!make_fp8_chunk_map(&tm_k8, kcache, cache_rows, 32, mla::kDqk / 64) ||
        !make_fp8_chunk_map(&tm_v8, kcache, cache_rows, 32, 4))
      return MLA_ERR_CUDA;
  } else if (!make_fp8_page_map(&tm_page8, kcache, cache_rows)) {
    return MLA_ERR_CUDA;
  }
  const size_t slots = static_cast<size_t>(batch) + static_cast<size_t>(num_workers);
  float* part_o = static_cast<float*>(workspace);
  float* part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                             round_up(slots * rows * dv * sizeof(float), 256));
  mla::DecodeParams p{};
  p.block_table = block_table;
  p.seqlens = cache_seqlens;
  p.tile_md = tile_md;
  p.num_splits = num_splits;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.status = device_status;
  p.kscale = kscale;
  p.bt_stride = bt_stride;
  p.num_blocks = num_blocks;
  p.batch = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.rows = rows;
  p.causal = causal;
  p.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  p.stall_flag = g_stall_flag.load(std::memory_order_relaxed);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (pairs) {
    CUtensorMap tm_po, tm_out;
    if (!make_partial_map(&tm_po, part_o, static_cast<uint64_t>(rows), slots)) return MLA_ERR_CUDA;
    if (!make_out_map(&tm_out, out, static_cast<uint64_t>(rows), static_cast<uint64_t>(batch)))
      return MLA_ERR_CUDA;
    if (mla::launch_decode_pair_fp8(tm_q, tm_k8, tm_v8, tm_po, tm_out, p, num_workers, st) !=
        cudaSuccess)
      return MLA_ERR_CUDA;
  } else if (mla::launch_decode_fp8(tm_q, tm_page8, p, num_workers, st) != cudaSuccess) {
    return MLA_ERR_CUDA;
  }
  return launch_combine_for(num_splits, part_o, part_lse, out, lse, batch, s_q, h_q, rows, st);
}

size_t mla_sparse_workspace_size(int batch, int s_q, int h_q, int topk, int num_workers) {
  if (batch < 1 || s_q < 1 || h_q < 1 || topk < 1 || num_workers < 1) return 0;
  const size_t pos = static_cast<size_t>(batch) * s_q;
  const size_t dec = mla_workspace_size(static_cast<int>(pos), 1, h_q, mla::kDv, num_workers);
  if (dec == 0) return 0;
  return round_up(pos * topk * 4, 256) + round_up(pos * 4, 256) +
         round_up(static_cast<size_t>(num_workers) * MLA_MD_STRIDE * 4, 256) +
         round_up((pos + 1) * 4, 256) + round_up(pos * h_q * 4, 256) + dec;
}

int mla_decode_sparse(const void* q, const void* kcache, int64_t num_blocks,
                      const int32_t* block_table, int bt_stride, const int32_t* cache_seqlens,
                      int batch, int s_q, int h_q, int d, int dv, const int32_t* indices,
                      int topk, float softmax_scale, int causal, int num_workers,
                      void* workspace, size_t workspace_bytes, void* out, float* lse,
                      int32_t* device_status, void* stream) {
  if (q == nullptr || kcache == nullptr || block_table == nullptr || cache_seqlens == nullptr ||
      indices == nullptr || workspace == nullptr || out == nullptr || lse == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (d != mla::kDqk || dv != mla::kDv) return MLA_ERR_UNSUPPORTED;
  if (batch < 1 || s_q < 1 || h_q < 1 || bt_stride < 1 || topk < 1 || topk > 65536 ||
      num_workers < 1 || num_workers > (1 << 20) || (causal != 0 && causal != 1))
    return MLA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(h_q) > 65536) return MLA_ERR_UNSUPPORTED;
  if (num_blocks < 1 || num_blocks * mla::kPage >= (int64_t(1) << 31)) return MLA_ERR_INVALID_ARG;
  const int64_t pos = static_cast<int64_t>(batch) * s_q;
  const int64_t ppp = (topk + mla::kPage - 1) / mla::kPage;
  if (pos > 65536 || pos * topk >= (int64_t(1) << 31) || pos * h_q >= (int64_t(1) << 31))
    return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(out, 16) || !aligned(workspace, 256) ||
      !aligned(lse, 4))
    return MLA_ERR_INVALID_ARG;
  const size_t need = mla_sparse_workspace_size(batch, s_q, h_q, topk, num_workers);
  if (need == 0 || workspace_bytes < need) return MLA_ERR_INVALID_ARG;

  char* w = static_cast<char*>(workspace);
  auto take = [&w](size_t bytes) {
    char* r = w;
    w += round_up(bytes, 256);
    return r;
  };
  mla::SparseParams sp{};
  sp.indices = indices;
  sp.seqlens = cache_seqlens;
  sp.block_table = block_table;
  sp.comp = reinterpret_cast<int32_t*>(take(static_cast<size_t>(pos) * topk * 4));
  sp.counts = reinterpret_cast<int32_t*>(take(static_cast<size_t>(pos) * 4));
  int32_t* tile_md = reinterpret_cast<int32_t*>(take(static_cast<size_t>(num_workers) * MLA_MD_STRIDE * 4));
  int32_t* num_splits = reinterpret_cast<int32_t*>(take(static_cast<size_t>(pos + 1) * 4));
  float* lse_pos = reinterpret_cast<float*>(take(static_cast<size_t>(pos) * h_q * 4));
  void* dec_ws = take(mla_workspace_size(static_cast<int>(pos), 1, h_q, mla::kDv, num_workers));
  sp.status = device_status;
  sp.bt_stride = bt_stride;
  sp.num_blocks = num_blocks;
  sp.batch = batch;
  sp.s_q = s_q;
  sp.topk = topk;
  sp.causal = causal;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (mla::launch_sparse_prepare(sp, st) != cudaSuccess) return MLA_ERR_CUDA;
  int rc = mla_get_metadata(sp.counts, static_cast<int>(pos), h_q, 1, tile_md, num_splits,
                            num_workers, stream);
  if (rc != MLA_OK) return rc;
  // the decode over b * s_q sequences (one query position each) whose rows the
  // decode kernel copies itself, by index, from the cache
  float* lse_dst = s_q > 1 ? lse_pos : lse;
  rc = decode_impl(q, kcache, num_blocks, sp.comp, static_cast<int>(ppp), sp.counts,
                   static_cast<int>(pos), 1, h_q, dv, softmax_scale, 0, tile_md, num_splits,
                   num_workers, dec_ws, out, lse_dst, device_status, stream, sp.comp, topk);
  if (rc != MLA_OK) return rc;
  if (s_q > 1 && mla::launch_sparse_lse(lse_pos, lse, batch, s_q, h_q, st) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

}  // extern "C"

namespace {
// The split combine after either decode kernel (it has work only where a
// sequence has more than one piece).
int launch_combine_for(const int32_t* num_splits, float* part_o, float* part_lse, void* out,
                       float* lse, int batch, int s_q, int h_q, int rows, cudaStream_t st) {
  mla::CombineParams c{};
  c.num_splits = num_splits;
  c.part_o = part_o;
  c.part_lse = part_lse;
  c.out = static_cast<__nv_bfloat16*>(out);
  c.lse = lse;
  c.batch = batch;
  c.s_q = s_q;
  c.h_q = h_q;
  c.rows = rows;
  if (mla::launch_combine(c, st) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}
}  // namespace

// mla_kernels.cuh -- parameter blocks and launch entry points shared by the
// C-ABI layer (mla_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mla_decode.h"

namespace mla {

constexpr int kPage = MLA_PAGE_SIZE;      // tokens per page
constexpr int kDqk = MLA_HEAD_DIM_QK;     // 576
constexpr int kDv = MLA_HEAD_DIM_V;       // 512
constexpr int kRowsPerCta = MLA_ROWS_PER_CTA;
constexpr int kMdStride = MLA_MD_STRIDE;

// Bounded device waits give up after this long (then report MLA_ERR_DEVICE_TIMEOUT).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct DecodeParams {
  const int32_t* block_table;
  const int32_t* seqlens;
  const int32_t* tile_md;
  const int32_t* num_splits;
  __nv_bfloat16* out;   // [b, s_q, h_q, 512]
  float* lse;           // [b, h_q, s_q]
  float* part_o;        // [pieces, rows, 512]
  float* part_lse;      // [pieces, rows]
  int32_t* status;      // nullable
  const float* kscale;  // FP8 cache only: [num_blocks * 64] per-token scales
  int64_t bt_stride;
  int64_t num_blocks;
  int batch, s_q, h_q, rows;  // rows = s_q * h_q
  int causal;
  float scale_log2;     // softmax_scale * log2(e)
  uint64_t wait_ns;     // limit of each bounded device wait (kWaitLimitNs unless lowered
                        // through mla_set_wait_limit_ns)
  const int32_t* stall_flag;  // test hook, normally null: when set, the PV issuer waits
                              // for it to become non-zero before its first PV
  // Gathered rows (sparse decode on CTA pairs): token k of sequence s is cached
  // row gather_rows[s * gather_stride + k] of gather_cache [rows, 576] bf16;
  // null for the dense decode, which reads pages through the block table.
  const int32_t* gather_rows;
  const void* gather_cache;
  int64_t gather_stride;
};

struct CombineParams {
  const int32_t* num_splits;
  const float* part_o;
  const float* part_lse;
  __nv_bfloat16* out;
  float* lse;
  int batch, s_q, h_q, rows;
};

// Append of new tokens' rows to the paged cache (mla_paged_cache.cu).
struct AppendParams {
  const uint4* rows;          // [batch, s_new, 576] bf16 as 72 16-byte vectors per row
  uint4* kcache;              // [num_blocks * 64, 576] bf16, likewise (bf16 cache)
  uint8_t* kcache8;           // [num_blocks * 64, 576] E4M3 codes (FP8 cache)
  float* kscale;              // [num_blocks * 64] per-token scales (FP8 cache)
  int32_t* block_table;       // [batch, bt_stride]
  const int32_t* seqlens;     // [batch], read by both kernels
  int32_t* seqlens_rw;        // the same array, written by the commit kernel only
  const int32_t* free_pages;  // [free_capacity]
  const int32_t* free_count;  // [1], read by both kernels
  int32_t* free_count_rw;     // the same word, written by the commit kernel only
  int32_t* status;            // nullable
  int64_t num_blocks;
  int64_t bt_stride;
  int batch, s_new, free_capacity;
  int seqs_per_cta, tokens_per_cta;  // set by launch_append
};

struct ReleaseParams {
  const int32_t* release_mask;  // [batch], nonzero = release
  const int32_t* block_table;   // [batch, bt_stride]
  int32_t* seqlens;             // [batch]
  int32_t* free_pages;          // [free_capacity]
  int32_t* free_count;          // [1]
  int32_t* status;              // nullable
  int64_t bt_stride;
  int batch, free_capacity;
};

// Sparse decode: compaction of the used index entries into cached rows (mla_sparse.cu).
struct SparseParams {
  const int32_t* indices;      // [batch * s_q, topk]
  const int32_t* seqlens;      // [batch]
  const int32_t* block_table;  // [batch, bt_stride]
  int32_t* comp;               // workspace [batch * s_q, topk]: cached rows of the used
                               // entries, in list order
  int32_t* counts;             // workspace [batch * s_q]
  int32_t* status;             // nullable
  int64_t bt_stride, num_blocks;
  int batch, s_q, topk, causal;
};

// Launchers (return cudaGetLastError() of their launch).
cudaError_t launch_sparse_prepare(const SparseParams& p, cudaStream_t stream);
cudaError_t launch_sparse_lse(const float* lse_pos, float* lse, int batch, int s_q, int h_q,
                              cudaStream_t stream);
cudaError_t launch_append(const AppendParams& p, bool fp8, cudaStream_t stream);
cudaError_t launch_release(const ReleaseParams& p, cudaStream_t stream);
cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_workers, int piece_cost,
                            int32_t* tile_md, int32_t* num_splits, cudaStream_t stream);
// Single-CTA kernel (up to 64 query rows per sequence; more rows run as several
// 64-row blocks).  With p.gather_rows set, each page's rows are copied by index
// from p.gather_cache (tm_page is not read).
cudaError_t launch_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_page,
                          const DecodeParams& p, int num_workers, cudaStream_t stream);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);
// FP8 (E4M3) cache on single CTAs (one CTA per worker and 64-row block):
// tm_page8 views the codes as [rows, 576] bytes in boxes of 128 bytes x 64
// rows; scales via p.kscale.
cudaError_t launch_decode_fp8(const CUtensorMap& tm_q, const CUtensorMap& tm_page8,
                              const DecodeParams& p, int num_workers, cudaStream_t stream);
// Pair kernel (more than 64 query rows per sequence): clusters of 2 CTAs.
// With p.gather_rows set, the K and V parts are copied row by row from
// p.gather_cache (tm_kpart and tm_vx are not read).
cudaError_t launch_decode_pair(const CUtensorMap& tm_q, const CUtensorMap& tm_kpart,
                               const CUtensorMap& tm_vx, const CUtensorMap& tm_po,
                               const CUtensorMap& tm_out, const DecodeParams& p, int num_workers,
                               cudaStream_t stream);
// The pair kernel over an FP8 (E4M3) cache: tm_k8 and tm_v8 view the codes as
// {128 bytes, rows, 9 chunks} with a 64-byte chunk stride, in boxes of 32 rows
// x 9 and x 4 chunks (started at x = -64); scales via p.kscale.
cudaError_t launch_decode_pair_fp8(const CUtensorMap& tm_q, const CUtensorMap& tm_k8,
                                   const CUtensorMap& tm_v8, const CUtensorMap& tm_po,
                                   const CUtensorMap& tm_out, const DecodeParams& p,
                                   int num_workers, cudaStream_t stream);
cudaError_t pair_kernel_max_clusters(int* clusters);
// Merge of decode results over disjoint parts of the cache (mla_merge.cu):
// outs [parts, nrows, 512] bf16, lses [parts, b, h_q, s_q] fp32.
cudaError_t launch_merge(const void* outs, const float* lses, int parts, int64_t nrows, int s_q,
                         int h_q, void* out, float* lse, cudaStream_t stream);

}  // namespace mla

// mla_sparse.cu -- sparse (top-k) decode given token indices.
//
// Dynamic sparse attention restricts each query to the most relevant cached
// tokens, reached by gathering them ("Boosting DeepSeek V3.2: Faster LLM
// Inference With FlashMLA", the paragraph on Dynamic Sparse Attention).  The
// selection is an input: indices[b][s_q][topk] lists logical token positions,
// shared by every head of a query position.  An entry is used when it lies in
// [0, L_i) and, with causal, at or before L_i - s_q + j; each used entry is one
// term.  Over the used entries the result is the dense decode's.
//
// This path is built from the dense decode: each query position (i, j) becomes
// a sequence of its own whose tokens are its used entries, in list order.
//   1. mla_sparse_compact_kernel: one CTA per query position keeps the used
//      entries (an ordered block compaction) and writes their count and an
//      identity block-table row over the position's pages in the workspace.
//   2. mla_sparse_gather_kernel: copies each used entry's cached row, through
//      the sequence's block table, into those pages; rows past the count in a
//      position's last page are zeroed (never read as data, but never NaN).
//   3. the scheduler, decode and combine kernels of the dense decode on the
//      gathered pages (b * s_q sequences, one query position each);
//   4. mla_sparse_lse_kernel (s_q > 1): lse from [b * s_q, h_q] to [b, h_q, s_q].
// The gather reads and writes each selected row once more than a decode that
// gathered in its own producer would.
#include "mla_kernels.cuh"

namespace mla {
namespace {

constexpr int kCompactThreads = 256;
constexpr int kGatherThreads = 256;
constexpr int kVecs = kDqk * 2 / 16;  // 72 16-byte vectors per cached row

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__global__ void __launch_bounds__(kCompactThreads)
mla_sparse_compact_kernel(SparseParams p) {
  __shared__ int warp_tot[kCompactThreads / 32];
  __shared__ int base;
  const int qp = blockIdx.x;  // query position i * s_q + j
  const int i = qp / p.s_q, j = qp - i * p.s_q;
  const int L = p.seqlens[i];
  int limit = p.causal ? L - p.s_q + j + 1 : L;
  if (limit > L) limit = L;
  const int32_t* idx = p.indices + static_cast<int64_t>(qp) * p.topk;
  int32_t* comp = p.comp + static_cast<int64_t>(qp) * p.topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  for (int e0 = 0; e0 < p.topk; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    const int t = e < p.topk ? idx[e] : -1;
    const bool used = t >= 0 && t < limit;
    const unsigned ballot = __ballot_sync(0xffffffffu, used);
    if (lane == 0) warp_tot[warp] = __popc(ballot);
    __syncthreads();
    int before = base;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    if (used) comp[before + __popc(ballot & ((1u << lane) - 1u))] = t;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += warp_tot[w];
      base += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) p.counts[qp] = base;
  for (int g = threadIdx.x; g < p.pages_per_pos; g += blockDim.x)
    p.comp_bt[static_cast<int64_t>(qp) * p.pages_per_pos + g] = qp * p.pages_per_pos + g;
}

__global__ void __launch_bounds__(kGatherThreads)
mla_sparse_gather_kernel(SparseParams p) {
  __shared__ int64_t src_row[kPage];  // cached row of each tile row, -1 = zero row
  const int qp = blockIdx.x, g = blockIdx.y;
  if (g >= p.pages_per_pos) return;
  const int count = p.counts[qp];
  if (g * kPage >= count && !(count == 0 && g == 0)) return;  // page never read
  const int i = qp / p.s_q;
  const int32_t* bt = p.block_table + static_cast<int64_t>(i) * p.bt_stride;
  const int32_t* comp = p.comp + static_cast<int64_t>(qp) * p.topk;
  if (threadIdx.x < kPage) {
    const int k = g * kPage + threadIdx.x;
    int64_t row = -1;
    if (k < count) {
      const int t = comp[k];
      const int lp = t / kPage;
      const int page = lp < p.bt_stride ? bt[lp] : -1;
      if (page >= 0 && page < p.num_blocks)
        row = static_cast<int64_t>(page) * kPage + t % kPage;
      else
        report(p.status, MLA_ERR_DEVICE_CHECK);
    }
    src_row[threadIdx.x] = row;
  }
  __syncthreads();
  const uint4* src = static_cast<const uint4*>(p.kcache);
  uint4* dst = reinterpret_cast<uint4*>(p.comp_cache) +
               (static_cast<int64_t>(qp) * p.pages_per_pos + g) * kPage * kVecs;
  for (int v0 = threadIdx.x; v0 < kPage * kVecs; v0 += 4 * blockDim.x) {
    uint4 buf[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * static_cast<int>(blockDim.x);
      buf[u] = make_uint4(0u, 0u, 0u, 0u);
      if (v < kPage * kVecs) {
        const int64_t row = src_row[v / kVecs];
        if (row >= 0) buf[u] = __ldg(src + row * kVecs + v % kVecs);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * static_cast<int>(blockDim.x);
      if (v < kPage * kVecs) dst[v] = buf[u];
    }
  }
}

__global__ void mla_sparse_lse_kernel(const float* lse_pos, float* lse, int batch, int s_q,
                                      int h_q) {
  const int64_t n = static_cast<int64_t>(batch) * s_q * h_q;
  for (int64_t x = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; x < n;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t qp = x / h_q;          // source [b * s_q, h_q]
    const int h = static_cast<int>(x - qp * h_q);
    const int64_t i = qp / s_q;
    const int j = static_cast<int>(qp - i * s_q);
    lse[(i * h_q + h) * s_q + j] = lse_pos[x];
  }
}

}  // namespace

cudaError_t launch_sparse_prepare(const SparseParams& p, cudaStream_t stream) {
  const int positions = p.batch * p.s_q;
  mla_sparse_compact_kernel<<<positions, kCompactThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mla_sparse_gather_kernel<<<dim3(positions, p.pages_per_pos), kGatherThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_sparse_lse(const float* lse_pos, float* lse, int batch, int s_q, int h_q,
                              cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(batch) * s_q * h_q;
  int blocks = static_cast<int>((n + 255) / 256);
  if (blocks > 4096) blocks = 4096;
  mla_sparse_lse_kernel<<<blocks, 256, 0, stream>>>(lse_pos, lse, batch, s_q, h_q);
  return cudaGetLastError();
}

}  // namespace mla

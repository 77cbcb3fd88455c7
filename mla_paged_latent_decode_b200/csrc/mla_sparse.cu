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
// Each query position (i, j) becomes a sequence of its own whose tokens are its
// used entries, in list order.
//   1. mla_sparse_compact_kernel: one CTA per query position keeps the used
//      entries (an ordered block compaction) and writes, for each, its cached
//      row (through the sequence's block table), and their count.
//   2. the scheduler, decode and combine kernels over b * s_q sequences, one
//      query position each; the decode kernel's producer copies the listed
//      rows itself (its gather mode), so each selected row leaves HBM once;
//   3. mla_sparse_lse_kernel (s_q > 1): lse from [b * s_q, h_q] to [b, h_q, s_q].
#include "mla_kernels.cuh"

namespace mla {
namespace {

constexpr int kCompactThreads = 256;

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
  const int32_t* bt = p.block_table + static_cast<int64_t>(i) * p.bt_stride;
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
    if (used) {
      // the token's cached row, through the sequence's block table; a page
      // outside the cache is reported and marked -1 (the decode reads zeros)
      const int lp = t / kPage;
      const int page = lp < p.bt_stride ? bt[lp] : -1;
      int row = -1;
      if (page >= 0 && page < p.num_blocks)
        row = page * kPage + t % kPage;
      else
        report(p.status, MLA_ERR_DEVICE_CHECK);
      comp[before + __popc(ballot & ((1u << lane) - 1u))] = row;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += warp_tot[w];
      base += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) p.counts[qp] = base;
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

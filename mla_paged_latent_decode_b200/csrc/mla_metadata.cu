// mla_metadata.cu -- the length-balanced split-KV tile scheduler.
//
// Rule (stated in include/mla_decode.h, mla_get_metadata): sequence i owns
// items_i = max(ceil(L_i / 64), 1) items and costs P + items_i units, P the
// per-sequence cost of the decode kernel the rows select; laid end to end, its
// item j sits at unit start_i + P + j, and the item at unit u belongs to worker
// u / cap with cap = ceil(total / W).  Exception: with batch <= W and every
// sequence costing at most cap + 2 P units, worker i takes sequence i whole.
//
// One CTA computes it with two block-wide scans (unit starts, then pieces per
// sequence); each thread owns a contiguous chunk of sequences and writes the
// worker rows whose first or last item falls in one of them.
#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kMdThreads = 256;
// Up to this many workers, the rows are assembled in shared memory and written
// out once; beyond it they are assembled in place in global memory.
constexpr int kSmemWorkers = 1024;

// Exclusive scan of one int64 per thread across the block; also returns the total.
__device__ int64_t block_exclusive_scan(int64_t v, int64_t* warp_sums, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int64_t w = lane < nw ? warp_sums[lane] : 0;
    int64_t winc = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t n = __shfl_up_sync(0xffffffffu, winc, o);
      if (lane >= o) winc += n;
    }
    if (lane < nw) warp_sums[lane] = winc - w;  // exclusive prefix of warp totals
    if (lane == nw - 1) *total = winc;
  }
  __syncthreads();
  const int64_t r = warp_sums[warp] + inc - v;
  __syncthreads();
  return r;
}

// Maximum of one int64 per thread across the block.
__device__ int64_t block_max(int64_t v, int64_t* warp_vals) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const int64_t n = __shfl_xor_sync(0xffffffffu, v, o);
    v = n > v ? n : v;
  }
  if (lane == 0) warp_vals[warp] = v;
  __syncthreads();
  int64_t m = warp_vals[0];
  for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) m = warp_vals[w] > m ? warp_vals[w] : m;
  __syncthreads();
  return m;
}

__device__ __forceinline__ int64_t items_of(int32_t L) {
  const int64_t n = L > 0 ? (static_cast<int64_t>(L) + kPage - 1) / kPage : 0;
  return n > 0 ? n : 1;
}

__global__ void __launch_bounds__(kMdThreads)
mla_metadata_kernel(const int32_t* __restrict__ seqlens, int batch, int num_workers, int piece_cost,
                    int32_t* __restrict__ tile_md_global, int32_t* __restrict__ num_splits) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t total_units, total_pieces;
  __shared__ int32_t srows[kSmemWorkers * kMdStride];
  const bool in_smem = num_workers <= kSmemWorkers;
  int32_t* tile_md = in_smem ? srows : tile_md_global;
  grid_dependency_wait();     // the lengths may come from the previous kernel
  grid_launch_dependents();   // the decode may be scheduled; it waits for this grid
  const int tid = threadIdx.x;
  const int chunk = (batch + blockDim.x - 1) / blockDim.x;
  const int i0 = min(batch, tid * chunk), i1 = min(batch, i0 + chunk);

  for (int k = tid; k < num_workers * kMdStride; k += blockDim.x) tile_md[k] = 0;
  if (in_smem) __syncthreads();

  // pass 1: unit starts
  int64_t my_units = 0;
  for (int i = i0; i < i1; ++i) my_units += piece_cost + items_of(seqlens[i]);
  const int64_t my_start = block_exclusive_scan(my_units, warp_sums, &total_units);
  __syncthreads();
  const int64_t total = total_units;
  const int64_t cap = total > 0 ? (total + num_workers - 1) / num_workers : 1;

  // Whole sequences: with no more sequences than workers, and no sequence
  // costing more than cap + 2 P units, worker i takes sequence i and nothing is
  // split (no partial outputs, nothing to merge).
  int64_t my_max = 0;
  for (int i = i0; i < i1; ++i) {
    const int64_t u = piece_cost + items_of(seqlens[i]);
    my_max = u > my_max ? u : my_max;
  }
  const int64_t umax = block_max(my_max, warp_sums);
  if (batch <= num_workers && umax <= cap + 2 * static_cast<int64_t>(piece_cost)) {
    if (tid == 0) num_splits[0] = 0;
    for (int i = i0; i < i1; ++i) {
      int32_t* row = tile_md + static_cast<int64_t>(i) * kMdStride;
      row[0] = i;
      row[1] = 0;
      row[2] = i;
      row[3] = static_cast<int32_t>(items_of(seqlens[i]));
      row[4] = 0;
      row[5] = 1;
      num_splits[i + 1] = i + 1;
    }
    if (in_smem) {
      __syncthreads();
      for (int k = tid; k < num_workers * kMdStride; k += blockDim.x) tile_md_global[k] = srows[k];
    }
    return;
  }

  // pass 2: pieces per sequence, and the worker rows that begin or end here
  int64_t my_pieces = 0;
  {
    int64_t s = my_start;
    for (int i = i0; i < i1; ++i) {
      const int64_t n = items_of(seqlens[i]);
      const int64_t f = s + piece_cost, g = f + n - 1;
      my_pieces += g / cap - f / cap + 1;
      s = g + 1;
    }
  }
  const int64_t my_first_piece = block_exclusive_scan(my_pieces, warp_sums, &total_pieces);
  if (tid == 0) num_splits[0] = 0;
  {
    int64_t s = my_start, pc = my_first_piece;
    for (int i = i0; i < i1; ++i) {
      const int64_t n = items_of(seqlens[i]);
      const int64_t f = s + piece_cost, g = f + n - 1;
      const int64_t w_first = f / cap, w_last = g / cap;
      pc += w_last - w_first + 1;
      num_splits[i + 1] = static_cast<int32_t>(pc);
      const int64_t next_first_item = g + 1 + piece_cost;  // first item unit of sequence i+1
      for (int64_t w = w_first; w <= w_last; ++w) {
        int32_t* row = tile_md + w * kMdStride;
        const int64_t lo = w * cap, hi = lo + cap;
        if (lo >= s) {  // no item of sequence i-1 lies in this worker: it begins here
          const int64_t j0 = lo > f ? lo - f : 0;
          row[0] = i;
          row[1] = static_cast<int32_t>(j0);
          row[4] = static_cast<int32_t>(w - w_first);
        }
        if (i == batch - 1 || next_first_item >= hi) {  // ... and it ends here
          const int64_t je = (hi - 1 - f) < (n - 1) ? (hi - 1 - f) : (n - 1);
          row[2] = i;
          row[3] = static_cast<int32_t>(je + 1);
        }
      }
      s = g + 1;
    }
  }
  __syncthreads();
  // pass 3: piece counts of the workers that own anything
  for (int w = tid; w < num_workers; w += blockDim.x) {
    int32_t* row = tile_md + static_cast<int64_t>(w) * kMdStride;
    const int64_t lo = static_cast<int64_t>(w) * cap;
    if (lo < total) {
      // a worker owns items iff some item unit lies in [lo, lo + cap); begin/end
      // rows were written above exactly for those workers
      if (row[3] > 0) row[5] = row[2] - row[0] + 1;
    }
  }
  if (in_smem) {  // one coalesced pass out
    __syncthreads();
    for (int k = tid; k < num_workers * kMdStride; k += blockDim.x) tile_md_global[k] = srows[k];
  }
}

}  // namespace

cudaError_t launch_metadata(const int32_t* seqlens, int batch, int num_workers, int piece_cost,
                            int32_t* tile_md, int32_t* num_splits, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kMdThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, mla_metadata_kernel, seqlens, batch, num_workers,
                                     piece_cost, tile_md, num_splits);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla

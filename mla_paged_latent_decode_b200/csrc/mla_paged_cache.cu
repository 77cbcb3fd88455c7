// mla_paged_cache.cu -- appending new tokens' latent rows to the paged cache,
// with 64-token pages taken from and given back to a free-page stack.
//
// After each decoding step the newest token's cached state joins the cache for
// later steps ("DeepSeek #OpenSourceWeek Day 1: Launch of FlashMLA", "How KV
// Caching Works?"); in MLA that state is one latent row per token ("How MLA
// Optimizes Memory Usage").  Pages are allocated on demand, so a sequence grows
// in 64-token increments, and a finished sequence's pages are released
// ("FlashMLA: Revolutionizing Efficient Decoding...", section 4.3.2).
//
// Free pages are the stack free_pages[0:free_count].  An append pops pages from
// the top, sequence after sequence in batch order; a release pushes pages back
// in the same order.
//
// The append runs as two kernels on the caller's stream:
//   1. mla_append_rows_kernel (a grid): every CTA computes, for its sequences,
//      how many pages the sequences before them take from the stack, copies its
//      rows into their pages with 16-byte loads and stores, and (token chunk 0)
//      writes the new block-table entries.  It reads the lengths and the free
//      count but writes neither; every write stays inside the buffers (a row or
//      entry whose page is out of range is skipped).
//   2. mla_append_commit_kernel (one CTA, a programmatic dependent of 1): checks
//      the whole request while kernel 1 copies, waits for kernel 1 to finish,
//      then grows every length by s_new and lowers the free count, or, if the
//      request is invalid, reports the reason and changes neither.  Rows that
//      kernel 1 wrote for a refused request lie in free pages or past a
//      sequence's length, and block-table entries past its pages: no reader
//      sees them.
// A release is one CTA: check, push, then zero the lengths and raise the count.
#include <cuda_fp8.h>

#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kVecsPerRow = kDqk * 2 / 16;  // 72 16-byte vectors per cached row
constexpr int kAppendThreads = 256;
constexpr int kMaxSeqsPerCta = 128;
constexpr int kMaxTokensPerCta = 32;
constexpr int kMaxRowsPerCta = kMaxSeqsPerCta * kMaxTokensPerCta;
constexpr int kCopyUnroll = 4;  // 16-byte loads in flight per thread
constexpr int kCommitThreads = 1024;

__device__ __forceinline__ int64_t pages_of(int64_t tokens) { return (tokens + kPage - 1) / kPage; }

// Pages sequence i takes from the free stack (0 for a negative length, which
// the commit kernel rejects).
__device__ __forceinline__ int64_t new_pages(int32_t L, int s_new) {
  if (L < 0) return 0;
  return pages_of(static_cast<int64_t>(L) + s_new) - pages_of(L);
}

template <typename Op>
__device__ int64_t block_reduce(int64_t v, int64_t* warp_vals, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) warp_vals[warp] = v;
  __syncthreads();
  int64_t r = warp_vals[0];
  for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) r = op(r, warp_vals[w]);
  __syncthreads();
  return r;
}

struct Sum {
  __device__ int64_t operator()(int64_t a, int64_t b) const { return a + b; }
};
struct Max {
  __device__ int64_t operator()(int64_t a, int64_t b) const { return a > b ? a : b; }
};

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// One row's E4M3 encoding, by one warp: lanes 0-23 hold 24 dims each.  The
// scale is the smallest 2^k with max|x| <= 448 * 2^k (k from the exponent of
// max|x|: max|x| = f * 2^e with f in [0.5, 1), k = e - 9 if f <= 0.875, else
// e - 8), and each code is x / 2^k rounded to nearest even, sign kept.
__device__ __forceinline__ void encode_row_e4m3(const uint4* src, uint8_t* dst_codes,
                                                float* dst_scale, int lane) {
  float x[24];
  float amax = 0.f;
  if (lane < 24) {
#pragma unroll
    for (int v = 0; v < 3; ++v) {
      const uint4 w = __ldg(src + 3 * lane + v);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        x[8 * v + 2 * h] = __uint_as_float(ws[h] << 16);
        x[8 * v + 2 * h + 1] = __uint_as_float(ws[h] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int c = 0; c < 24; ++c) amax = fmaxf(amax, fabsf(x[c]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int k = 0;
  if (amax > 0.f) {
    int e = 0;
    const float f = frexpf(amax, &e);
    k = f <= 0.875f ? e - 9 : e - 8;
  }
  if (lane < 24) {
    uint32_t packed[6];
#pragma unroll
    for (int q = 0; q < 6; ++q) {
      uint32_t word = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 pair = make_float2(ldexpf(x[4 * q + 2 * h], -k), ldexpf(x[4 * q + 2 * h + 1], -k));
        const uint32_t two = __nv_cvt_float2_to_fp8x2(pair, __NV_SATFINITE, __NV_E4M3);
        word |= (two & 0xFFFFu) << (16 * h);
      }
      packed[q] = word;
    }
    uint2* out = reinterpret_cast<uint2*>(dst_codes + 24 * lane);
    out[0] = make_uint2(packed[0], packed[1]);
    out[1] = make_uint2(packed[2], packed[3]);
    out[2] = make_uint2(packed[4], packed[5]);
  }
  if (lane == 0) *dst_scale = ldexpf(1.f, k);
}

template <bool kFp8>
__global__ void __launch_bounds__(kAppendThreads)
mla_append_rows_kernel(AppendParams p) {
  __shared__ int64_t warp_vals[32];
  __shared__ int32_t seq_len[kMaxSeqsPerCta];
  __shared__ int64_t seq_off[kMaxSeqsPerCta];
  __shared__ int32_t dst_row[kMaxRowsPerCta];
  // The commit kernel is a programmatic dependent: it may start checking now,
  // and writes only after this grid has finished.
  grid_launch_dependents();
  const int tid = threadIdx.x;
  const int s0 = blockIdx.x * p.seqs_per_cta;
  const int s1 = min(p.batch, s0 + p.seqs_per_cta);
  const int ns = s1 - s0;
  const int64_t fc = *p.free_count;
  const bool fc_ok = fc >= 0 && fc <= p.free_capacity;

  // this CTA's lengths, and the pages popped for the sequences before them
  for (int j = tid; j < ns; j += blockDim.x) seq_len[j] = p.seqlens[s0 + j];
  int64_t part = 0;
  for (int i = tid; i < s0; i += blockDim.x) part += new_pages(p.seqlens[i], p.s_new);
  const int64_t before = block_reduce(part, warp_vals, Sum());  // also publishes seq_len
  if (tid == 0) {
    int64_t off = before;
    for (int j = 0; j < ns; ++j) {
      seq_off[j] = off;
      off += new_pages(seq_len[j], p.s_new);
    }
  }
  __syncthreads();
  if (!fc_ok) return;  // the commit kernel reports it

  // new block-table entries (token chunk 0 writes them)
  if (blockIdx.y == 0) {
    for (int j = tid; j < ns; j += blockDim.x) {
      const int32_t L = seq_len[j];
      if (L < 0) continue;
      const int64_t first = pages_of(L);
      const int64_t k = new_pages(L, p.s_new);
      for (int64_t r = 0; r < k; ++r) {
        const int64_t slot = fc - 1 - (seq_off[j] + r);
        if (first + r >= p.bt_stride || slot < 0) break;
        const int32_t page = p.free_pages[slot];
        if (page < 0 || page >= p.num_blocks) continue;
        p.block_table[static_cast<int64_t>(s0 + j) * p.bt_stride + first + r] = page;
      }
    }
  }

  for (int k0 = blockIdx.y * p.tokens_per_cta; k0 < p.s_new;
       k0 += gridDim.y * p.tokens_per_cta) {
    const int nt = min(p.tokens_per_cta, p.s_new - k0);
    const int nrows = ns * nt;
    // destination row of each (sequence, token) of this chunk, -1 = skip
    for (int r = tid; r < nrows; r += blockDim.x) {
      const int j = r / nt;
      const int32_t L = seq_len[j];
      int32_t dst = -1;
      if (L >= 0) {
        const int64_t t = static_cast<int64_t>(L) + k0 + r % nt;
        const int64_t lp = t / kPage, first = pages_of(L);
        int64_t page = -1;
        if (lp < p.bt_stride) {
          if (lp < first) {
            page = p.block_table[static_cast<int64_t>(s0 + j) * p.bt_stride + lp];
          } else {
            const int64_t slot = fc - 1 - (seq_off[j] + lp - first);
            if (slot >= 0) page = p.free_pages[slot];
          }
        }
        // num_blocks * 64 < 2^31 (checked on the host), so the row index fits
        if (page >= 0 && page < p.num_blocks) dst = static_cast<int32_t>(page * kPage + t % kPage);
      }
      dst_row[r] = dst;
    }
    __syncthreads();
    if constexpr (kFp8) {
      // one warp per row: encode into codes and a per-token scale
      const int warp = tid >> 5, lane = tid & 31;
      for (int r = warp; r < nrows; r += blockDim.x >> 5) {
        const int32_t dst = dst_row[r];
        if (dst < 0) continue;
        const int64_t src = static_cast<int64_t>(s0 + r / nt) * p.s_new + k0 + r % nt;
        encode_row_e4m3(p.rows + src * kVecsPerRow, p.kcache8 + static_cast<int64_t>(dst) * kDqk,
                        p.kscale + dst, lane);
      }
      __syncthreads();
      continue;
    }
    // kCopyUnroll loads in flight per thread before their stores
    const int nvec = nrows * kVecsPerRow;
    for (int v0 = tid; v0 < nvec; v0 += blockDim.x * kCopyUnroll) {
      uint4 buf[kCopyUnroll];
      int64_t to[kCopyUnroll];
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int v = v0 + u * static_cast<int>(blockDim.x);
        to[u] = -1;
        if (v < nvec) {
          const int r = v / kVecsPerRow, c = v - r * kVecsPerRow;
          const int32_t dst = dst_row[r];
          if (dst >= 0) {
            const int64_t src = static_cast<int64_t>(s0 + r / nt) * p.s_new + k0 + r % nt;
            buf[u] = __ldg(p.rows + src * kVecsPerRow + c);
            to[u] = static_cast<int64_t>(dst) * kVecsPerRow + c;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u)
        if (to[u] >= 0) p.kcache[to[u]] = buf[u];
    }
    __syncthreads();
  }
}

// Full check of an append request; the same answer for every thread.
__device__ int check_append(const AppendParams& p, int64_t fc, int64_t* total_out,
                            int64_t* warp_vals) {
  int64_t bad = (fc < 0 || fc > p.free_capacity) ? MLA_ERR_DEVICE_CHECK : 0;
  int64_t part = 0;
  for (int i = threadIdx.x; i < p.batch; i += blockDim.x) {
    const int32_t L = p.seqlens[i];
    if (L < 0) { bad = MLA_ERR_DEVICE_CHECK; continue; }
    const int64_t grown = static_cast<int64_t>(L) + p.s_new;
    if (grown > INT32_MAX || pages_of(grown) > p.bt_stride) { bad = MLA_ERR_DEVICE_CHECK; continue; }
    if (L % kPage != 0) {
      const int32_t last = p.block_table[static_cast<int64_t>(i) * p.bt_stride + L / kPage];
      if (last < 0 || last >= p.num_blocks) bad = MLA_ERR_DEVICE_CHECK;
    }
    part += new_pages(L, p.s_new);
  }
  bad = block_reduce(bad, warp_vals, Max());
  const int64_t total = block_reduce(part, warp_vals, Sum());
  *total_out = total;
  if (bad) return static_cast<int>(bad);
  if (total > fc) return MLA_ERR_NO_FREE_PAGES;
  int64_t bad_page = 0;
  for (int64_t slot = fc - total + threadIdx.x; slot < fc; slot += blockDim.x) {
    const int32_t page = p.free_pages[slot];
    if (page < 0 || page >= p.num_blocks) bad_page = 1;
  }
  return block_reduce(bad_page, warp_vals, Max()) ? MLA_ERR_DEVICE_CHECK : MLA_OK;
}

__global__ void __launch_bounds__(kCommitThreads)
mla_append_commit_kernel(AppendParams p) {
  __shared__ int64_t warp_vals[32];
  const int64_t fc = *p.free_count;
  int64_t total = 0;
  const int rc = check_append(p, fc, &total, warp_vals);
  // The rows kernel reads the lengths and the free count: write them only once
  // it has finished (this kernel is its programmatic dependent).
  grid_dependency_wait();
  if (rc != MLA_OK) {
    if (threadIdx.x == 0) report(p.status, rc);
    return;
  }
  for (int i = threadIdx.x; i < p.batch; i += blockDim.x) p.seqlens_rw[i] += p.s_new;
  if (threadIdx.x == 0) *p.free_count_rw = static_cast<int32_t>(fc - total);
}

__global__ void __launch_bounds__(kCommitThreads)
mla_release_kernel(ReleaseParams p) {
  __shared__ int64_t warp_vals[32];
  __shared__ int64_t scan_tmp[32];
  const int tid = threadIdx.x;
  const int64_t fc = *p.free_count;
  const int chunk = (p.batch + blockDim.x - 1) / blockDim.x;
  const int i0 = min(p.batch, tid * chunk), i1 = min(p.batch, i0 + chunk);
  int64_t bad = (fc < 0 || fc > p.free_capacity) ? MLA_ERR_DEVICE_CHECK : 0;
  int64_t give = 0;
  for (int i = i0; i < i1; ++i) {
    if (p.release_mask[i] == 0) continue;
    const int32_t L = p.seqlens[i];
    if (L < 0 || pages_of(L) > p.bt_stride) { bad = MLA_ERR_DEVICE_CHECK; continue; }
    give += pages_of(L);
  }
  bad = block_reduce(bad, warp_vals, Max());
  // exclusive scan of `give` over threads (contiguous chunks keep batch order)
  const int lane = tid & 31, warp = tid >> 5;
  int64_t inc = give;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) scan_tmp[warp] = inc;
  __syncthreads();
  if (tid == 0) {
    int64_t run = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
      const int64_t t = scan_tmp[w];
      scan_tmp[w] = run;
      run += t;
    }
    warp_vals[0] = run;
  }
  __syncthreads();
  const int64_t my_off = scan_tmp[warp] + inc - give;
  const int64_t total = warp_vals[0];
  __syncthreads();
  if (bad == 0 && fc + total > p.free_capacity) bad = MLA_ERR_NO_FREE_PAGES;
  if (bad) {
    if (tid == 0) report(p.status, static_cast<int>(bad));
    return;
  }
  int64_t slot = fc + my_off;
  for (int i = i0; i < i1; ++i) {
    if (p.release_mask[i] == 0) continue;
    const int64_t n = pages_of(p.seqlens[i]);
    const int32_t* row = p.block_table + static_cast<int64_t>(i) * p.bt_stride;
    for (int64_t r = 0; r < n; ++r) p.free_pages[slot++] = row[r];
    p.seqlens[i] = 0;
  }
  if (tid == 0) *p.free_count = static_cast<int32_t>(fc + total);
}

}  // namespace

cudaError_t launch_append(const AppendParams& p_in, bool fp8, cudaStream_t stream) {
  AppendParams p = p_in;
  p.tokens_per_cta = p.s_new < kMaxTokensPerCta ? p.s_new : kMaxTokensPerCta;
  int spc = (kMaxTokensPerCta + p.tokens_per_cta - 1) / p.tokens_per_cta;
  const int spc_batch = (p.batch + 511) / 512;  // at most 512 sequence groups
  if (spc_batch > spc) spc = spc_batch;
  p.seqs_per_cta = spc;  // <= 128 for batch <= 65536
  const int gx = (p.batch + spc - 1) / spc;
  const int chunks = (p.s_new + p.tokens_per_cta - 1) / p.tokens_per_cta;
  int gy = 2048 / gx;
  if (gy < 1) gy = 1;
  if (gy > chunks) gy = chunks;
  if (fp8)
    mla_append_rows_kernel<true><<<dim3(gx, gy), kAppendThreads, 0, stream>>>(p);
  else
    mla_append_rows_kernel<false><<<dim3(gx, gy), kAppendThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the commit kernel checks the request while the rows kernel copies
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kCommitThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, mla_append_commit_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_release(const ReleaseParams& p, cudaStream_t stream) {
  mla_release_kernel<<<1, kCommitThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla

namespace {
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

extern "C" {

int mla_append_latent(const void* rows, int s_new, void* kcache, int64_t num_blocks,
                      int32_t* block_table, int bt_stride, int32_t* cache_seqlens, int batch,
                      int32_t* free_pages, int free_capacity, int32_t* free_count,
                      int32_t* device_status, void* stream) {
  if (rows == nullptr || kcache == nullptr || block_table == nullptr || cache_seqlens == nullptr ||
      free_pages == nullptr || free_count == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (s_new < 1 || s_new > 65536 || batch < 1 || batch > 65536 || bt_stride < 1 ||
      free_capacity < 1)
    return MLA_ERR_INVALID_ARG;
  if (num_blocks < 1 || num_blocks * mla::kPage >= (int64_t(1) << 31)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(rows) || !aligned16(kcache)) return MLA_ERR_INVALID_ARG;
  mla::AppendParams p{};
  p.rows = static_cast<const uint4*>(rows);
  p.kcache = static_cast<uint4*>(kcache);
  p.block_table = block_table;
  p.seqlens = cache_seqlens;
  p.seqlens_rw = cache_seqlens;
  p.free_pages = free_pages;
  p.free_count = free_count;
  p.free_count_rw = free_count;
  p.status = device_status;
  p.num_blocks = num_blocks;
  p.bt_stride = bt_stride;
  p.batch = batch;
  p.s_new = s_new;
  p.free_capacity = free_capacity;
  return mla::launch_append(p, false, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

int mla_append_latent_fp8(const void* rows, int s_new, void* kcache, float* kscale,
                          int64_t num_blocks, int32_t* block_table, int bt_stride,
                          int32_t* cache_seqlens, int batch, int32_t* free_pages,
                          int free_capacity, int32_t* free_count, int32_t* device_status,
                          void* stream) {
  if (rows == nullptr || kcache == nullptr || kscale == nullptr || block_table == nullptr ||
      cache_seqlens == nullptr || free_pages == nullptr || free_count == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (s_new < 1 || s_new > 65536 || batch < 1 || batch > 65536 || bt_stride < 1 ||
      free_capacity < 1)
    return MLA_ERR_INVALID_ARG;
  if (num_blocks < 1 || num_blocks * mla::kPage >= (int64_t(1) << 31)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(rows) || !aligned16(kcache) || !aligned16(kscale)) return MLA_ERR_INVALID_ARG;
  mla::AppendParams p{};
  p.rows = static_cast<const uint4*>(rows);
  p.kcache8 = static_cast<uint8_t*>(kcache);
  p.kscale = kscale;
  p.block_table = block_table;
  p.seqlens = cache_seqlens;
  p.seqlens_rw = cache_seqlens;
  p.free_pages = free_pages;
  p.free_count = free_count;
  p.free_count_rw = free_count;
  p.status = device_status;
  p.num_blocks = num_blocks;
  p.bt_stride = bt_stride;
  p.batch = batch;
  p.s_new = s_new;
  p.free_capacity = free_capacity;
  return mla::launch_append(p, true, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

int mla_release_pages(const int32_t* release_mask, int32_t* block_table, int bt_stride,
                      int32_t* cache_seqlens, int batch, int32_t* free_pages, int free_capacity,
                      int32_t* free_count, int32_t* device_status, void* stream) {
  if (release_mask == nullptr || block_table == nullptr || cache_seqlens == nullptr ||
      free_pages == nullptr || free_count == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65536 || bt_stride < 1 || free_capacity < 1) return MLA_ERR_INVALID_ARG;
  mla::ReleaseParams p{};
  p.release_mask = release_mask;
  p.block_table = block_table;
  p.seqlens = cache_seqlens;
  p.free_pages = free_pages;
  p.free_count = free_count;
  p.status = device_status;
  p.bt_stride = bt_stride;
  p.batch = batch;
  p.free_capacity = free_capacity;
  return mla::launch_release(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MLA_OK
                                                                                  : MLA_ERR_CUDA;
}

}  // extern "C"

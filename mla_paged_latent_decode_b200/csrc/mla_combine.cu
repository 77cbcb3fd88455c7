// mla_combine.cu -- merge the partial results of split sequences by log-sum-exp.
//
// For a sequence cut into k > 1 pieces, piece s holds o_s = (its softmax-
// weighted values, normalised over its own tokens) and lse_s.  Then
//   lse = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - lse) * o_s,
// and pieces with lse_s = -inf (no visible token) weigh nothing.  This is the
// identity that lets the decode spread one sequence over several SMs; the
// pages give no such step (their decode kernel is described only as
// "optimized for variable-length" serving, "OpenSourceWeek Day 1: FlashMLA").
//
// 64 threads per query row, each owning 8 of the 512 values as two float4
// (a warp reads two rows' 1 KB halves, coalesced).  Pieces are taken four at a
// time: the four lse values (the same address across the row's threads) and
// the four partial rows are loaded together, then merged into a running
// maximum m, sum and accumulator, so a sequence of up to four pieces costs one
// round trip to memory.  out = acc / sum and lse = m + ln(sum) at the end,
// which equals the formula above.
#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kCombineThreads = 256;
constexpr int kRowThreads = 64;                  // threads per query row
constexpr int kVec = kDv / 4 / kRowThreads;      // float4 per thread
constexpr int kPiecesPerRound = 4;

__global__ void __launch_bounds__(kCombineThreads)
mla_combine_kernel(const CombineParams p) {
  // Launched as a programmatic dependent of the decode kernel.  The piece
  // counts come from the scheduler, which finished before any decode CTA got
  // past its own dependency wait, so they are read before this grid's wait: a
  // sequence with one piece (its output written by the decode) needs nothing,
  // and its blocks leave without waiting for the decode to finish.
  const int seq = blockIdx.x;
  const int base = p.num_splits[seq];
  const int k = p.num_splits[seq + 1] - base;
  if (k <= 1) return;
  grid_dependency_wait();  // the decode's partial outputs are complete and visible
  const int t = blockIdx.y * kCombineThreads + threadIdx.x;
  const int row = t / kRowThreads, c = t % kRowThreads;
  if (row >= p.rows) return;
  const float* lse_col = p.part_lse + static_cast<int64_t>(base) * p.rows + row;
  const float4* part = reinterpret_cast<const float4*>(
      p.part_o + (static_cast<int64_t>(base) * p.rows + row) * kDv) + c;
  const int64_t piece_stride = static_cast<int64_t>(p.rows) * kDv / 4;  // in float4

  float m = -INFINITY, sum = 0.f;
  float4 acc[kVec];
#pragma unroll
  for (int u = 0; u < kVec; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < k; s0 += kPiecesPerRound) {
    float ls[kPiecesPerRound];
    float4 v[kPiecesPerRound][kVec];
#pragma unroll
    for (int i = 0; i < kPiecesPerRound; ++i) {
      const bool in = s0 + i < k;
      ls[i] = in ? lse_col[static_cast<int64_t>(s0 + i) * p.rows] : -INFINITY;
#pragma unroll
      for (int u = 0; u < kVec; ++u)
        v[i][u] = in ? part[(s0 + i) * piece_stride + kRowThreads * u]
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mn = m;
#pragma unroll
    for (int i = 0; i < kPiecesPerRound; ++i) mn = fmaxf(mn, ls[i]);
    if (mn == -INFINITY) continue;  // no visible token so far
    const float a = __expf(m - mn);  // weight of what came before (0 while m = -inf)
    sum *= a;
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      acc[u].x *= a; acc[u].y *= a; acc[u].z *= a; acc[u].w *= a;
    }
#pragma unroll
    for (int i = 0; i < kPiecesPerRound; ++i) {
      const float w = __expf(ls[i] - mn);  // 0 for a piece with lse = -inf
      sum += w;
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        acc[u].x += w * v[i][u].x; acc[u].y += w * v[i][u].y;
        acc[u].z += w * v[i][u].z; acc[u].w += w * v[i][u].w;
      }
    }
    m = mn;
  }

  // every piece empty: out = 0 and lse = -inf (the log of an empty sum)
  const float inv = m == -INFINITY ? 0.f : 1.f / sum;
  __nv_bfloat16* out = p.out + (static_cast<int64_t>(seq) * p.rows + row) * kDv;
#pragma unroll
  for (int u = 0; u < kVec; ++u) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x * inv, acc[u].y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc[u].z * inv, acc[u].w * inv);
    uint2 w;
    w.x = *reinterpret_cast<uint32_t*>(&lo);
    w.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(out + 4 * (c + kRowThreads * u)) = w;
  }
  if (c == 0) {
    const int jq = row / p.h_q, hq = row % p.h_q;
    p.lse[(static_cast<int64_t>(seq) * p.h_q + hq) * p.s_q + jq] =
        m == -INFINITY ? -INFINITY : m + __logf(sum);
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  // x: sequences (any batch size); y: blocks of four query rows (rows <= 65536)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.batch, (p.rows * kRowThreads + kCombineThreads - 1) / kCombineThreads);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, mla_combine_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla

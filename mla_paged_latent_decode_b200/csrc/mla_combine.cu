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
// One warp per query row.  Lane s holds piece s's lse (pieces in groups of 32),
// so the maximum, the sum and every weight come from shuffles after a single
// load; each lane owns 16 of the 512 values as 4 float4 (coalesced 512-byte
// warp loads), and the loads of several pieces are in flight together.
#include "mla_kernels.cuh"

namespace mla {
namespace {

constexpr int kCombineWarps = 8;

__global__ void __launch_bounds__(kCombineWarps * 32)
mla_combine_kernel(const CombineParams p) {
  const int seq = blockIdx.x;
  const int base = p.num_splits[seq];
  const int k = p.num_splits[seq + 1] - base;
  if (k <= 1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.y * kCombineWarps + warp;
  if (row >= p.rows) return;
  const int jq = row / p.h_q, hq = row % p.h_q;
  const float* lse_col = p.part_lse + static_cast<int64_t>(base) * p.rows + row;

  float mx = -INFINITY;
  for (int s = lane; s < k; s += 32) mx = fmaxf(mx, lse_col[static_cast<int64_t>(s) * p.rows]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));

  __nv_bfloat16* out = p.out + (static_cast<int64_t>(seq) * p.rows + row) * kDv;
  float* lse_out = p.lse + (static_cast<int64_t>(seq) * p.h_q + hq) * p.s_q + jq;
  if (mx == -INFINITY) {
    for (int c = lane * 8; c < kDv; c += 32 * 8)
      *reinterpret_cast<uint4*>(out + c) = make_uint4(0u, 0u, 0u, 0u);
    if (lane == 0) *lse_out = -INFINITY;
    return;
  }
  float sum = 0.f;
  for (int s = lane; s < k; s += 32) sum += __expf(lse_col[static_cast<int64_t>(s) * p.rows] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float lse = mx + __logf(sum);

  float4 acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* part = reinterpret_cast<const float4*>(
      p.part_o + (static_cast<int64_t>(base) * p.rows + row) * kDv) + lane;
  const int64_t piece_stride = static_cast<int64_t>(p.rows) * kDv / 4;  // in float4
  for (int s0 = 0; s0 < k; s0 += 32) {
    // lane s: weight of piece s0 + s (the lse was read above, so this hits in cache)
    const float ls = s0 + lane < k ? lse_col[static_cast<int64_t>(s0 + lane) * p.rows] : -INFINITY;
    const float my_w = ls == -INFINITY ? 0.f : __expf(ls - lse);
    const int n = k - s0 < 32 ? k - s0 : 32;
#pragma unroll 2
    for (int s = 0; s < n; ++s) {
      const float w = __shfl_sync(0xffffffffu, my_w, s);
      const float4* src = part + (s0 + s) * piece_stride;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 v = src[32 * u];
        acc[u].x += w * v.x;
        acc[u].y += w * v.y;
        acc[u].z += w * v.z;
        acc[u].w += w * v.w;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x, acc[u].y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc[u].z, acc[u].w);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&lo);
    v.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(out + 4 * (lane + 32 * u)) = v;
  }
  if (lane == 0) *lse_out = lse;
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  dim3 grid(p.batch, (p.rows + kCombineWarps - 1) / kCombineWarps);
  mla_combine_kernel<<<grid, kCombineWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla

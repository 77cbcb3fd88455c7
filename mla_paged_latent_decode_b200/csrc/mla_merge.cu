// mla_merge.cu -- merge decode results over disjoint parts of each sequence's
// cache (the parts of a cache sharded across GPUs) by log-sum-exp.
//
// Part r holds o_r (bf16, normalised over its own tokens) and lse_r (fp32,
// natural log; -inf when the part has no visible token).  Then
//   lse = ln sum_r exp(lse_r),   out = sum_r exp(lse_r - lse) * o_r,
// the same identity the split combine uses inside one GPU, here over the
// results that ranks exchange.  The pages name this cross-device form only as
// the partition-then-combine step of tensor-parallel latent attention ("TPLA:
// Tensor Parallel Latent Attention...", abstract); sharding the cached tokens
// instead of the latent dims keeps the result exact.
//
// 64 threads per query row, each owning 8 of the 512 values (one 16-byte load
// per part); parts are merged four at a time into a running maximum, sum and
// accumulator.
#include "mla_kernels.cuh"

namespace mla {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kRowThreads = 64;   // threads per query row; 8 values each
constexpr int kPartsPerRound = 4;

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], uint4 v, float w) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += w * __uint_as_float(u[i] << 16);
    acc[2 * i + 1] += w * __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(kMergeThreads)
mla_merge_kernel(const uint4* __restrict__ outs, const float* __restrict__ lses, int parts,
                 int64_t nrows, int s_q, int h_q, uint4* __restrict__ out, float* __restrict__ lse) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kMergeThreads + threadIdx.x;
  const int64_t row = t / kRowThreads;  // flattened (sequence, query position, head)
  const int c = static_cast<int>(t % kRowThreads);
  if (row >= nrows) return;
  const int rows = s_q * h_q;
  const int64_t seq = row / rows;
  const int r = static_cast<int>(row % rows), jq = r / h_q, hq = r % h_q;
  const int64_t lse_idx = (seq * h_q + hq) * s_q + jq;  // [b, h_q, s_q]
  const int64_t part_stride = nrows * (kDv / 8);           // in uint4
  const uint4* src = outs + row * (kDv / 8) + c;

  float m = -INFINITY, sum = 0.f;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int r0 = 0; r0 < parts; r0 += kPartsPerRound) {
    float ls[kPartsPerRound];
    uint4 v[kPartsPerRound];
#pragma unroll
    for (int i = 0; i < kPartsPerRound; ++i) {
      const bool in = r0 + i < parts;
      ls[i] = in ? lses[static_cast<int64_t>(r0 + i) * nrows + lse_idx] : -INFINITY;
      v[i] = in ? src[(r0 + i) * part_stride] : make_uint4(0u, 0u, 0u, 0u);
    }
    float mn = m;
#pragma unroll
    for (int i = 0; i < kPartsPerRound; ++i) mn = fmaxf(mn, ls[i]);
    if (mn == -INFINITY) continue;  // nothing visible so far
    const float a = __expf(m - mn);  // weight of what came before (0 while m = -inf)
    sum *= a;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= a;
#pragma unroll
    for (int i = 0; i < kPartsPerRound; ++i) {
      const float w = __expf(ls[i] - mn);  // 0 for a part with lse = -inf
      sum += w;
      if (w != 0.f) add_bf16x8(acc, v[i], w);
    }
    m = mn;
  }
  const float inv = m == -INFINITY ? 0.f : 1.f / sum;
  uint4 o;
  __nv_bfloat162 b0 = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  __nv_bfloat162 b1 = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[4] * inv, acc[5] * inv);
  __nv_bfloat162 b3 = __floats2bfloat162_rn(acc[6] * inv, acc[7] * inv);
  o.x = *reinterpret_cast<uint32_t*>(&b0);
  o.y = *reinterpret_cast<uint32_t*>(&b1);
  o.z = *reinterpret_cast<uint32_t*>(&b2);
  o.w = *reinterpret_cast<uint32_t*>(&b3);
  out[row * (kDv / 8) + c] = o;
  if (c == 0) lse[lse_idx] = m == -INFINITY ? -INFINITY : m + __logf(sum);
}

}  // namespace

cudaError_t launch_merge(const void* outs, const float* lses, int parts, int64_t nrows, int s_q,
                         int h_q, void* out, float* lse, cudaStream_t stream) {
  const int64_t threads = nrows * kRowThreads;
  const int64_t blocks = (threads + kMergeThreads - 1) / kMergeThreads;
  mla_merge_kernel<<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(
      static_cast<const uint4*>(outs), lses, parts, nrows, s_q, h_q, static_cast<uint4*>(out), lse);
  return cudaGetLastError();
}

}  // namespace mla

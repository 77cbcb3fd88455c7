// mla_decode_sm100.cu -- MLA decode over a paged latent cache on sm_100a.
//
// One CTA owns one 64-row block of the flattened (s_q, h_q) query rows of one
// worker's run of (sequence, page) items (see mla_metadata.cu).  Per page:
//
//   TMA   : the 64 x 576 bf16 page (72 KB) -> shared memory, 9 boxes of 64 x 64
//           with 128-byte swizzle, through the block table; two stages.
//   MMA   : S  = Q . K^T     tcgen05 M=64 N=64  K=576, A=Q (smem), B=page (smem)
//           O += P . V       tcgen05 M=64 N=256 K=64 (x2 halves of dv=512),
//                            A=P (smem), B=the same page tile read MN-major:
//                            the value is dims 0..511 of the row already in
//                            shared memory, so each page leaves HBM once.
//   softmax warps: online softmax on S read from TMEM, P (bf16) -> shared
//           memory, O rescaled in TMEM when the running max grows.
//   epilogue: O / l -> bf16 out and lse, or fp32 partials for split sequences.
//
// TMEM (512 columns x 128 lanes): an M=64 accumulator occupies lanes 0-15 of
// each 32-lane quarter.  O (64 x 512 fp32) takes all 512 columns of those
// lanes; S (64 x 64 fp32) sits in the other half of each quarter (lane offset
// 16), columns 0..63.  Thread t of softmax warp w therefore sees O row
// 16w + t (t < 16) or S row 16w + t - 16 (t >= 16) in its lane.
//
// Warp roles (192 threads): warps 0-3 softmax/correction/epilogue, warp 4 TMA
// producer, warp 5 MMA issuer (and TMEM allocator).
//
// The method is "FlashMLA: Revolutionizing Efficient Decoding...", sections
// 4.2.1-4.2.3 (TMA prefetch of 64-row latent blocks into shared memory, tensor
// cores for QK^T and PV, softmax fused into the kernel) re-designed for the
// 5th-generation tensor core: accumulators live in TMEM instead of registers.
#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kThreads = 192;
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kChunkBytes = 64 * 128;              // 64 rows x 64 bf16 (one swizzle column block)
constexpr int kChunks = kDqk / 64;                 // 9
constexpr int kTileBytes = kChunks * kChunkBytes;  // 73728 = 64 x 576 bf16
constexpr int kStages = 2;
constexpr int kPBytes = 64 * 128;                  // P: 64 rows x 64 tokens bf16

constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kTileBytes;
constexpr int kOffP = kOffKV + kStages * kTileBytes;
constexpr int kOffBar = kOffP + kPBytes;
enum Bar { kFull0 = 0, kEmpty0 = kStages, kQFull = 2 * kStages, kQEmpty, kSFull, kPFull, kOFull,
           kOFree, kNumBars };
constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem address + abort flag
constexpr int kSmemUsed = kOffMisc + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;       // slack to align the base to 1024 B

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 16u << 16;             // lane offset 16, column 0
constexpr float kRescaleThreshold = 8.0f;          // log2 units: P <= 2^8 before a rescale

constexpr uint32_t kIdescQK = idesc_bf16_f32(64, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(64, 256, false, true);

static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Piece {
  int seq, pg0, npg, split_idx;
};

// Piece `pc` of a worker: its sequence, first page, page count and split index.
// The page count never exceeds the block-table row (bt_stride entries).
__device__ __forceinline__ Piece piece_of(const int32_t* md, int pc, const int32_t* seqlens,
                                          int64_t bt_stride) {
  const int npieces = md[5];
  Piece p;
  p.seq = md[0] + pc;
  const int L = seqlens[p.seq];
  int npages = L > 0 ? (L + kPage - 1) / kPage : 0;
  if (npages > bt_stride) npages = static_cast<int>(bt_stride);
  const int it0 = pc == 0 ? md[1] : 0;
  const int it1 = pc == npieces - 1 ? md[3] : (npages > 0 ? npages : 1);
  const int pg1 = it1 < npages ? it1 : npages;
  p.pg0 = it0;
  p.npg = pg1 > it0 ? pg1 - it0 : 0;
  p.split_idx = pc == 0 ? md[4] : 0;
  return p;
}

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__global__ void __launch_bounds__(kThreads, 1)
mla_decode_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_kv, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sq = smem + kOffQ;
  uint8_t* skv = smem + kOffKV;
  uint8_t* sp = smem + kOffP;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int worker = blockIdx.x, rb = blockIdx.y;
  const int32_t* md = p.tile_md + static_cast<int64_t>(worker) * kMdStride;
  const int npieces = md[5];
  if (npieces == 0) return;  // idle worker: uniform exit before any barrier or TMEM use
  if (md[0] < 0 || npieces < 0 || md[0] + npieces > p.batch) {  // metadata not from this batch
    if (threadIdx.x == 0) report(p.status, MLA_ERR_DEVICE_CHECK);
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar[kFull0 + s], 1);
      mbar_init(&bar[kEmpty0 + s], 1);
    }
    mbar_init(&bar[kQFull], 1);
    mbar_init(&bar[kQEmpty], 1);
    mbar_init(&bar[kSFull], 1);
    mbar_init(&bar[kPFull], 128);
    mbar_init(&bar[kOFull], 1);
    mbar_init(&bar[kOFree], 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_kv);
      int q_loads = 0, kv_loads = 0;
      bool ok = true;
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (p.seqlens[pz.seq] > p.bt_stride * kPage) report(p.status, MLA_ERR_DEVICE_CHECK);
        if (pz.npg == 0) continue;
        if (q_loads > 0) ok = mbar_wait(&bar[kQEmpty], (q_loads - 1) & 1, abort_flag, kWaitLimitNs);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar[kQFull], kTileBytes);
        const int qrow = pz.seq * p.rows + rb * kRowsPerCta;
        for (int c = 0; c < kChunks; ++c)
          tma_load_2d(sq + c * kChunkBytes, &tm_q, c * 64, qrow, &bar[kQFull]);
        ++q_loads;
        const int32_t* bt = p.block_table + static_cast<int64_t>(pz.seq) * p.bt_stride;
        for (int j = 0; j < pz.npg; ++j) {
          const int stage = kv_loads % kStages, use = kv_loads / kStages;
          if (use > 0) {
            ok = mbar_wait(&bar[kEmpty0 + stage], (use - 1) & 1, abort_flag, kWaitLimitNs);
            if (!ok) break;
          }
          const int page = __ldg(bt + pz.pg0 + j);
          mbar_arrive_expect_tx(&bar[kFull0 + stage], kTileBytes);
          uint8_t* dst = skv + stage * kTileBytes;
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(dst + c * kChunkBytes, &tm_kv, c * 64, page * kPage, &bar[kFull0 + stage]);
          ++kv_loads;
        }
      }
      // Before leaving, let every copy this thread issued land (bounded).
      for (int s = 0; s < kStages && s < kv_loads; ++s) {
        const int n = kv_loads - 1 - s;  // the last load issued into some stage
        mbar_wait(&bar[kFull0 + n % kStages], (n / kStages) & 1, abort_flag, kWaitLimitNs);
      }
      if (q_loads > 0) mbar_wait(&bar[kQFull], (q_loads - 1) & 1, abort_flag, kWaitLimitNs);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int q_uses = 0, kv_uses = 0, p_uses = 0, pieces_done = 0;
      bool ok = true;
      const uint32_t q_base = smem_addr(sq), kv_base = smem_addr(skv), p_base = smem_addr(sp);
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (pz.npg == 0) continue;
        ok = mbar_wait(&bar[kQFull], q_uses & 1, abort_flag, kWaitLimitNs);
        ++q_uses;
        if (ok && pieces_done > 0)
          ok = mbar_wait(&bar[kOFree], (pieces_done - 1) & 1, abort_flag, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        for (int j = 0; j < pz.npg; ++j) {
          const int stage = kv_uses % kStages;
          ok = mbar_wait(&bar[kFull0 + stage], (kv_uses / kStages) & 1, abort_flag, kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t tile = kv_base + stage * kTileBytes;
          // S = Q . K^T over 576 dims: 9 swizzle blocks x 4 K-steps of 16
#pragma unroll 4
          for (int kk = 0; kk < kDqk / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
            umma_bf16_ss(tmem + kTmemS, smem_desc_sw128(q_base + off, 16, 1024),
                         smem_desc_sw128(tile + off, 16, 1024), kIdescQK, kk > 0);
          }
          umma_commit(&bar[kSFull]);
          if (j == pz.npg - 1) umma_commit(&bar[kQEmpty]);
          ok = mbar_wait(&bar[kPFull], p_uses & 1, abort_flag, kWaitLimitNs);
          ++p_uses;
          if (!ok) break;
          tc_fence_after();
          // O += P . V, V = columns 0..511 of the same tile, read MN-major
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < kPage / 16; ++kk) {
              umma_bf16_ss(tmem + half * 256, smem_desc_sw128(p_base + kk * 32, 16, 1024),
                           smem_desc_sw128(tile + half * 4 * kChunkBytes + kk * 2048,
                                           kChunkBytes, 1024),
                           kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&bar[kEmpty0 + stage]);
          ++kv_uses;
        }
        if (!ok) break;
        umma_commit(&bar[kOFull]);
        ++pieces_done;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const bool is_s = lane >= 16;
    const int r_local = 16 * warp + (lane & 15);
    const int row = rb * kRowsPerCta + r_local;
    const bool row_ok = row < p.rows;
    const int jq = row_ok ? row / p.h_q : 0;
    const int hq = row_ok ? row % p.h_q : 0;
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    int s_uses = 0, o_uses = 0;
    bool ok = true;
    for (int pc = 0; pc < npieces && ok; ++pc) {
      const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
      const int L = p.seqlens[pz.seq];
      int limit = p.causal ? L - p.s_q + jq + 1 : L;
      limit = limit < 0 ? 0 : (limit > L ? L : limit);
      if (static_cast<int64_t>(limit) > p.bt_stride * kPage) limit = static_cast<int>(p.bt_stride * kPage);
      const int base_split = p.num_splits[pz.seq];
      const int k_pieces = p.num_splits[pz.seq + 1] - base_split;
      const int64_t slot = static_cast<int64_t>(base_split) + pz.split_idx;
      const int64_t out_row = static_cast<int64_t>(pz.seq) * p.rows + row;
      float m = -INFINITY, l = 0.f;

      if (pz.npg > 0) {
        for (int j = 0; j < pz.npg; ++j) {
          ok = mbar_wait(&bar[kSFull], s_uses & 1, abort_flag, kWaitLimitNs);
          ++s_uses;
          if (!ok) break;
          tc_fence_after();
          uint32_t sa[32], sb[32];
          // 32x32b loads read all 32 lanes of the warp's quarter: lanes 16-31 carry
          // this page's S row (columns 0..63), lanes 0-15 O values that are unused here.
          tmem_ld32(tmem + lane_base + 0, sa);
          tmem_ld32(tmem + lane_base + 32, sb);
          tmem_ld_wait(sa);
          tmem_ld_wait(sb);
          float alpha = 1.f;
          if (is_s) {
            const int nvalid_raw = limit - (pz.pg0 + j) * kPage;
            const int nvalid = nvalid_raw < 0 ? 0 : (nvalid_raw > kPage ? kPage : nvalid_raw);
            float tmax = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c < nvalid) tmax = fmaxf(tmax, __uint_as_float(sa[c]) * p.scale_log2);
              if (c + 32 < nvalid) tmax = fmaxf(tmax, __uint_as_float(sb[c]) * p.scale_log2);
            }
            float m_new = m;
            if (tmax > m + kRescaleThreshold) {
              m_new = tmax;
              alpha = ex2_approx(m - m_new);  // m = -inf gives 0
            }
            float psum = 0.f;
            uint32_t packed[32];
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float p0 = c < nvalid ? ex2_approx(__uint_as_float(sa[c]) * p.scale_log2 - m_new) : 0.f;
              const float p1 = c + 1 < nvalid ? ex2_approx(__uint_as_float(sa[c + 1]) * p.scale_log2 - m_new) : 0.f;
              const float p2 = c + 32 < nvalid ? ex2_approx(__uint_as_float(sb[c]) * p.scale_log2 - m_new) : 0.f;
              const float p3 = c + 33 < nvalid ? ex2_approx(__uint_as_float(sb[c + 1]) * p.scale_log2 - m_new) : 0.f;
              psum += (p0 + p1) + (p2 + p3);
              packed[c >> 1] = pack_bf16x2(p0, p1);
              packed[16 + (c >> 1)] = pack_bf16x2(p2, p3);
            }
            l = l * alpha + psum;
            m = m_new;
            // P row r_local: 64 tokens = 8 units of 16 B, 128-byte swizzle
            uint8_t* prow = sp + r_local * 128;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              uint4 v = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2],
                                   packed[4 * u + 3]);
              *reinterpret_cast<uint4*>(prow + ((u ^ (r_local & 7)) << 4)) = v;
            }
          }
          const float alpha_o = __shfl_xor_sync(0xffffffffu, alpha, 16);
          const bool need = (j > 0) && __any_sync(0xffffffffu, (!is_s) && alpha_o != 1.f);
          if (need) {
            for (int c0 = 0; c0 < kDv; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(tmem + lane_base + c0, o);
              tmem_ld_wait(o);
              if (!is_s) {
#pragma unroll
                for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha_o);
              }
              tmem_st32(tmem + lane_base + c0, o);
            }
            tmem_st_wait();
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&bar[kPFull]);
        }
        if (!ok) break;
        ok = mbar_wait(&bar[kOFull], o_uses & 1, abort_flag, kWaitLimitNs);
        ++o_uses;
        if (!ok) break;
        tc_fence_after();
      }
      // epilogue
      const float l_o = __shfl_xor_sync(0xffffffffu, l, 16);
      const float inv = l_o > 0.f ? 1.f / l_o : 0.f;
      for (int c0 = 0; c0 < kDv; c0 += 32) {
        uint32_t o[32];
        if (pz.npg > 0) {
          tmem_ld32(tmem + lane_base + c0, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        if (!is_s && row_ok) {
          if (k_pieces == 1) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + out_row * kDv + c0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[8 * u + 0]) * inv, __uint_as_float(o[8 * u + 1]) * inv);
              v.y = pack_bf16x2(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv);
              v.z = pack_bf16x2(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv);
              v.w = pack_bf16x2(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv);
              dst[u] = v;
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(p.part_o + (slot * p.rows + row) * kDv + c0);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              dst[u] = make_float4(__uint_as_float(o[4 * u]) * inv, __uint_as_float(o[4 * u + 1]) * inv,
                                   __uint_as_float(o[4 * u + 2]) * inv, __uint_as_float(o[4 * u + 3]) * inv);
          }
        }
      }
      if (is_s && row_ok) {
        const float lse = l > 0.f ? (m + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
        if (k_pieces == 1)
          p.lse[(static_cast<int64_t>(pz.seq) * p.h_q + hq) * p.s_q + jq] = lse;
        else
          p.part_lse[slot * p.rows + row] = lse;
      }
      if (pz.npg > 0) {
        tc_fence_before();
        mbar_arrive(&bar[kOFree]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(p.status, MLA_ERR_DEVICE_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_kv,
                          const DecodeParams& p, int num_workers, cudaStream_t stream) {
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(mla_decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int row_blocks = (p.rows + kRowsPerCta - 1) / kRowsPerCta;
  dim3 grid(num_workers, row_blocks);
  mla_decode_sm100_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm_q, tm_kv, p);
  return cudaGetLastError();
}

}  // namespace mla

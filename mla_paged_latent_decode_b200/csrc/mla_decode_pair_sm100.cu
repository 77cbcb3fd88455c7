// mla_decode_pair_sm100.cu -- MLA decode on CTA pairs (clusters of 2), sm_100a.
//
// Used when a sequence has more than 64 query rows (s_q * h_q > 64).  A pair
// of CTAs owns a 128-row block of the query rows of one worker's run of
// (sequence, page) items; CTA r of the pair holds rows 64r..64r+63.  Every MMA
// is a pair MMA (tcgen05 .cta_group::2, M = 128 rows split over the two SMs),
// which runs at the full rate of the tensor cores, where the single-CTA kernel
// for narrow rows (mla_decode_sm100.cu) issues half-rate M=64 MMAs.
//
// Per page (64 tokens x 576 bf16):
//   S  = Q . K^T   N = 64 tokens: CTA r supplies tokens 32r..32r+31 of the page
//                  (all 576 dims) as its half of B; each CTA receives S for its
//                  64 rows and all 64 tokens.  Dims 0..383 of Q are read from
//                  tensor memory, dims 384..575 from shared memory.
//   O += P . V     N = 256 dv per MMA, two MMAs: CTA 0 supplies dv 128h..128h+127
//                  of MMA h and CTA 1 dv 256+128h..256+128h+127, for all 64 tokens.
// Each CTA loads its 32 token rows in full (K part, 36 KB, nine 64-dim chunks of
// 32 rows x 128 bytes) into a ring slot.  The same slot then serves as V:
//   PV K-steps 0-1 (tokens  0..31) read chunks 0..3 of the slot,
//   PV K-steps 2-3 (tokens 32..63) read chunks 4..7,
// at the same shared-memory offsets in both CTAs (a pair MMA has one descriptor).
// CTA 0's chunks 0..3 already hold what it supplies for tokens 0..31 (its own
// tokens, dims 0..255), and CTA 1's chunks 4..7 what it supplies for tokens
// 32..63.  The other half is the peer's tokens: once the QK^T MMAs have read
// them, CTA 0 overwrites its chunks 4..7 with tokens 32..63 x dims 0..255 and
// CTA 1 its chunks 0..3 with tokens 0..31 x dims 256..511 (16 KB each, one TMA
// box; the bytes were just read from HBM by the peer, so they come from L2).
// Shared memory therefore receives 1.44x the page bytes (36 + 16 KB per CTA
// for a 72 KB page), and HBM is read once.  Both loads are TMA boxes through
// the block table with 128-byte swizzle; their completion is counted on the
// leader's barriers.
//
// Tensor memory per CTA (512 columns, all 128 lanes):
//   O   columns   0..255  64 rows x 512 fp32: lane L holds row L % 64, dv half
//                         L / 64 of each 256-wide MMA
//   S   columns 256..319  two buffers of 32 columns: lane L, row L % 64,
//                         tokens 32 (L / 64) + c
//   Q   columns 320..511  dims 0..383 of the 64 rows, two bf16 per column, each
//                         row held in lanes L and L + 64
// The rest of Q (dims 384..575, 24 KB) stays in shared memory, which leaves room
// for five 36 KB slots and two P buffers.  A slot is held from its K-part load
// until PV of its page has completed.
//
// The K-part ring also stages the query rows: per piece, two ring entries carry
// dims 0..255 and 256..383 of this CTA's 64 rows (plain TMA, counted on this
// CTA's own barrier); the softmax warps copy them into tensor memory, and the
// leader's QK^T warp releases both slots once the copies of both CTAs are done.
//
// Warp roles (288 threads per CTA):
//   warps 0-3  softmax / correction / epilogue (both CTAs); thread L owns half
//              of row L % 64; the two halves of a row exchange maxima and sums
//              through shared memory.
//   warp 4     TMA: query rows and K parts (both CTAs).
//   warp 8     TMA: the peer-token value chunks (both CTAs), each as soon as the
//              QK^T MMAs have read the chunks it replaces.
//   warps 5, 7 QK^T of even / odd pages (leader CTA only); warp 5 also
//              allocates the pair's tensor memory in each CTA.
//   warp 6     PV (leader CTA only).
// P is double-buffered, so the softmax of page g overlaps PV of page g - 1; the
// softmax waits for that PV only when it has to rescale O.
//
// FP8 cache (template argument kFp8, 640 threads): E4M3 codes with one
// power-of-two scale per token.  The same slots, MMAs and barriers, with the
// loads and their completion changed: one TMA box per K part lands each
// chunk's codes in the upper half of its 128-byte row slots (a view of the
// codes whose chunks are 64 bytes apart, started 64 bytes early), and the
// page's 64 scales come with it; two groups of four converter warps (even and
// odd pages) widen the codes in place to bf16 values code * scale, exactly,
// and three more warps widen the peer tokens' value chunks the value warp loads
// the same way.  Each group signals the leader's barrier once per CTA.  The
// softmax, the MMAs and the epilogue are those of the bf16 cache.
//
// The method is that of the single-CTA kernel ("FlashMLA: Revolutionizing
// Efficient Decoding...", sections 4.2.1-4.2.3: TMA prefetch of 64-row latent
// blocks, tensor cores for QK^T and PV, softmax fused in the kernel), mapped
// onto the pair tensor-core instructions of sm_100a.
#include <atomic>

#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kSoftmaxWarps = 4;
constexpr int kTmaKWarp = 4;
constexpr int kQkEvenWarp = 5;
constexpr int kPvWarp = 6;
constexpr int kQkOddWarp = 7;
// Threads and the warp of the value loads: 288 threads (warp 8 loads values)
// for a bf16 cache.  For an FP8 cache, 640: two groups of four warps (8-11 and
// 12-15) widen the K parts of even and odd pages, warp 16 loads values and
// warps 17-19 widen them.
template <bool kFp8>
struct PairRoles {
  static constexpr int kThreads = kFp8 ? 640 : 288;
  static constexpr int kTmaVWarp = kFp8 ? 16 : 8;
};
constexpr int kKConvWarp0 = 8;                 // FP8: K-part converters, warps 8..15
constexpr int kKConvGroups = 2;                // of four warps each, alternating pages
constexpr int kKConvThreads = 128;             // per group
constexpr int kVConvWarp0 = 17;                // FP8: value converters, warps 17..19
constexpr int kVConvThreads = 96;
constexpr int kVConvBarrier = 1;               // named barriers: the value converters,
constexpr int kKConvBarrier0 = 2;              //   then one per K-converter group
// FP8 register budget: 640 threads are launched with at most 102 registers
// each (the launcher checks kFp8LaunchRegs); the converter warpgroups lower
// theirs and the softmax warpgroup raises its own.
constexpr int kFp8LaunchRegs = 96;
constexpr int kFp8RegsSoftmax = 176, kFp8RegsConv = 64;
static_assert(128 * kFp8RegsSoftmax + 128 * kFp8LaunchRegs + 384 * kFp8RegsConv <=
                  640 * kFp8LaunchRegs,
              "FP8 setmaxnreg split within the launch's registers");

constexpr int kChunk = 64 * 128;          // 64 rows x 64 bf16 (one 128-byte swizzle column block)
constexpr int kHalfChunk = 32 * 128;      // 32 rows x 64 bf16
constexpr int kChunks = kDqk / 64;        // 9
constexpr int kQTmemChunks = 6;           // dims 0..383 of Q live in tensor memory
constexpr int kQSmemChunks = kChunks - kQTmemChunks;   // dims 384..575 stay in shared memory
constexpr int kQStageA = 4;               // first staging entry: chunks 0..3
constexpr int kQ2Bytes = kQSmemChunks * kChunk;        // 24576
constexpr int kKBytes = kChunks * kHalfChunk;          // 36864: 32 tokens x 576
constexpr int kXChunks = 4;                            // chunks replaced by peer-token values
constexpr int kXBytes = kXChunks * kHalfChunk;         // 16384: 32 tokens x 256 dv
constexpr int kPBytes = kChunk;                        // 64 rows x 64 tokens
constexpr int kKSlots = 5;
constexpr int kQKSteps = kDqk / 16;                    // 36
constexpr int kQTmemKSteps = kQTmemChunks * 4;         // 24
// QK^T K-steps after which chunks 0..3 (resp. 4..7) of the slot have been issued
constexpr int kXDoneStep0 = 4 * kXChunks - 1;          // 15
constexpr int kXDoneStep1 = 8 * kXChunks - 1;          // 31
static_assert(kQStageA * kChunk <= kKBytes && (kQTmemChunks - kQStageA) * kChunk <= kKBytes,
              "query staging entries fit a K-part slot");

constexpr int kOffQ2 = 0;
constexpr int kOffK = kOffQ2 + kQ2Bytes;
constexpr int kOffP = kOffK + kKSlots * kKBytes;
constexpr int kOffX = kOffP + 2 * kPBytes;       // row-half exchange: [2 pages][2 halves][64] f32
constexpr int kOffL = kOffX + 2 * 2 * 64 * 4;    // epilogue sum exchange: [2 pieces][2 halves][64] f32
constexpr int kOffScale = kOffL + 2 * 2 * 64 * 4;  // FP8: [slot][64] fp32: this CTA's 32
                                                    // tokens, then the 32 peer tokens' values
constexpr int kOffBar = kOffScale + kKSlots * kPage * 4;
static_assert(kOffK % 1024 == 0 && kKBytes % 1024 == 0 && kOffP % 1024 == 0,
              "swizzled tiles start on 1024-byte boundaries");
enum Bar {
  kKFull0 = 0,                                    // leader: K parts of both CTAs, per slot
  kVFull0 = kKFull0 + kKSlots,                    // leader: peer-token values of both CTAs
  kQFull = kVFull0 + kKSlots,                     // leader: Q dims 384..575 of both CTAs
  kKEmpty0,                                       // both: pair commits (multicast), per slot:
                                                  //   PV of the slot's page (or the query
                                                  //   copies of a staging entry) is done
  kXFree0 = kKEmpty0 + kKSlots,                   // both: pair commits, [slot][2]: QK^T has
                                                  //   read chunks 0..3 / 4..7 of the slot
  kQEmpty = kXFree0 + 2 * kKSlots,
  kSFull0, kSFull1, kPvDone0, kPvDone1, kOFull,   // both: pair commits (multicast)
  kSFree0, kSFree1, kPFull0, kPFull1, kQReady,    // leader: softmax warps of both CTAs
  kQStage,                                        // local: this CTA's query staging copies
  kXBar, kLBar,                                   // local: softmax exchanges
  kDrain0,                                        // leader: MMA drain after an abort, one
                                                  //   per issuing warp (5, 6, 7)
  kKLanded0 = kDrain0 + 3,                        // FP8, local: a K part's codes and scales
  kVLanded0 = kKLanded0 + kKSlots,                // FP8, local: values' codes and scales
  kNumBars = kVLanded0 + kKSlots
};
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemUsed = kOffMisc + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;       // 256 columns
constexpr uint32_t kTmemS = 256;     // S buffer b at 256 + 32 b
constexpr uint32_t kTmemQ = 320;     // 192 columns
static_assert(kTmemQ + kQTmemChunks * 32 == kTmemCols, "tensor memory budget");
constexpr float kRescaleThreshold = 8.0f;

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);
constexpr uint32_t kSoftmaxArrivals = 2 * kSoftmaxWarps;   // one per softmax warp, both CTAs

struct Piece {
  int seq, pg0, npg, split_idx;
};

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

__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, uint64_t limit_ns) {
  const bool ok = mbar_wait_cluster(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// One arrival per warp on a barrier of the pair leader (CTA 0).
__device__ __forceinline__ void warp_arrive_leader(uint64_t* bar, uint32_t rank, int lane) {
  __syncwarp();
  if (lane == 0) {
    if (rank == 0)
      mbar_arrive(bar);
    else
      mbar_arrive_remote(bar, 0);
  }
}

// Softmax warps: dims 0..383 of the query rows of the piece whose staging
// entries come next in the K ring, staging slots -> tensor memory (row r in
// lanes r and r + 64).  Both QK^T warps have finished the previous piece (their
// Q-empty commit), so no MMA still reads the old rows and neither warp can miss
// a phase of the Q-ready barrier.
__device__ __forceinline__ bool copy_query_rows(const uint8_t* sk, uint64_t* bar,
                                                volatile int* abort_flag, uint32_t tmem_q, int r,
                                                uint32_t rank, int lane, int& entries,
                                                int& qcopies, uint64_t wait_ns) {
  const uint8_t* qa = sk + (entries % kKSlots) * kKBytes;
  const uint8_t* qb = sk + ((entries + 1) % kKSlots) * kKBytes;
  entries += 2;
  if (qcopies > 0 && !warp_wait_cluster(&bar[kQEmpty], (qcopies - 1) & 1, abort_flag, wait_ns))
    return false;
  if (!warp_wait_cluster(&bar[kQStage], qcopies & 1, abort_flag, wait_ns)) return false;
  ++qcopies;
  for (int c = 0; c < kQTmemChunks; ++c) {
    const uint8_t* rowp = (c < kQStageA ? qa + c * kChunk : qb + (c - kQStageA) * kChunk) + r * 128;
    uint32_t q[32];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((u ^ (r & 7)) << 4));
      q[4 * u] = v.x;
      q[4 * u + 1] = v.y;
      q[4 * u + 2] = v.z;
      q[4 * u + 3] = v.w;
    }
    tmem_st32(tmem_q + 32 * c, q);
  }
  tmem_st_wait();
  tc_fence_before();
  warp_arrive_leader(&bar[kQReady], rank, lane);
  return true;
}

// FP8 converters: wait for a landed barrier (bounded), then decide together
// after a named barrier, so that a wait that gave up in one warp (it raises the
// abort flag) stops all of them.  Returns false to stop.
__device__ __forceinline__ bool convert_wait(uint64_t* landed, uint32_t parity,
                                             volatile int* abort_flag, uint64_t wait_ns,
                                             int named_barrier, int threads) {
  mbar_wait(landed, parity, abort_flag, wait_ns);
  named_bar_sync(named_barrier, threads);
  return *abort_flag == 0;
}

// 2^60 * scale as bf16x2 (the scale is a power of two: its fp32 bits end in 16
// zeros), or 0 for a row past the sequence's end (which must not reach an MMA:
// its codes and scale may be anything).
__device__ __forceinline__ uint32_t fp8_row_factor(bool row_ok, float scale) {
  return row_ok ? (__float_as_uint(scale * 0x1p60f) >> 16) * 0x10001u : 0u;
}

// Widen one 128-byte row slot in place: its 64 E4M3 codes (bytes 64..127, as
// the TMA box landed them) become the 64 bf16 values code * scale over the
// whole slot, in the 128-byte-swizzled layout (16-byte unit u of row r at
// (u ^ (r % 8)) * 16); f_lo is fp8_row_factor of the row (see
// e4m3x2_to_bf16x2: every step is exact).  The four 16-byte loads start at
// unit (r mod 4), so the lanes of a warp spread over the banks.
__device__ __forceinline__ void widen_row_slot(uint8_t* slot, int r, uint32_t f_lo) {
  constexpr uint32_t f_hi = 0x5D805D80u;  // 2^60 in both halves
  uint4 v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    v[k] = *reinterpret_cast<const uint4*>(slot + 64 + 16 * ((k + r) & 3));
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int kk = (k + r) & 3;  // v[k] holds dims 16 kk .. 16 kk + 15 of the chunk
    uint4 lo, hi;
    lo.x = e4m3x2_to_bf16x2(v[k].x, 0x1404u, f_hi, f_lo);
    lo.y = e4m3x2_to_bf16x2(v[k].x, 0x3424u, f_hi, f_lo);
    lo.z = e4m3x2_to_bf16x2(v[k].y, 0x1404u, f_hi, f_lo);
    lo.w = e4m3x2_to_bf16x2(v[k].y, 0x3424u, f_hi, f_lo);
    hi.x = e4m3x2_to_bf16x2(v[k].z, 0x1404u, f_hi, f_lo);
    hi.y = e4m3x2_to_bf16x2(v[k].z, 0x3424u, f_hi, f_lo);
    hi.z = e4m3x2_to_bf16x2(v[k].w, 0x1404u, f_hi, f_lo);
    hi.w = e4m3x2_to_bf16x2(v[k].w, 0x3424u, f_hi, f_lo);
    *reinterpret_cast<uint4*>(slot + (((2 * kk) ^ (r & 7)) << 4)) = lo;
    *reinterpret_cast<uint4*>(slot + (((2 * kk + 1) ^ (r & 7)) << 4)) = hi;
  }
}

// The MMA-issuing roles run either on a whole warp (kWarp: every lane runs the
// loop, one elected lane issues each MMA and commit) or on lane 0 alone.
template <bool kWarp>
__device__ __forceinline__ bool issuer_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                            uint64_t limit_ns) {
  const bool ok = mbar_wait_cluster(bar, parity, abort, limit_ns);
  if constexpr (kWarp) return __all_sync(0xffffffffu, ok);
  return ok;
}
template <bool kWarp>
__device__ __forceinline__ void issue_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                         uint32_t acc) {
  if constexpr (kWarp) umma_bf16_ts_pair_warp(d, a, b, idesc, acc);
  else umma_bf16_ts_pair(d, a, b, idesc, acc);
}
template <bool kWarp>
__device__ __forceinline__ void issue_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t acc) {
  if constexpr (kWarp) umma_bf16_ss_pair_warp(d, a, b, idesc, acc);
  else umma_bf16_ss_pair(d, a, b, idesc, acc);
}
template <bool kWarp>
__device__ __forceinline__ void issue_commit(uint64_t* bar) {
  if constexpr (kWarp) umma_commit_pair_warp(bar);
  else umma_commit_pair(bar);
}

// Gathered rows: copy 32 cached rows (this lane holds the row index of row
// `lane`; -1 = a zero row) into a slot, chunks src_chunk .. src_chunk +
// nchunks - 1 of each row to chunks dst_chunk .. of the slot, in the
// 128-byte-swizzled layout of the TMA boxes.  Lane l copies 16-byte unit l % 8
// of rows 4 g + l / 8, g = 0..7, so that eight lanes read one 128-byte segment
// of a row.
__device__ __forceinline__ void gather_rows32(uint8_t* slot, int dst_chunk, int src_chunk,
                                              int nchunks, const void* cache, int my_row,
                                              int lane) {
  const int u = lane & 7;
#pragma unroll
  for (int grp = 0; grp < 8; ++grp) {
    const int r = 4 * grp + (lane >> 3);
    const int row = __shfl_sync(0xffffffffu, my_row, r);
    const uint8_t* src = static_cast<const uint8_t*>(cache) +
                         static_cast<int64_t>(row < 0 ? 0 : row) * (kDqk * 2) + src_chunk * 128 +
                         u * 16;
    uint8_t* dst = slot + dst_chunk * kHalfChunk + r * 128 + ((u ^ (r & 7)) << 4);
    for (int c = 0; c < nchunks; ++c)
      cp_async16_zfill(dst + c * kHalfChunk, src + c * 128, row >= 0);
  }
}

template <bool kGather, bool kFp8>
__global__ void __launch_bounds__(PairRoles<kFp8>::kThreads, 1)
mla_decode_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_kpart,
                       const __grid_constant__ CUtensorMap tm_vx,
                       const __grid_constant__ CUtensorMap tm_po,
                       const __grid_constant__ CUtensorMap tm_out, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  static_assert(!(kGather && kFp8), "gathered rows come from a bf16 cache");
  constexpr int kThreads = PairRoles<kFp8>::kThreads;
  constexpr int kTmaVWarp = PairRoles<kFp8>::kTmaVWarp;
  // full barriers of the K and V parts: one TMA-counted arrival (dense bf16
  // pages), or one arrival per CTA (gathered rows, copied by the threads; FP8
  // codes, widened by the converter warps)
  constexpr uint32_t kFullArrivals = (kGather || kFp8) ? 2 : 1;
  constexpr bool kWarpIssue = !kFp8;  // MMAs issued by whole warps (see the QK^T issuers)
  (void)kThreads;
  uint8_t* sq2 = smem + kOffQ2;
  uint8_t* sk = smem + kOffK;
  uint8_t* sp = smem + kOffP;
  float* sx = reinterpret_cast<float*>(smem + kOffX);
  float* sl = reinterpret_cast<float*>(smem + kOffL);
  float* sscale = reinterpret_cast<float*>(smem + kOffScale);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int worker = blockIdx.x >> 1, rb2 = blockIdx.y;
  const int row0 = rb2 * 128 + 64 * static_cast<int>(rank);  // first query row of this CTA
  const uint64_t wait_ns = p.wait_ns;  // limit of every bounded wait (normally kWaitLimitNs)

  // Set-up first: the kernel is launched as a programmatic dependent of the
  // scheduler kernel, so its CTAs may start while the scheduler runs; barriers
  // and tensor memory are made ready meanwhile, and the metadata is read only
  // after the dependency wait below.
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(&bar[kKFull0 + s], kFullArrivals);
      mbar_init(&bar[kVFull0 + s], kFullArrivals);
      mbar_init(&bar[kKEmpty0 + s], 1);
      mbar_init(&bar[kXFree0 + 2 * s], 1);
      mbar_init(&bar[kXFree0 + 2 * s + 1], 1);
    }
    mbar_init(&bar[kQFull], 1);
    mbar_init(&bar[kQEmpty], 2);  // one commit from each QK^T warp
    mbar_init(&bar[kSFull0], 1);
    mbar_init(&bar[kSFull1], 1);
    mbar_init(&bar[kPvDone0], 1);
    mbar_init(&bar[kPvDone1], 1);
    mbar_init(&bar[kOFull], 1);
    mbar_init(&bar[kSFree0], kSoftmaxArrivals);
    mbar_init(&bar[kSFree1], kSoftmaxArrivals);
    mbar_init(&bar[kPFull0], kSoftmaxArrivals);
    mbar_init(&bar[kPFull1], kSoftmaxArrivals);
    mbar_init(&bar[kQReady], kSoftmaxArrivals);
    mbar_init(&bar[kQStage], 1);
    mbar_init(&bar[kXBar], 32 * kSoftmaxWarps);
    mbar_init(&bar[kLBar], 32 * kSoftmaxWarps);
    for (int i = 0; i < 3; ++i) mbar_init(&bar[kDrain0 + i], 1);
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(&bar[kKLanded0 + s], 1);
      mbar_init(&bar[kVLanded0 + s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kQkEvenWarp) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kTmaKWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    if (!kGather) prefetch_tensormap(&tm_kpart);
  }
  if (warp == kTmaVWarp && lane == 0 && !kGather) prefetch_tensormap(&tm_vx);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers and tensor memory of both CTAs exist before either uses them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  grid_dependency_wait();  // the scheduler's metadata is complete and visible
  const int32_t* md = p.tile_md + static_cast<int64_t>(worker) * kMdStride;
  int npieces = md[5];
  if (npieces != 0 && (md[0] < 0 || npieces < 0 || md[0] + npieces > p.batch)) {
    if (threadIdx.x == 0 && rank == 0) report(p.status, MLA_ERR_DEVICE_CHECK);
    npieces = 0;
  }
  // An idle worker (or bad metadata) runs no role: both CTAs of the pair read
  // the same row and go straight to the common teardown.
  if constexpr (kFp8) {
    if (warp >= 8) setmaxnreg_dec<kFp8RegsConv>();
  }

  // Every role walks the same sequence of K-ring entries: per piece with pages,
  // two query-staging entries, then one entry per page.
  if (warp == kTmaKWarp) {
    // ------------------------------------------------------------ query rows + K parts
    // Dense pages: lane 0 issues one TMA box per page.  Gathered rows (kGather):
    // all 32 lanes copy the page's 32 rows of this CTA in 16-byte pieces, and a
    // page is signalled once two newer pages have been issued (up to three
    // pages of copies in flight), a piece's last pages at the piece's end.
    if (kGather || lane == 0) {
      // a wait of the lanes running this loop, with the same outcome in each
      auto wait = [&](uint64_t* b, uint32_t parity) {
        bool r = mbar_wait_cluster(b, parity, abort_flag, wait_ns);
        if constexpr (kGather) r = __all_sync(0xffffffffu, r);
        return r;
      };
      int entries = 0, qloads = 0;
      int pending[2] = {-1, -1};  // gather: slots of the two newest pages not yet signalled
      bool ok = true;
      for (int pc = 0; pc < npieces && ok; ++pc) {
        // dense pages: the block-table entry of the piece's first page, loaded
        // together with the piece's length (both follow from the metadata alone)
        const int32_t* bt = p.block_table + static_cast<int64_t>(md[0] + pc) * p.bt_stride;
        int page_next = 0;
        if constexpr (!kGather) {
          const int pg0 = pc == 0 ? md[1] : 0;
          page_next = __ldg(bt + (pg0 >= 0 && pg0 < p.bt_stride ? pg0 : 0));
        }
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (lane == 0 && rank == 0 && p.seqlens[pz.seq] > p.bt_stride * kPage)
          report(p.status, MLA_ERR_DEVICE_CHECK);
        if (pz.npg == 0) continue;
        const int qrow = pz.seq * p.rows + row0;
        // dims 384..575 of the query rows: shared memory, counted on the leader
        if (qloads > 0) {
          ok = wait(&bar[kQEmpty], (qloads - 1) & 1);
          if (!ok) break;
        }
        if (lane == 0) {
          if (rank == 0) mbar_arrive_expect_tx(&bar[kQFull], 2 * kQ2Bytes);
          for (int c = 0; c < kQSmemChunks; ++c)
            tma_load_2d_pair(sq2 + c * kChunk, &tm_q, (kQTmemChunks + c) * 64, qrow,
                             &bar[kQFull]);
        }
        ++qloads;
        // dims 0..383: two staging entries of the K ring, counted on this CTA's barrier
        for (int e = 0; e < 2; ++e) {
          const int slot = entries % kKSlots, use = entries / kKSlots;
          if (use > 0) ok = wait(&bar[kKEmpty0 + slot], (use - 1) & 1);
          if (!ok) break;
          if (lane == 0) {
            if (e == 0) mbar_arrive_expect_tx(&bar[kQStage], kQTmemChunks * kChunk);
            uint8_t* dst = sk + slot * kKBytes;
            const int c0 = e == 0 ? 0 : kQStageA, c1 = e == 0 ? kQStageA : kQTmemChunks;
            for (int c = c0; c < c1; ++c)
              tma_load_2d(dst + (c - c0) * kChunk, &tm_q, c * 64, qrow, &bar[kQStage]);
            // the leader's full barrier of the slot completes one phase per entry
            if (rank == 0)
              for (int a = 0; a < kFullArrivals; ++a) mbar_arrive(&bar[kKFull0 + slot]);
          }
          ++entries;
        }
        if (!ok) break;
        // gather: row of this lane's token (tokens 32 rank .. 32 rank + 31) of a
        // piece page, loaded one page ahead of its copies
        const int cnt = kGather ? p.seqlens[pz.seq] : 0;
        const int32_t* grows =
            kGather ? p.gather_rows + static_cast<int64_t>(pz.seq) * p.gather_stride : nullptr;
        auto row_of = [&](int jj) {
          const int vt0 = (pz.pg0 + jj) * kPage;
          const int tok = vt0 + 32 * static_cast<int>(rank) + lane;
          return tok < cnt ? __ldg(grows + tok) : -1;  // past the count: a zero row
        };
        int next_row = kGather ? row_of(0) : 0;
        for (int j = 0; j < pz.npg && ok; ++j, ++entries) {
          const int slot = entries % kKSlots, use = entries / kKSlots;
          if constexpr (kGather) {
            const int my_row = next_row;
            if (j + 1 < pz.npg) next_row = row_of(j + 1);
            if (use > 0) {
              ok = wait(&bar[kKEmpty0 + slot], (use - 1) & 1);
              if (!ok) break;
            }
            gather_rows32(sk + slot * kKBytes, 0, 0, kChunks, p.gather_cache, my_row, lane);
            cp_async_commit();
            // two pages of copies stay in flight behind the newest: signal the
            // page issued two pages ago once its copies have landed
            if (pending[0] >= 0) {
              cp_async_wait_group<2>();
              fence_proxy_async_smem();
              warp_arrive_leader(&bar[kKFull0 + pending[0]], rank, lane);
            }
            pending[0] = pending[1];
            pending[1] = slot;
            if (j + 1 == pz.npg) {
              // the piece's last pages: signal them now (the next piece's query rows
              // reach the MMAs only after this piece is finished)
              cp_async_wait_group<0>();
              fence_proxy_async_smem();
              for (int k = 0; k < 2; ++k)
                if (pending[k] >= 0) warp_arrive_leader(&bar[kKFull0 + pending[k]], rank, lane);
              pending[0] = pending[1] = -1;
            }
          } else if constexpr (kFp8) {
            // FP8 codes of this CTA's 32 tokens, one box of 128 bytes x 32 rows x
            // 9 chunks through a view whose chunks are 64 bytes apart, started at
            // x = -64: each chunk's codes land in bytes 64..127 of its 128-byte
            // row slots (bytes 0..63 are zeros, overwritten when the converters
            // widen the slot); plus the page's 64 scales.  Both count on this
            // CTA's K-landed barrier; the converters signal the leader's full
            // barrier.
            int page = page_next;
            if (j + 1 < pz.npg) page_next = __ldg(bt + pz.pg0 + j + 1);
            // the tensor map bounds the codes, but the untiled scale copy has no
            // bounds: a page id outside the cache is reported and replaced
            if (page < 0 || page >= p.num_blocks) {
              report(p.status, MLA_ERR_DEVICE_CHECK);
              page = 0;
            }
            if (use > 0) {
              ok = wait(&bar[kKEmpty0 + slot], (use - 1) & 1);
              if (!ok) break;
            }
            uint64_t* landed = &bar[kKLanded0 + slot];
            const int row = page * kPage + 32 * static_cast<int>(rank);
            mbar_arrive_expect_tx(landed, kChunks * kHalfChunk + kPage * 4);
            tma_load_3d(sk + slot * kKBytes, &tm_kpart, -64, row, 0, landed);
            // all 64 tokens' scales: the softmax applies them to both halves of S
            bulk_load(sscale + slot * kPage, p.kscale + static_cast<int64_t>(page) * kPage,
                      kPage * 4, landed);
          } else {
            // this page's entry was loaded one page ahead; load the next one
            // before waiting for the slot
            const int page = page_next;
            if (j + 1 < pz.npg) page_next = __ldg(bt + pz.pg0 + j + 1);
            if (use > 0) {
              ok = wait(&bar[kKEmpty0 + slot], (use - 1) & 1);
              if (!ok) break;
            }
            // the slot's previous entry is consumed, so the leader's full barrier is
            // in the phase of this entry
            if (rank == 0) mbar_arrive_expect_tx(&bar[kKFull0 + slot], 2 * kKBytes);
            // one box: this CTA's 32 token rows x all nine chunks
            tma_load_3d_pair(sk + slot * kKBytes, &tm_kpart, 0,
                             page * kPage + 32 * static_cast<int>(rank), 0,
                             &bar[kKFull0 + slot]);
          }
        }
      }
      if constexpr (kGather) {
        // no copy may still be in flight when the CTA releases its shared memory
        // (after an abort the loop may have left pages unsignalled; nothing reads them)
        cp_async_wait_group<0>();
      }
    }
  } else if (warp == kTmaVWarp) {
    // ------------------------------------------------------------ peer-token values
    // CTA 0 replaces chunks 4..7 of each page's slot with tokens 32..63 x dims
    // 0..255, CTA 1 chunks 0..3 with tokens 0..31 x dims 256..511, each once the
    // QK^T MMAs have read the chunks being replaced (of both CTAs: one commit).
    // Dense pages: one TMA box (lane 0).  Gathered rows: all lanes copy the
    // peer tokens' rows and signal the page once their copies have landed.
    if (kGather || lane == 0) {
      const int xgrp = rank == 0 ? 1 : 0;
      const int dst_chunk = rank == 0 ? kXChunks : 0;
      const int src_row = rank == 0 ? 32 : 0, src_chunk = rank == 0 ? 0 : kXChunks;
      int entries = 0;
      uint32_t xbits = 0;  // parity of the next phase of each slot's X-free barrier
      bool ok = true;
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (pz.npg == 0) continue;
        entries += 2;  // the piece's query staging entries
        for (int j = 0; j < pz.npg; ++j, ++entries) {
          const int slot = entries % kKSlots;
          int my_row = 0;
          if constexpr (kGather) {
            const int vt0 = (pz.pg0 + j) * kPage, cnt = p.seqlens[pz.seq];
            const int32_t* rows = p.gather_rows + static_cast<int64_t>(pz.seq) * p.gather_stride;
            const int tok = vt0 + src_row + lane;
            my_row = tok < cnt ? __ldg(rows + tok) : -1;  // past the count: a zero row
          }
          ok = mbar_wait_cluster(&bar[kXFree0 + 2 * slot + xgrp], (xbits >> slot) & 1u, abort_flag,
                                 wait_ns);
          if constexpr (kGather) ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          xbits ^= 1u << slot;
          if constexpr (kGather) {
            gather_rows32(sk + slot * kKBytes, dst_chunk, src_chunk, kXChunks, p.gather_cache,
                          my_row, lane);
            cp_async_commit();
            cp_async_wait_group<0>();
            fence_proxy_async_smem();
            warp_arrive_leader(&bar[kVFull0 + slot], rank, lane);
          } else if constexpr (kFp8) {
            // FP8: the four chunks' codes (one box, as for the K parts) on this
            // CTA's V-landed barrier; the value converters widen them and signal
            // the leader's V barrier (the page's scales came with the K part)
            const int32_t* bt = p.block_table + static_cast<int64_t>(pz.seq) * p.bt_stride;
            const int page = __ldg(bt + pz.pg0 + j);
            uint64_t* landed = &bar[kVLanded0 + slot];
            const int row = page * kPage + src_row;
            mbar_arrive_expect_tx(landed, kXChunks * kHalfChunk);
            tma_load_3d(sk + slot * kKBytes + dst_chunk * kHalfChunk, &tm_vx, -64, row, src_chunk,
                        landed);
          } else {
            const int32_t* bt = p.block_table + static_cast<int64_t>(pz.seq) * p.bt_stride;
            const int page = __ldg(bt + pz.pg0 + j);
            // the PV of the slot's previous page is done (its K part was reloaded
            // after it), so the leader's V barrier is in the phase of this page
            if (rank == 0) mbar_arrive_expect_tx(&bar[kVFull0 + slot], 2 * kXBytes);
            tma_load_3d_pair(sk + slot * kKBytes + dst_chunk * kHalfChunk, &tm_vx, 0,
                             page * kPage + src_row, src_chunk, &bar[kVFull0 + slot]);
          }
        }
      }
      if constexpr (kGather) cp_async_wait_group<0>();
    }
  } else if (kFp8 && warp >= kKConvWarp0 && warp < kTmaVWarp) {
    // ------------------------------------------------------------ FP8: K-part converters
    // Two groups of four warps widen the K parts of even and odd pages, so two
    // pages are widened at once.  In a group, thread t owns row r = t % 32 of
    // chunks t / 32, t / 32 + 4, ... (3 or 2 of the 9); the group signals the
    // leader's full barrier once per page (one arrival per CTA).
    const int group = (warp - kKConvWarp0) / 4;
    const int ct = threadIdx.x - (kKConvWarp0 + 4 * group) * 32;
    const int r = ct & 31, c0 = ct >> 5;
    const int named = kKConvBarrier0 + group;
    int entries = 0, pages = 0;
    uint32_t landed_parity = 0;  // per slot: K parts landed there (mod 2), both groups'
    for (int pc = 0; pc < npieces; ++pc) {
      const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
      if (pz.npg == 0) continue;
      const int L = p.seqlens[pz.seq];
      entries += 2;  // the query staging entries go straight to the consumers
      bool stop = false;
      for (int j = 0; j < pz.npg; ++j, ++entries) {
        const int slot = entries % kKSlots;
        const uint32_t parity = (landed_parity >> slot) & 1;
        landed_parity ^= 1u << slot;
        if (((pages + j) % kKConvGroups) != group) continue;
        if (!convert_wait(&bar[kKLanded0 + slot], parity, abort_flag, wait_ns, named,
                          kKConvThreads)) {
          stop = true;
          break;
        }
        uint8_t* row_slot = sk + slot * kKBytes + r * 128;
        const int tok = 32 * static_cast<int>(rank) + r;  // this CTA's token of the page
        const uint32_t f_lo =
            fp8_row_factor((pz.pg0 + j) * kPage + tok < L, sscale[slot * kPage + tok]);
        for (int c = c0; c < kChunks; c += 4) widen_row_slot(row_slot + c * kHalfChunk, r, f_lo);
        fence_proxy_async_smem();  // the MMAs read the slot through the async proxy
        named_bar_sync(named, kKConvThreads);
        if (ct == 0) {
          if (rank == 0)
            mbar_arrive(&bar[kKFull0 + slot]);
          else
            mbar_arrive_remote(&bar[kKFull0 + slot], 0);
        }
      }
      if (stop) break;
      pages += pz.npg;
    }
  } else if (kFp8 && warp >= kVConvWarp0) {
    // ------------------------------------------------------------ FP8: value converters
    // Widen the peer tokens' value chunks: 4 chunks x 32 rows, row slot i
    // (row i % 32 of chunk i / 32) for i = t and t + 96.  The tokens' scales
    // came with this CTA's K part: its landed barrier (still in this page's
    // phase: the slot is not reloaded before PV of the page, which waits for
    // these converters) makes them visible here.
    const int ct = threadIdx.x - kVConvWarp0 * 32;
    const int dst_chunk = rank == 0 ? kXChunks : 0;
    const int src_row = rank == 0 ? 32 : 0;
    int entries = 0;
    uint32_t landed_parity = 0, k_parity = 0;
    for (int pc = 0; pc < npieces; ++pc) {
      const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
      if (pz.npg == 0) continue;
      const int L = p.seqlens[pz.seq];
      entries += 2;
      bool stop = false;
      for (int j = 0; j < pz.npg; ++j, ++entries) {
        const int slot = entries % kKSlots;
        const uint32_t parity = (landed_parity >> slot) & 1, kpar = (k_parity >> slot) & 1;
        landed_parity ^= 1u << slot;
        k_parity ^= 1u << slot;
        mbar_wait(&bar[kKLanded0 + slot], kpar, abort_flag, wait_ns);
        if (!convert_wait(&bar[kVLanded0 + slot], parity, abort_flag, wait_ns, kVConvBarrier,
                          kVConvThreads)) {
          stop = true;
          break;
        }
        for (int i = ct; i < kXChunks * 32; i += kVConvThreads) {
          const int r = i & 31;
          const uint32_t f_lo = fp8_row_factor((pz.pg0 + j) * kPage + src_row + r < L,
                                               sscale[slot * kPage + src_row + r]);
          widen_row_slot(sk + slot * kKBytes + (dst_chunk + (i >> 5)) * kHalfChunk + r * 128, r,
                         f_lo);
        }
        fence_proxy_async_smem();
        named_bar_sync(kVConvBarrier, kVConvThreads);
        if (ct == 0) {
          if (rank == 0)
            mbar_arrive(&bar[kVFull0 + slot]);
          else
            mbar_arrive_remote(&bar[kVFull0 + slot], 0);
        }
      }
      if (stop) break;
    }
  } else if (warp == kQkEvenWarp || warp == kQkOddWarp) {
    // ------------------------------------------------------------ QK^T issuers (leader)
    // With a bf16 cache each warp issues as a whole (every lane runs the loop,
    // one elected lane issues each MMA and commit): about one MMA per 27 cycles
    // against 60 for a single thread.  The FP8 variant issues from lane 0 (with
    // its fewer registers the whole-warp form measured slower).  Even and odd
    // pages (one S buffer each) come from two warps so the tensor core stays fed.
    if (rank == 0 && (kWarpIssue || lane == 0)) {
      const int parity = warp == kQkEvenWarp ? 0 : 1;
      int entries = 0, pages = 0, qloads = 0;
      bool ok = true;
      const uint32_t q2_base = smem_addr(sq2), k_base = smem_addr(sk);
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (pz.npg == 0) continue;
        const int stage_a = entries % kKSlots, stage_b = (entries + 1) % kKSlots;
        entries += 2;
        ok = issuer_wait<kWarpIssue>(&bar[kQFull], qloads & 1, abort_flag, wait_ns) &&
             issuer_wait<kWarpIssue>(&bar[kQReady], qloads & 1, abort_flag, wait_ns);
        ++qloads;
        if (!ok) break;
        tc_fence_after();
        if (parity == 0) {  // both CTAs hold Q in tensor memory: the staging slots are free
          issue_commit<kWarpIssue>(&bar[kKEmpty0 + stage_a]);
          issue_commit<kWarpIssue>(&bar[kKEmpty0 + stage_b]);
        }
        for (int j = 0; j < pz.npg && ok; ++j) {
          const int g = pages + j, b = g & 1, entry = entries + j;
          if (b != parity) continue;
          if (g >= 2) {  // both CTAs' softmax have read S of page g - 2 from buffer b
            ok = issuer_wait<kWarpIssue>(&bar[kSFree0 + b], ((g >> 1) - 1) & 1, abort_flag,
                                   wait_ns);
            if (!ok) break;
          }
          const int slot = entry % kKSlots;
          ok = issuer_wait<kWarpIssue>(&bar[kKFull0 + slot], (entry / kKSlots) & 1, abort_flag,
                                 wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint64_t b0 = smem_desc_sw128(k_base + slot * kKBytes, 16, 1024);
          const uint64_t a2 = smem_desc_sw128(q2_base, 16, 1024);
          const uint32_t d = tmem + kTmemS + 32 * b;
          if constexpr (kFp8) {
            // the same K-steps, one chunk (four K-steps) per iteration: the
            // fully unrolled form below needs more registers than the FP8
            // kernel's issuing warps have (descriptor addresses count 16-byte
            // units)
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
              const uint64_t bc = b0 + static_cast<uint32_t>((c * kHalfChunk) >> 4);
              if (c < kQTmemChunks) {
                const uint32_t ac = tmem + kTmemQ + 32 * c;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  issue_ts<kWarpIssue>(d, ac + 8 * k, bc + 2 * k, kIdescQK, (c | k) != 0 ? 1u : 0u);
              } else {
                const uint64_t ac = a2 + static_cast<uint32_t>(((c - kQTmemChunks) * kChunk) >> 4);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  issue_ss<kWarpIssue>(d, ac + 2 * k, bc + 2 * k, kIdescQK, 1u);
              }
              // chunks 0..3 / 4..7 of the slot read: the peer-token values may land there
              if (4 * c + 3 == kXDoneStep0) issue_commit<kWarpIssue>(&bar[kXFree0 + 2 * slot]);
              if (4 * c + 3 == kXDoneStep1) issue_commit<kWarpIssue>(&bar[kXFree0 + 2 * slot + 1]);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kQKSteps; ++kk) {
              // K-step kk: swizzle block kk/4, 32-byte step kk%4 inside it
              const uint32_t boff = ((kk >> 2) * kHalfChunk + (kk & 3) * 32) >> 4;
              if (kk < kQTmemKSteps) {
                issue_ts<kWarpIssue>(d, tmem + kTmemQ + 8 * kk, b0 + boff, kIdescQK,
                                  kk > 0 ? 1u : 0u);
              } else {
                const int k2 = kk - kQTmemKSteps;
                const uint32_t aoff = ((k2 >> 2) * kChunk + (k2 & 3) * 32) >> 4;
                issue_ss<kWarpIssue>(d, a2 + aoff, b0 + boff, kIdescQK, 1u);
              }
              // chunks 0..3 / 4..7 of the slot read: the peer-token values may land there
              if (kk == kXDoneStep0) issue_commit<kWarpIssue>(&bar[kXFree0 + 2 * slot]);
              if (kk == kXDoneStep1) issue_commit<kWarpIssue>(&bar[kXFree0 + 2 * slot + 1]);
            }
          }
          issue_commit<kWarpIssue>(&bar[kSFull0 + b]);
        }
        if (!ok) break;
        issue_commit<kWarpIssue>(&bar[kQEmpty]);  // this warp's reads of Q for the piece are done
        entries += pz.npg;
        pages += pz.npg;
      }
    }
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ PV issuer (leader)
    if (rank == 0 && (kWarpIssue || lane == 0)) {  // as for QK^T
      int pages = 0, entries = 0;
      uint32_t vbits = 0;  // parity of the next phase of each slot's V barrier
      bool ok = true;
      const uint32_t k_base = smem_addr(sk), p_base = smem_addr(sp);
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (pz.npg == 0) continue;
        entries += 2;  // the piece's query staging entries
        for (int j = 0; j < pz.npg; ++j, ++entries) {
          const int g = pages + j, slot = entries % kKSlots, pb = g & 1;
          ok = issuer_wait<kWarpIssue>(&bar[kPFull0 + pb], (g >> 1) & 1, abort_flag, wait_ns);
          if (!ok) break;
          // test hook: a wait that nothing ends, with copies and MMAs in flight
          if (g == 0 && p.stall_flag != nullptr) {
            ok = flag_wait(p.stall_flag, abort_flag, wait_ns);
            if constexpr (kWarpIssue) ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          }
          ok = issuer_wait<kWarpIssue>(&bar[kVFull0 + slot], (vbits >> slot) & 1u, abort_flag,
                                 wait_ns);
          if (!ok) break;
          vbits ^= 1u << slot;
          tc_fence_after();
          const uint32_t st = k_base + slot * kKBytes;
          const uint32_t pt = p_base + pb * kPBytes;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int kk = 0; kk < kPage / 16; ++kk) {
              // tokens 16kk..16kk+15: chunk block 0..3 (tokens 0..31) or 4..7
              // (tokens 32..63) of the slot, 16 rows of 128 bytes per K-step;
              // this CTA's 128 dv of MMA h are chunks 2h, 2h + 1 of the block
              // (LBO = one 32-row chunk, SBO = 8 rows)
              const uint32_t vaddr = st + ((kk >> 1) * kXChunks + 2 * h) * kHalfChunk +
                                     (kk & 1) * 2048;
              issue_ss<kWarpIssue>(tmem + kTmemO + 128 * h, smem_desc_sw128(pt + kk * 32, 16, 1024),
                                smem_desc_sw128(vaddr, kHalfChunk, 1024), kIdescPV,
                                (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          issue_commit<kWarpIssue>(&bar[kKEmpty0 + slot]);
          issue_commit<kWarpIssue>(&bar[kPvDone0 + pb]);
        }
        if (!ok) break;
        issue_commit<kWarpIssue>(&bar[kOFull]);
        pages += pz.npg;
      }
    }
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax / epilogue
    if constexpr (kFp8) setmaxnreg_inc<kFp8RegsSoftmax>();
    const int L = 32 * warp + lane;       // TMEM lane
    const int r = L & 63;                 // row within this CTA's 64
    const int th = L >> 6;                // which half of the 64 tokens / of each dv 256-block
    const int row = row0 + r;             // row within the sequence's query rows
    const bool row_ok = row < p.rows;
    const int jq = row_ok ? row / p.h_q : 0, hq = row_ok ? row % p.h_q : 0;
    const uint32_t quarter = static_cast<uint32_t>(32 * warp) << 16;
    int entries = 0, pages = 0, pieces_done = 0, qcopies = 0;
    bool ok = true;
    bool q_copied_ahead = false;
    for (int pc = 0; pc < npieces && ok; ++pc) {
      const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
      const int Lseq = p.seqlens[pz.seq];
      const int cap_tokens =
          static_cast<int>(p.bt_stride * kPage < Lseq ? p.bt_stride * kPage : Lseq);
      int lim = p.causal ? Lseq - p.s_q + jq + 1 : Lseq;
      lim = lim < 0 ? 0 : (lim < cap_tokens ? lim : cap_tokens);
      const int base_split = p.num_splits[pz.seq];
      const int k_pieces = p.num_splits[pz.seq + 1] - base_split;
      const int64_t slot = static_cast<int64_t>(base_split) + pz.split_idx;
      float m = -INFINITY, l = 0.f;

      if (pz.npg > 0) {
        if (!q_copied_ahead) {
          ok = copy_query_rows(sk, bar, abort_flag, tmem + quarter + kTmemQ, r, rank, lane, entries,
                               qcopies, wait_ns);
          if (!ok) break;
        }
        q_copied_ahead = false;
        for (int j = 0; j < pz.npg; ++j) {
          const int g = pages + j, pb = g & 1;
          ok = warp_wait_cluster(&bar[kSFull0 + pb], (g >> 1) & 1, abort_flag, wait_ns);
          if (!ok) break;
          tc_fence_after();
          uint32_t s[32];
          tmem_ld32(tmem + quarter + kTmemS + 32 * pb, s);
          tmem_ld_wait(s);
          tc_fence_before();
          warp_arrive_leader(&bar[kSFree0 + pb], rank, lane);
          const int nv = lim - (pz.pg0 + j) * kPage - 32 * th;
          float x[32];
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = c < nv ? __uint_as_float(s[c]) * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, x[c]);
          }
          // the other half of the row is in lane L ^ 64
          float* xb = sx + pb * 128;
          xb[th * 64 + r] = mx;
          mbar_arrive(&bar[kXBar]);
          ok = warp_wait_cluster(&bar[kXBar], g & 1, abort_flag, wait_ns);
          if (!ok) break;
          mx = fmaxf(mx, xb[(th ^ 1) * 64 + r]);
          float alpha = 1.f;
          if (mx > m + kRescaleThreshold) {
            alpha = ex2_approx(m - mx);
            m = mx;
          }
          float sum = 0.f;
          uint32_t pw[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = x[c] == -INFINITY ? 0.f : ex2_approx(x[c] - m);
            const float p1 = x[c + 1] == -INFINITY ? 0.f : ex2_approx(x[c + 1] - m);
            sum += p0 + p1;
            pw[c >> 1] = pack_bf16x2(p0, p1);
          }
          l = l * alpha + sum;
          // O is rescaled only once PV of the previous page is done; the first
          // PV of a piece overwrites O, so its page needs no rescale.
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            ok = warp_wait_cluster(&bar[kPvDone0 + ((g - 1) & 1)], ((g - 1) >> 1) & 1,
                                   abort_flag, wait_ns);
            if (!ok) break;
            tc_fence_after();
            for (int cb = 0; cb < 256; cb += 16) {
              uint32_t o[16];
              tmem_ld32x16(tmem + quarter + kTmemO + cb, o);
              tmem_ld_wait16(o);
#pragma unroll
              for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st32x16(tmem + quarter + kTmemO + cb, o);
            }
            tmem_st_wait();
          }
          // P buffer pb was last read by PV of page g - 2
          if (g >= 2) {
            ok = warp_wait_cluster(&bar[kPvDone0 + pb], ((g >> 1) - 1) & 1, abort_flag, wait_ns);
            if (!ok) break;
          }
          // P row r, tokens 32 th .. 32 th + 31: 16-byte units 4 th .. 4 th + 3 (swizzled)
          uint8_t* prow = sp + pb * kPBytes + r * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int u = 4 * th + i;
            *reinterpret_cast<uint4*>(prow + ((u ^ (r & 7)) << 4)) =
                make_uint4(pw[4 * i], pw[4 * i + 1], pw[4 * i + 2], pw[4 * i + 3]);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          warp_arrive_leader(&bar[kPFull0 + pb], rank, lane);
        }
        if (!ok) break;
        ok = warp_wait_cluster(&bar[kOFull], pieces_done & 1, abort_flag, wait_ns);
        ++pieces_done;
        entries += pz.npg;
        pages += pz.npg;
        if (!ok) break;
        tc_fence_after();
        // The next piece with pages gets its query rows now, so that its QK^T
        // runs while this piece's epilogue drains O.
        for (int pn = pc + 1; pn < npieces; ++pn) {
          if (piece_of(md, pn, p.seqlens, p.bt_stride).npg > 0) {
            ok = copy_query_rows(sk, bar, abort_flag, tmem + quarter + kTmemQ, r, rank, lane,
                                 entries, qcopies, wait_ns);
            q_copied_ahead = true;
            break;
          }
        }
        if (!ok) break;
      }
      // ---- epilogue: sums of the two row halves, then O / l.  Each warp owns
      // rows 32 (warp & 1) .. +31 of this CTA and dv half `th` of each 256-wide
      // block.  Blocks go TMEM -> registers -> shared memory (the P buffers,
      // idle until this piece's output is written, or the idle ring after the
      // CTA's last piece; 16-byte units XOR-swizzled by row, so neither side has
      // bank conflicts) -> global memory: by TMA store
      // for fp32 partials and for the bf16 output of the CTA's last piece, by
      // the load/store units (one contiguous row segment per instruction) for
      // the bf16 output of an earlier piece.
      float* lb = sl + (pc & 1) * 128;
      lb[th * 64 + r] = l;
      mbar_arrive(&bar[kLBar]);
      ok = warp_wait_cluster(&bar[kLBar], pc & 1, abort_flag, wait_ns);
      if (!ok) break;
      const float lt = l + lb[(th ^ 1) * 64 + r];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      float* stg = reinterpret_cast<float*>(sp) + warp * 1024;
      const int wrow0 = row0 + 32 * (warp & 1);  // sequence row of this warp's lane 0
      // The dependent grid (the split combine) may be scheduled once every CTA
      // has reached its last epilogue; it still waits for this grid's end
      // before it reads anything, and a step without splits ends it at once.
      if (pc == npieces - 1 && threadIdx.x == 0) grid_launch_dependents();
      if (k_pieces == 1 && pc == npieces - 1) {
        // bf16 output of this CTA's last piece: blocks of 32 rows x 64 dv columns
        // (128 bytes per row), one TMA store each (rows past the sequence's query
        // rows fall outside the map and are not written).  Only the last piece:
        // earlier, TMA stores would queue with the next piece's page loads.  The
        // ring is idle by now (every load landed and every MMA that read it is
        // done), so each block gets its own 4 KB staging buffer there and the
        // four stores of a warp go out back to back.
        for (int h = 0; h < 2; ++h) {
          for (int cb = 0; cb < 128; cb += 64) {
            const int col = 128 * h + 256 * th + cb;
            float* stg_blk = reinterpret_cast<float*>(sk) + (warp * 4 + 2 * h + cb / 64) * 1024;
            uint32_t w[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t o[32];
              if (pz.npg > 0) {
                tmem_ld32(tmem + quarter + kTmemO + 128 * h + cb + 32 * half, o);
                tmem_ld_wait(o);
              } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) o[k] = 0u;
              }
#pragma unroll
              for (int k = 0; k < 16; ++k)
                w[16 * half + k] = pack_bf16x2(__uint_as_float(o[2 * k]) * inv,
                                               __uint_as_float(o[2 * k + 1]) * inv);
            }
            // row `lane` -> 16-byte unit u ^ (lane & 7) of staging row `lane` (the
            // layout of a 128-byte-swizzled TMA box of 32 rows x 64 bf16)
            uint4* srow = reinterpret_cast<uint4*>(stg_blk + lane * 32);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              srow[u ^ (lane & 7)] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tm_out, stg_blk, col, wrow0, pz.seq);
              tma_store_commit();
            }
            __syncwarp();
          }
        }
      } else {
        const int64_t orow0 = static_cast<int64_t>(pz.seq) * p.rows + wrow0;
        for (int h = 0; h < 2; ++h) {
          for (int cb = 0; cb < 128; cb += 32) {
            const int col = 128 * h + 256 * th + cb;
            uint32_t o[32];
            if (pz.npg > 0) {
              tmem_ld32(tmem + quarter + kTmemO + 128 * h + cb, o);
              tmem_ld_wait(o);
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = 0u;
            }
            // the TMA store of the previous block has read the staging buffer
            if (lane == 0) tma_store_wait_read();
            __syncwarp();
            // row `lane` -> 16-byte unit u ^ (lane & 7) of staging row `lane` (the
            // layout of a 128-byte-swizzled TMA box of 32 rows x 32 fp32)
            float4* srow = reinterpret_cast<float4*>(stg + lane * 32);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              srow[u ^ (lane & 7)] = make_float4(
                  __uint_as_float(o[4 * u]) * inv, __uint_as_float(o[4 * u + 1]) * inv,
                  __uint_as_float(o[4 * u + 2]) * inv, __uint_as_float(o[4 * u + 3]) * inv);
            __syncwarp();
            if (k_pieces == 1) {
              // bf16 output of an earlier piece, through the load/store units: row
              // i of the block per instruction, lane l holding column l; eight
              // rows at a time, the shared loads back to back, then the stores
              const int sw_unit = lane >> 2, sw_word = lane & 3;
              const float* scol = stg + sw_word;
              for (int i0 = 0; i0 < 32; i0 += 8) {
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = scol[(i0 + i) * 32 + ((sw_unit ^ i) << 2)];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float w = __shfl_down_sync(0xffffffffu, v[i], 1);
                  if ((lane & 1) == 0 && wrow0 + i0 + i < p.rows)
                    *reinterpret_cast<uint32_t*>(p.out + (orow0 + i0 + i) * kDv + col + lane) =
                        pack_bf16x2(v[i], w);
                }
              }
            } else {
              // fp32 partial: one TMA store of the block (rows past the sequence's
              // query rows fall outside the map and are not written)
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(&tm_po, stg, col, wrow0, static_cast<int32_t>(slot));
                tma_store_commit();
              }
            }
            __syncwarp();
          }
        }
      }
      // the P buffers are the staging area: their last store must have read them
      // before the next piece writes P
      if (lane == 0) tma_store_wait_read();
      __syncwarp();
      if (row_ok && th == 0) {
        const float lse = lt > 0.f ? (m + lg2_approx(lt)) * 0.69314718055994531f : -INFINITY;
        if (k_pieces == 1)
          p.lse[(static_cast<int64_t>(pz.seq) * p.h_q + hq) * p.s_q + jq] = lse;
        else
          p.part_lse[slot * p.rows + row] = lse;
      }
    }
  }

  // The stores have read their staging buffers before the CTA exits; their
  // writes complete with the grid (the combine kernel and the host see them
  // after its end).
  if (warp < kSoftmaxWarps && lane == 0) tma_store_wait_read();
  // After an abort, work this CTA issued may still be in flight: pair MMAs of the
  // leader's issuing threads (each waits for its own to complete, through a
  // commit), and TMA loads of either CTA (they cannot be cancelled and land
  // within microseconds; a grace period covers them).  Both must be done before
  // the shared and tensor memory they write is released at the exit.
  if (*abort_flag) {
    if (rank == 0 && warp >= kQkEvenWarp && warp <= kQkOddWarp) {
      // the lane that issued the MMAs commits (the elected one of a whole warp)
      uint64_t* db = &bar[kDrain0 + (warp - kQkEvenWarp)];
      __syncwarp();
      if constexpr (kWarpIssue) {
        umma_commit_leader_warp(db);
        mbar_wait_drain(db, 0, kWaitLimitNs);
      } else if (lane == 0) {
        umma_commit_leader(db);
        mbar_wait_drain(db, 0, kWaitLimitNs);
      }
    }
    if (threadIdx.x == 0) abort_grace();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no pair MMA still writes either CTA's tensor memory
  if (*abort_flag && threadIdx.x == 0) report(p.status, MLA_ERR_DEVICE_TIMEOUT);
  if (warp == kQkEvenWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}


// Shared memory attribute of the three variants (once per device), and the
// register count the FP8 variant's setmaxnreg split relies on: with fewer
// registers at launch than its warpgroups ask for in all, the softmax
// warpgroup's increase could never be granted.
cudaError_t configure_pair_kernels() {
  static std::atomic<bool> configured[64];  // per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (configured[dev].load(std::memory_order_acquire)) return cudaSuccess;
  const void* kernels[3] = {reinterpret_cast<const void*>(mla_decode_pair_kernel<false, false>),
                            reinterpret_cast<const void*>(mla_decode_pair_kernel<true, false>),
                            reinterpret_cast<const void*>(mla_decode_pair_kernel<false, true>)};
  for (const void* k : kernels) {
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  cudaFuncAttributes fa{};
  e = cudaFuncGetAttributes(&fa, kernels[2]);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kFp8LaunchRegs) return cudaErrorInvalidConfiguration;
  configured[dev].store(true, std::memory_order_release);
  return cudaSuccess;
}

template <bool kGather, bool kFp8>
cudaError_t launch_pair(const CUtensorMap& tm_q, const CUtensorMap& tm_kpart,
                        const CUtensorMap& tm_vx, const CUtensorMap& tm_po,
                        const CUtensorMap& tm_out, const DecodeParams& p, int num_workers,
                        cudaStream_t stream) {
  cudaError_t e = configure_pair_kernels();
  if (e != cudaSuccess) return e;
  const int blocks128 = (p.rows + 127) / 128;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * num_workers, blocks128, 1);
  cfg.blockDim = dim3(PairRoles<kFp8>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, mla_decode_pair_kernel<kGather, kFp8>, tm_q, tm_kpart, tm_vx,
                         tm_po, tm_out, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_pair(const CUtensorMap& tm_q, const CUtensorMap& tm_kpart,
                               const CUtensorMap& tm_vx, const CUtensorMap& tm_po,
                               const CUtensorMap& tm_out, const DecodeParams& p, int num_workers,
                               cudaStream_t stream) {
  if (p.gather_rows != nullptr)
    return launch_pair<true, false>(tm_q, tm_kpart, tm_vx, tm_po, tm_out, p, num_workers, stream);
  return launch_pair<false, false>(tm_q, tm_kpart, tm_vx, tm_po, tm_out, p, num_workers, stream);
}

cudaError_t launch_decode_pair_fp8(const CUtensorMap& tm_q, const CUtensorMap& tm_k8,
                                   const CUtensorMap& tm_v8, const CUtensorMap& tm_po,
                                   const CUtensorMap& tm_out, const DecodeParams& p,
                                   int num_workers, cudaStream_t stream) {
  return launch_pair<false, true>(tm_q, tm_k8, tm_v8, tm_po, tm_out, p, num_workers, stream);
}

// Pairs (clusters of 2) of this kernel that fit on the device at once.
cudaError_t pair_kernel_max_clusters(int* clusters) {
  static std::atomic<int> cached[64];  // per device: 0 until computed
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int known = cached[dev].load(std::memory_order_acquire);
  if (known > 0) {
    *clusters = known;
    return cudaSuccess;
  }
  e = configure_pair_kernels();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(PairRoles<false>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, mla_decode_pair_kernel<false, false>, &cfg);
  if (e != cudaSuccess) return e;
  if (n < 1) n = 1;
  cached[dev].store(n, std::memory_order_release);
  *clusters = n;
  return cudaSuccess;
}

}  // namespace mla

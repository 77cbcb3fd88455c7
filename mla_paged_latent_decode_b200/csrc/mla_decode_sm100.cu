// mla_decode_sm100.cu -- MLA decode over a paged latent cache on sm_100a.
//
// One CTA owns one 64-row block of the flattened (s_q, h_q) query rows of one
// worker's run of (sequence, page) items (see mla_metadata.cu).
//
// Data movement and math per page:
//   TMA   : the 64 x 576 bf16 page (72 KB) -> shared memory as one 3-D box
//           (nine 64-dim chunks of 64 rows) with 128-byte swizzle, through the
//           block table; a ring of three stages.  In gather mode (sparse
//           decode) the producer warp's lanes copy the page's listed rows
//           instead, with 16-byte cp.async copies into the same layout.  At the start of each piece the same ring also
//           carries the piece's 64 query rows (72 KB), which the softmax warps
//           move into tensor memory.
//   MMA   : S  = Q . K^T    tcgen05 M=64 N=64 K=576, A = Q in TMEM, B = page
//           O += P . V      tcgen05 M=64 N=256 K=64 (two halves of dv = 512),
//                           A = P in SMEM, B = the same page tile read MN-major:
//                           the value is dims 0..511 of the rows already in
//                           shared memory, so each page leaves HBM once.
//           S is double-buffered: QK^T of page j+1 runs while the softmax of
//           page j does, and PV of page j follows.
//   softmax warps: online softmax on S read from TMEM, P (bf16) -> SMEM, O
//           rescaled in TMEM only when the running maximum grows past a
//           threshold.
//   epilogue: O / l -> bf16 out and lse, or fp32 partials for split sequences.
//
// Tensor memory (512 columns x 128 lanes).  An M=64 operand or accumulator
// occupies 16 lanes of each 32-lane quarter; row r of a block lives in quarter
// r / 16.  Lanes 0-15 of each quarter hold Q (columns 0..287, two bf16 per
// column) and the two S buffers (columns 320..383, 384..447): the A operand and
// the accumulator of QK^T must share lanes.  Lanes 16-31 hold O (columns
// 0..511).  Softmax, rescale and epilogue use 16-lane TMEM accesses, so they
// never touch lanes an MMA in flight is writing.
//
// Warp roles (256 threads): warps 0-3 softmax/correction/epilogue, warp 4 TMA
// producer, warps 5 and 7 QK^T issuers for even and odd pages (warp 5 also
// allocates TMEM), warp 6 PV issuer.
//
// FP8 cache (template argument kFp8): the same kernel over E4M3 codes with one
// power-of-two scale per token.  The TMA warp lands each page chunk's codes in
// the upper half of that chunk's 128-byte row slots inside the bf16 stage, and
// eight more warps (512 threads) widen them in place into the bf16 tile, exactly;
// the MMAs, softmax and epilogue are unchanged.
//
// The method follows "FlashMLA: Revolutionizing Efficient Decoding...",
// sections 4.2.1-4.2.3 (TMA prefetch of 64-row latent blocks into shared
// memory, tensor cores for QK^T and PV, softmax fused into the kernel),
// re-designed for the 5th-generation tensor core: operands and accumulators
// live in tensor memory, MMAs are issued by one thread, and the softmax runs in
// warps of its own.
#include <cuda_bf16.h>

#include <atomic>

#include "mla_kernels.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kSoftmaxThreads = 128;
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;    // issues QK^T of even pages; allocates tensor memory
constexpr int kPvWarp = 6;     // issues PV
constexpr int kQkOddWarp = 7;  // issues QK^T of odd pages
constexpr int kConvWarp0 = 8;  // FP8 cache: first of eight converter warps
constexpr int kConvThreads = 256;
constexpr int kConvChunkStep = kConvThreads / 64;  // chunks apart of one thread's row slots
constexpr int kConvBarrier = 1;                    // named barrier of the converter warps
constexpr int kChunkBytes = 64 * 128;              // 64 rows x 64 bf16 (one swizzle column block)
constexpr int kChunks = kDqk / 64;                 // 9
constexpr int kTileBytes = kChunks * kChunkBytes;  // 73728 = 64 x 576 bf16
constexpr int kPBytes = 64 * 128;                  // P: 64 rows x 64 tokens bf16

// Shared-memory layout, barriers and threads of the bf16-cache kernel
// (kFp8 = false) and of the FP8-cache kernel (kFp8 = true).  The FP8 kernel
// keeps the same three-stage ring of bf16 tiles.  TMA lands each 64-dim chunk
// of a page's codes in the upper half of that chunk's 128-byte row slots
// inside the stage, and the converter warps widen every (row, chunk) in place;
// a page's 64 scales go to a small per-stage area.
template <bool kFp8>
struct Cfg {
  static constexpr int kThreads = kFp8 ? 256 + kConvThreads : 256;
  static constexpr int kStages = 3;
  static constexpr int kOffKV = 0;
  static constexpr int kOffP = kOffKV + kStages * kTileBytes;
  static constexpr int kOffScale = kOffP + kPBytes;                 // FP8: [stage][64] fp32
  static constexpr int kOffBar = kOffScale + (kFp8 ? kStages * kPage * 4 : 0);
  static constexpr int kFull0 = 0, kEmpty0 = kStages, kQFull = 2 * kStages;
  static constexpr int kSFull0 = kQFull + 1, kSFull1 = kQFull + 2;
  static constexpr int kSFree0 = kQFull + 3, kSFree1 = kQFull + 4;
  static constexpr int kPFull = kQFull + 5, kPvDone = kQFull + 6, kOFull = kQFull + 7;
  static constexpr int kLanded0 = kQFull + 8;                      // FP8: codes in the stage
  static constexpr int kDrain0 = kLanded0 + (kFp8 ? kStages : 0);  // MMA drain after an abort
  static constexpr int kNumBars = kDrain0 + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem address + abort flag
  static constexpr int kSmemUsed = kOffMisc + 16;
  static constexpr int kSmemBytes = kSmemUsed + 1024;      // slack to align the base to 1024 B
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kOffP % 1024 == 0 && kOffScale % 16 == 0, "alignment");
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQ = 0;                     // lanes 0-15, columns 0..287
constexpr uint32_t kTmemS = 320;                   // lanes 0-15, S buffer b at 320 + 64 b
constexpr uint32_t kTmemO = 16u << 16;             // lanes 16-31, columns 0..511
constexpr float kRescaleThreshold = 8.0f;          // log2 units: P <= 2^8 before a rescale

constexpr uint32_t kIdescQK = idesc_bf16_f32(64, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(64, 256, false, true);

static_assert(kTmemS + 128 <= kTmemCols, "tensor memory budget");

struct Piece {
  int seq, pg0, npg, split_idx;
};

// The MMA-issuing roles run either on a whole warp (kWarp: every lane runs the
// loop, one elected lane issues each MMA and commit) or on lane 0 alone.
template <bool kWarp>
__device__ __forceinline__ bool issuer_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                            uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns);
  if constexpr (kWarp) return __all_sync(0xffffffffu, ok);
  return ok;
}
template <bool kWarp>
__device__ __forceinline__ void issue_commit(uint64_t* bar) {
  if constexpr (kWarp) umma_commit_warp(bar);
  else umma_commit(bar);
}

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

// Bounded wait whose outcome is the same for every lane of the warp, so that
// warp-collective TMEM accesses that follow are reached by all lanes or none.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

template <bool kFp8, bool kGather = false>
__global__ void __launch_bounds__(Cfg<kFp8>::kThreads, 1)
mla_decode_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_page, const DecodeParams p) {
  using C = Cfg<kFp8>;
  constexpr int kStages = C::kStages;
  constexpr int kFull0 = C::kFull0, kEmpty0 = C::kEmpty0, kQFull = C::kQFull;
  constexpr int kSFull0 = C::kSFull0, kSFull1 = C::kSFull1, kSFree0 = C::kSFree0;
  constexpr int kSFree1 = C::kSFree1, kPFull = C::kPFull, kPvDone = C::kPvDone;
  constexpr int kOFull = C::kOFull;
  // MMAs issued by whole warps with a bf16 cache; from lane 0 in the FP8
  // variant, whose issuing warps run with 56 registers
  constexpr bool kWarpIssue = !kFp8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* skv = smem + C::kOffKV;
  uint8_t* sp = smem + C::kOffP;
  float* sscale = reinterpret_cast<float*>(smem + C::kOffScale);  // FP8 cache only
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int worker = blockIdx.x, rb = blockIdx.y;
  const uint64_t wait_ns = p.wait_ns;  // limit of every bounded wait (normally kWaitLimitNs)

  // Set-up first: the kernel is launched as a programmatic dependent of the
  // scheduler kernel, so its CTAs may start while the scheduler runs; barriers
  // and tensor memory are made ready meanwhile, and the metadata is read only
  // after the dependency wait below.
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar[kFull0 + s], 1);
      mbar_init(&bar[kEmpty0 + s], 1);
    }
    mbar_init(&bar[kQFull], kSoftmaxThreads);
    mbar_init(&bar[kSFull0], 1);
    mbar_init(&bar[kSFull1], 1);
    mbar_init(&bar[kSFree0], kSoftmaxThreads);
    mbar_init(&bar[kSFree1], kSoftmaxThreads);
    mbar_init(&bar[kPFull], kSoftmaxThreads);
    mbar_init(&bar[kPvDone], 1);
    mbar_init(&bar[kOFull], 1);
    if constexpr (kFp8) {
      for (int s = 0; s < kStages; ++s) mbar_init(&bar[C::kLanded0 + s], 1);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&bar[C::kDrain0 + i], 1);
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

  grid_dependency_wait();  // the scheduler's metadata is complete and visible
  const int32_t* md = p.tile_md + static_cast<int64_t>(worker) * kMdStride;
  int npieces = md[5];
  if (npieces != 0 && (md[0] < 0 || npieces < 0 || md[0] + npieces > p.batch)) {
    if (threadIdx.x == 0) report(p.status, MLA_ERR_DEVICE_CHECK);  // metadata not from this batch
    npieces = 0;
  }
  // An idle worker (or bad metadata) runs no role and goes straight to the
  // common teardown.
  // FP8 cache: 512 threads launched with 128 registers each; the softmax
  // warpgroup raises its budget to 232, the single-thread roles (warps 4-7)
  // lower theirs to 56 and the two converter warpgroups to 96: 61440 of the
  // 65536 in all.
  if constexpr (kFp8) {
    if (warp >= 4 && warp < kConvWarp0) setmaxnreg_dec<56>();
  }

  // The stage ring carries, per piece with pages, one entry for the query rows
  // followed by one entry per page; every role counts entries the same way.
  if (kFp8 && warp == kTmaWarp) {
    // ------------------------------------------------------------ FP8 producer
    // Query rows as in the bf16 kernel (straight to the stage's full barrier).
    // A page: for chunk c, one 128-byte x 64-row box whose x window is
    // [64 c - 64, 64 c + 64) of the 576-byte row, so chunk c's codes land in
    // bytes 64..127 of each 128-byte row slot of the tile's chunk c (bytes
    // 0..63 get chunk c - 1's codes, or zeros for c = 0, and are overwritten by
    // the converters); plus the page's 64 scales.  Both signal the stage's
    // landed barrier; the converters signal full.
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_page);
      int entries = 0, last_q = -1;
      uint32_t landed_parity = 0, landed_used = 0;  // per stage: page loads issued (mod 2), any
      bool ok = true;
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (p.seqlens[pz.seq] > p.bt_stride * kPage) report(p.status, MLA_ERR_DEVICE_CHECK);
        if (pz.npg == 0) continue;
        const int32_t* bt = p.block_table + static_cast<int64_t>(pz.seq) * p.bt_stride;
        for (int e = -1; e < pz.npg; ++e) {
          const int stage = entries % kStages, use = entries / kStages;
          if (use > 0) {
            ok = mbar_wait(&bar[kEmpty0 + stage], (use - 1) & 1, abort_flag, wait_ns);
            if (!ok) break;
          }
          uint8_t* dst = skv + stage * kTileBytes;
          if (e < 0) {
            last_q = entries;
            mbar_arrive_expect_tx(&bar[kFull0 + stage], kTileBytes);
            const int qrow = pz.seq * p.rows + blockIdx.y * kRowsPerCta;
            for (int c = 0; c < kChunks; ++c)
              tma_load_2d(dst + c * kChunkBytes, &tm_q, c * 64, qrow, &bar[kFull0 + stage]);
          } else {
            int page = __ldg(bt + pz.pg0 + e);
            // The tensor map bounds the codes, but the untiled scale copy has no
            // bounds: a page id outside the cache is reported and replaced.
            if (page < 0 || page >= p.num_blocks) {
              report(p.status, MLA_ERR_DEVICE_CHECK);
              page = 0;
            }
            uint64_t* landed = &bar[C::kLanded0 + stage];
            mbar_arrive_expect_tx(landed, kTileBytes + kPage * 4);
            for (int c = 0; c < kChunks; ++c)
              tma_load_2d(dst + c * kChunkBytes, &tm_page, 64 * c - 64, page * kPage, landed);
            bulk_load(sscale + stage * kPage, p.kscale + static_cast<int64_t>(page) * kPage,
                      kPage * 4, landed);
            landed_parity ^= 1u << stage;
            landed_used |= 1u << stage;
          }
          ++entries;
        }
      }
      // Before leaving, let every copy this thread issued land (bounded): the
      // last page load of each stage, and the last query load if no later
      // entry reused its stage.
      for (int s = 0; s < kStages; ++s)
        if ((landed_used >> s) & 1)
          mbar_wait_drain(&bar[C::kLanded0 + s], ((landed_parity >> s) & 1) ^ 1, kWaitLimitNs);
      if (last_q >= 0 && last_q >= entries - kStages)
        mbar_wait_drain(&bar[kFull0 + last_q % kStages], (last_q / kStages) & 1, kWaitLimitNs);
    }
  } else if (kFp8 && warp >= kConvWarp0) {
    // ------------------------------------------------------------ FP8 converters
    // Widen each landed page in place: thread t owns row r = t % 64 of chunks
    // t / 64, t / 64 + 4, ... (3 or 2 of the 9).  For each it reads the 64
    // codes (bytes 64..127 of the row slot) into registers, then writes the 64
    // bf16 values over the whole 128-byte slot, swizzled.  No other thread
    // touches that slot, so reading before writing makes the in-place update
    // safe.  The four 16-byte loads start at unit (r mod 4) and the eight 8-lane
    // store phases cover 8 rows, so neither hits a bank more than twice.  Rows
    // past the sequence's end are written as zeros, so stale codes or scales
    // there never reach an MMA.  The eight warps decide together after a named
    // barrier, so that a wait that gave up in one warp stops all of them.
    if constexpr (kFp8) setmaxnreg_dec<96>();
    const int ct = threadIdx.x - kConvWarp0 * 32;
    const int r = ct & 63, c0 = ct >> 6;
    int entries = 0;
    uint32_t landed_parity = 0;  // per stage: pages converted there (mod 2)
    for (int pc = 0; pc < npieces; ++pc) {
      const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
      if (pz.npg == 0) continue;
      const int L = p.seqlens[pz.seq];
      entries += 1;  // the query entry goes straight to the consumers
      bool stop = false;
      for (int e = 0; e < pz.npg; ++e, ++entries) {
        const int stage = entries % kStages;
        const uint32_t parity = (landed_parity >> stage) & 1;
        landed_parity ^= 1u << stage;
        warp_wait(&bar[C::kLanded0 + stage], parity, abort_flag, wait_ns);  // gives up at once on abort
        named_bar_sync(kConvBarrier, kConvThreads);
        if (*abort_flag) { stop = true; break; }
        uint8_t* tile = skv + stage * kTileBytes;
        const bool row_ok = r < L - (pz.pg0 + e) * kPage;  // row inside the sequence
        // 2^60 * scale as bf16x2 (a power of two: its fp32 bits end in 16 zeros)
        const uint32_t f_lo = row_ok ? (__float_as_uint(sscale[stage * kPage + r] * 0x1p60f) >> 16) *
                                           0x10001u
                                     : 0u;
        constexpr uint32_t f_hi = 0x5D805D80u;  // 2^60 in both halves
        for (int c = c0; c < kChunks; c += kConvChunkStep) {
          uint8_t* slot = tile + c * kChunkBytes + r * 128;
          uint4 v[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            v[k] = *reinterpret_cast<const uint4*>(slot + 64 + 16 * ((k + r) & 3));
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int kk = (k + r) & 3;  // v[k] holds dims 16 kk .. 16 kk + 15 of the chunk
            uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
            if (row_ok) {
              lo.x = e4m3x2_to_bf16x2(v[k].x, 0x1404u, f_hi, f_lo);
              lo.y = e4m3x2_to_bf16x2(v[k].x, 0x3424u, f_hi, f_lo);
              lo.z = e4m3x2_to_bf16x2(v[k].y, 0x1404u, f_hi, f_lo);
              lo.w = e4m3x2_to_bf16x2(v[k].y, 0x3424u, f_hi, f_lo);
              hi.x = e4m3x2_to_bf16x2(v[k].z, 0x1404u, f_hi, f_lo);
              hi.y = e4m3x2_to_bf16x2(v[k].z, 0x3424u, f_hi, f_lo);
              hi.z = e4m3x2_to_bf16x2(v[k].w, 0x1404u, f_hi, f_lo);
              hi.w = e4m3x2_to_bf16x2(v[k].w, 0x3424u, f_hi, f_lo);
            }
            *reinterpret_cast<uint4*>(slot + (((2 * kk) ^ (r & 7)) << 4)) = lo;
            *reinterpret_cast<uint4*>(slot + (((2 * kk + 1) ^ (r & 7)) << 4)) = hi;
          }
        }
        fence_proxy_async_smem();  // the MMAs read the tile through the async proxy
        named_bar_sync(kConvBarrier, kConvThreads);
        if (ct == 0) mbar_arrive(&bar[kFull0 + stage]);
      }
      if (stop) break;
    }
  } else if (kGather && warp == kTmaWarp) {
    // ------------------------------------------------------------ gather producer
    // The sparse decode's rows: token k of sequence s is cached row
    // gather_rows[s * gather_stride + k].  The query rows come by TMA as in the
    // dense producer (lane 0); a page's 64 rows are copied by all 32 lanes in
    // 16-byte pieces (eight lanes per 128-byte row segment) into the same
    // swizzled tile layout.  Each lane waits for its own copies, issues a proxy
    // fence, and lane 0 signals the page once the next page has been issued
    // (one page of copies in flight behind the newest; a piece's last page at
    // the piece's end).
    prefetch_tensormap(&tm_q);
    auto wait = [&](uint64_t* b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, wait_ns));
    };
    int entries = 0, last_q = -1, pending = -1;
    bool ok = true;
    for (int pc = 0; pc < npieces && ok; ++pc) {
      const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
      if (lane == 0 && p.seqlens[pz.seq] > p.bt_stride * kPage)
        report(p.status, MLA_ERR_DEVICE_CHECK);
      if (pz.npg == 0) continue;
      const int cnt = p.seqlens[pz.seq];
      const int32_t* grows = p.gather_rows + static_cast<int64_t>(pz.seq) * p.gather_stride;
      auto rows_of = [&](int jj, int (&r)[2]) {  // this lane's rows: lane and lane + 32
        const int vt0 = (pz.pg0 + jj) * kPage;
        for (int h = 0; h < 2; ++h) {
          const int tok = vt0 + 32 * h + lane;
          r[h] = tok < cnt ? __ldg(grows + tok) : -1;  // past the count: a zero row
        }
      };
      int next[2];
      rows_of(0, next);
      for (int e = -1; e < pz.npg; ++e) {  // e = -1: the query rows
        const int stage = entries % kStages, use = entries / kStages;
        if (use > 0) {
          ok = wait(&bar[kEmpty0 + stage], (use - 1) & 1);
          if (!ok) break;
        }
        uint8_t* dst = skv + stage * kTileBytes;
        if (e < 0) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&bar[kFull0 + stage], kTileBytes);
            const int qrow = pz.seq * p.rows + rb * kRowsPerCta;
            for (int c = 0; c < kChunks; ++c)
              tma_load_2d(dst + c * kChunkBytes, &tm_q, c * 64, qrow, &bar[kFull0 + stage]);
          }
          last_q = entries;
        } else {
          const int mine[2] = {next[0], next[1]};
          if (e + 1 < pz.npg) rows_of(e + 1, next);
          const int u = lane & 7;
#pragma unroll
          for (int grp = 0; grp < 16; ++grp) {
            const int r = 4 * grp + (lane >> 3);
            const int row = __shfl_sync(0xffffffffu, grp < 8 ? mine[0] : mine[1], r & 31);
            const uint8_t* src = static_cast<const uint8_t*>(p.gather_cache) +
                                 static_cast<int64_t>(row < 0 ? 0 : row) * (kDqk * 2) + u * 16;
            uint8_t* d = dst + r * 128 + ((u ^ (r & 7)) << 4);
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
              cp_async16_zfill(d + c * kChunkBytes, src + c * 128, row >= 0);
          }
          cp_async_commit();
          if (pending >= 0) {
            cp_async_wait_group<1>();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kFull0 + pending]);
          }
          pending = stage;
          if (e + 1 == pz.npg) {  // the piece's last page: signal it now
            cp_async_wait_group<0>();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kFull0 + pending]);
            pending = -1;
          }
        }
        ++entries;
      }
    }
    // Before leaving, let every copy this warp issued land (bounded): the page
    // copies, and the last query load if no later entry reused its stage.
    cp_async_wait_group<0>();
    if (lane == 0 && last_q >= 0 && last_q >= entries - kStages)
      mbar_wait_drain(&bar[kFull0 + last_q % kStages], (last_q / kStages) & 1, kWaitLimitNs);
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_page);
      int entries = 0;
      bool ok = true;
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (p.seqlens[pz.seq] > p.bt_stride * kPage) report(p.status, MLA_ERR_DEVICE_CHECK);
        if (pz.npg == 0) continue;
        const int32_t* bt = p.block_table + static_cast<int64_t>(pz.seq) * p.bt_stride;
        for (int e = -1; e < pz.npg; ++e) {  // e = -1: the query rows
          const int stage = entries % kStages, use = entries / kStages;
          if (use > 0) {
            ok = mbar_wait(&bar[kEmpty0 + stage], (use - 1) & 1, abort_flag, wait_ns);
            if (!ok) break;
          }
          uint8_t* dst = skv + stage * kTileBytes;
          mbar_arrive_expect_tx(&bar[kFull0 + stage], kTileBytes);
          if (e < 0) {
            const int qrow = pz.seq * p.rows + rb * kRowsPerCta;
            for (int c = 0; c < kChunks; ++c)
              tma_load_2d(dst + c * kChunkBytes, &tm_q, c * 64, qrow, &bar[kFull0 + stage]);
          } else {
            const int page = __ldg(bt + pz.pg0 + e);
            tma_load_3d(dst, &tm_page, 0, page * kPage, 0, &bar[kFull0 + stage]);
          }
          ++entries;
        }
      }
      // Before leaving, let every copy this thread issued land (bounded).
      for (int s = 0; s < kStages && s < entries; ++s) {
        const int n = entries - 1 - s;
        mbar_wait_drain(&bar[kFull0 + n % kStages], (n / kStages) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == kMmaWarp || warp == kQkOddWarp) {
    // ------------------------------------------------------------ QK^T issuers
    // A single thread issues a tcgen05.mma only every ~60 cycles, longer than an
    // M=64 N=64 MMA takes.  So QK^T of even pages (S buffer 0), QK^T of odd
    // pages (S buffer 1) and PV come from three warps, and the tensor core runs
    // their MMAs back to back; with a bf16 cache each warp issues as a whole
    // (every lane runs the loop, an elected lane issues), which is faster still.
    // QK^T runs up to two pages ahead of the softmax.
    const int parity = warp == kMmaWarp ? 0 : 1;
    if (kWarpIssue || lane == 0) {
      int entries = 0, pages = 0, qloads = 0;
      bool ok = true;
      const uint32_t kv_base = smem_addr(skv);
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (pz.npg == 0) continue;
        const int q_entry = entries;   // copied into TMEM by the softmax warps
        const int first = entries + 1;
        entries += 1 + pz.npg;
        ok = issuer_wait<kWarpIssue>(&bar[kQFull], qloads & 1, abort_flag, wait_ns);
        ++qloads;
        if (!ok) break;
        if (parity == 0 && lane == 0) mbar_arrive(&bar[kEmpty0 + q_entry % kStages]);  // query stage free
        tc_fence_after();
        for (int j = 0; j < pz.npg && ok; ++j) {
          const int g = pages + j, b = g & 1;
          if (b != parity) continue;
          if (g >= 2) {  // the softmax has read S of page g - 2 from buffer b
            ok = issuer_wait<kWarpIssue>(&bar[kSFree0 + b], ((g >> 1) - 1) & 1, abort_flag, wait_ns);
            if (!ok) break;
          }
          const int entry = first + j, stage = entry % kStages;
          ok = issuer_wait<kWarpIssue>(&bar[kFull0 + stage], (entry / kStages) & 1, abort_flag,
                                       wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint64_t b0 = smem_desc_sw128(kv_base + stage * kTileBytes, 16, 1024);
          const uint32_t d = tmem + kTmemS + 64 * b;
#pragma unroll
          for (int kk = 0; kk < kDqk / 16; ++kk) {
            // K-step kk: swizzle block kk/4, 32-byte step (kk%4) inside it
            const uint32_t boff = ((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4;
            if constexpr (kWarpIssue)
              umma_bf16_ts_warp(d, tmem + kTmemQ + 8 * kk, b0 + boff, kIdescQK, kk > 0 ? 1u : 0u);
            else
              umma_bf16_ts(d, tmem + kTmemQ + 8 * kk, b0 + boff, kIdescQK, kk > 0 ? 1u : 0u);
          }
          issue_commit<kWarpIssue>(&bar[kSFull0 + b]);
        }
        pages += pz.npg;
      }
    }
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ PV issuer
    if (kWarpIssue || lane == 0) {  // as for QK^T
      int entries = 0, pages = 0;
      bool ok = true;
      const uint32_t kv_base = smem_addr(skv), p_base = smem_addr(sp);
      for (int pc = 0; pc < npieces && ok; ++pc) {
        const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
        if (pz.npg == 0) continue;
        const int first = entries + 1;
        entries += 1 + pz.npg;
        for (int j = 0; j < pz.npg; ++j) {
          const int g = pages + j;
          // P of page g is in shared memory (and QK^T of page g, which read the
          // same stage, has completed: the softmax saw its S)
          ok = issuer_wait<kWarpIssue>(&bar[kPFull], g & 1, abort_flag, wait_ns);
          if (!ok) break;
          // test hook: a wait that nothing ends, with copies and MMAs in flight
          if (g == 0 && p.stall_flag != nullptr) {
            ok = flag_wait(p.stall_flag, abort_flag, wait_ns);
            if constexpr (kWarpIssue) ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          }
          tc_fence_after();
          const int stage = (first + j) % kStages;
          const uint32_t tile = kv_base + stage * kTileBytes;
          // O += P . V, V = columns 0..511 of the same tile, read MN-major
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < kPage / 16; ++kk) {
              const uint64_t pa = smem_desc_sw128(p_base + kk * 32, 16, 1024);
              const uint64_t vb =
                  smem_desc_sw128(tile + half * 4 * kChunkBytes + kk * 2048, kChunkBytes, 1024);
              if constexpr (kWarpIssue)
                umma_bf16_ss_warp(tmem + kTmemO + half * 256, pa, vb, kIdescPV,
                                  (j > 0 || kk > 0) ? 1u : 0u);
              else
                umma_bf16_ss(tmem + kTmemO + half * 256, pa, vb, kIdescPV,
                             (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          issue_commit<kWarpIssue>(&bar[kEmpty0 + stage]);
          issue_commit<kWarpIssue>(&bar[kPvDone]);
        }
        if (!ok) break;
        // every MMA of the piece is complete once this fires: the last PV
        // follows (through the softmax) the last QK^T
        issue_commit<kWarpIssue>(&bar[kOFull]);
        pages += pz.npg;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    if constexpr (kFp8) setmaxnreg_inc<232>();
    // 16-lane TMEM accesses: thread t holds rows t/4 and t/4 + 8 of its quarter's
    // 16, at columns 2(t%4) + {0,1} + 8g.
    const uint32_t quarter = static_cast<uint32_t>(32 * warp) << 16;
    const int ra = 16 * warp + (lane >> 2);
    const int rbb = ra + 8;
    const int row_a = rb * kRowsPerCta + ra, row_b = rb * kRowsPerCta + rbb;
    const bool ok_a = row_a < p.rows, ok_b = row_b < p.rows;
    const int jq_a = ok_a ? row_a / p.h_q : 0, jq_b = ok_b ? row_b / p.h_q : 0;
    const int hq_a = ok_a ? row_a % p.h_q : 0, hq_b = ok_b ? row_b % p.h_q : 0;
    const int c2 = 2 * (lane & 3);
    const int qr = 16 * warp + lane;  // Q row this thread copies (lanes 0-15)
    int entries = 0, pages = 0, pieces_done = 0;
    bool ok = true;
    for (int pc = 0; pc < npieces && ok; ++pc) {
      const Piece pz = piece_of(md, pc, p.seqlens, p.bt_stride);
      const int L = p.seqlens[pz.seq];
      const int cap_tokens = static_cast<int>(p.bt_stride * kPage < L ? p.bt_stride * kPage : L);
      auto visible = [&](int jq) {
        int v = p.causal ? L - p.s_q + jq + 1 : L;
        v = v < 0 ? 0 : v;
        return v < cap_tokens ? v : cap_tokens;
      };
      const int lim_a = visible(jq_a), lim_b = visible(jq_b);
      const int base_split = p.num_splits[pz.seq];
      const int k_pieces = p.num_splits[pz.seq + 1] - base_split;
      const int64_t slot = static_cast<int64_t>(base_split) + pz.split_idx;
      float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

      if (pz.npg > 0) {
        // ---- query rows: stage -> TMEM lanes 0-15 (lanes 16-31 write the dead O region)
        const int q_entry = entries;
        entries += 1 + pz.npg;
        const int qstage = q_entry % kStages;
        ok = warp_wait(&bar[kFull0 + qstage], (q_entry / kStages) & 1, abort_flag, wait_ns);
        if (!ok) break;
        {
          const uint8_t* qt = skv + qstage * kTileBytes;
          for (int c = 0; c < kChunks; ++c) {
            uint32_t r[32];
            if (lane < 16) {
              const uint8_t* rowp = qt + c * kChunkBytes + qr * 128;
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((u ^ (qr & 7)) << 4));
                r[4 * u] = v.x;
                r[4 * u + 1] = v.y;
                r[4 * u + 2] = v.z;
                r[4 * u + 3] = v.w;
              }
            } else {
#pragma unroll
              for (int u = 0; u < 32; ++u) r[u] = 0u;
            }
            tmem_st32(tmem + quarter + kTmemQ + 32 * c, r);
          }
          tmem_st_wait();
        }
        // Q is in TMEM and the stage has been read: the MMA warp, once all 128
        // threads have arrived, hands the stage back to the producer.
        tc_fence_before();
        mbar_arrive(&bar[kQFull]);

        for (int j = 0; j < pz.npg; ++j) {
          const int g = pages + j;
          ok = warp_wait(&bar[kSFull0 + (g & 1)], (g >> 1) & 1, abort_flag, wait_ns);
          if (!ok) break;
          tc_fence_after();
          uint32_t s[32];
          tmem_ld16x64(tmem + quarter + kTmemS + 64 * (g & 1), s);
          tmem_ld_wait(s);
          tc_fence_before();
          mbar_arrive(&bar[kSFree0 + (g & 1)]);
          const int tok0 = (pz.pg0 + j) * kPage;
          const int nv_a = lim_a - tok0, nv_b = lim_b - tok0;
          float x[32];
          float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            const int tok = c2 + (r & 1) + 8 * (r >> 2);
            const bool second = (r >> 1) & 1;
            const bool valid = tok < (second ? nv_b : nv_a);
            x[r] = valid ? __uint_as_float(s[r]) * p.scale_log2 : -INFINITY;
            if (second)
              mx_b = fmaxf(mx_b, x[r]);
            else
              mx_a = fmaxf(mx_a, x[r]);
          }
          mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
          mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
          mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
          mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
          float alpha_a = 1.f, alpha_b = 1.f;
          if (mx_a > m_a + kRescaleThreshold) {
            alpha_a = ex2_approx(m_a - mx_a);
            m_a = mx_a;
          }
          if (mx_b > m_b + kRescaleThreshold) {
            alpha_b = ex2_approx(m_b - mx_b);
            m_b = mx_b;
          }
          float sum_a = 0.f, sum_b = 0.f;
          uint32_t pw[16];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float p0 = x[4 * q4] == -INFINITY ? 0.f : ex2_approx(x[4 * q4] - m_a);
            const float p1 = x[4 * q4 + 1] == -INFINITY ? 0.f : ex2_approx(x[4 * q4 + 1] - m_a);
            const float p2 = x[4 * q4 + 2] == -INFINITY ? 0.f : ex2_approx(x[4 * q4 + 2] - m_b);
            const float p3 = x[4 * q4 + 3] == -INFINITY ? 0.f : ex2_approx(x[4 * q4 + 3] - m_b);
            sum_a += p0 + p1;
            sum_b += p2 + p3;
            pw[q4] = pack_bf16x2(p0, p1);
            pw[8 + q4] = pack_bf16x2(p2, p3);
          }
          l_a = l_a * alpha_a + sum_a;
          l_b = l_b * alpha_b + sum_b;
          // P and O may be touched only after PV of the previous page is done.
          if (j > 0) {
            ok = warp_wait(&bar[kPvDone], (g - 1) & 1, abort_flag, wait_ns);
            if (!ok) break;
            tc_fence_after();
            if (__any_sync(0xffffffffu, alpha_a != 1.f || alpha_b != 1.f)) {
              for (int cb = 0; cb < kDv; cb += 64) {
                uint32_t o[32];
                tmem_ld16x64(tmem + quarter + kTmemO + cb, o);
                tmem_ld_wait(o);
#pragma unroll
                for (int r = 0; r < 32; ++r)
                  o[r] = __float_as_uint(__uint_as_float(o[r]) * (((r >> 1) & 1) ? alpha_b : alpha_a));
                tmem_st16x64(tmem + quarter + kTmemO + cb, o);
              }
              tmem_st_wait();
            }
          }
          // P rows ra and rbb: token pair (8g + c2, +1) -> 4 bytes in 16-byte unit g (swizzled)
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            *reinterpret_cast<uint32_t*>(sp + ra * 128 + ((q4 ^ (ra & 7)) << 4) + 2 * c2) = pw[q4];
            *reinterpret_cast<uint32_t*>(sp + rbb * 128 + ((q4 ^ (rbb & 7)) << 4) + 2 * c2) =
                pw[8 + q4];
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&bar[kPFull]);
        }
        if (!ok) break;
        ok = warp_wait(&bar[kOFull], pieces_done & 1, abort_flag, wait_ns);
        ++pieces_done;
        pages += pz.npg;
        if (!ok) break;
        tc_fence_after();
      }
      // The dependent grid (the split combine) may be scheduled once every CTA
      // has reached its last epilogue; it still waits for this grid's end
      // before it reads anything.
      if (pc == npieces - 1 && threadIdx.x == 0) grid_launch_dependents();
      // ---- epilogue: the four threads of a row group hold disjoint columns
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      const float inv_a = l_a > 0.f ? 1.f / l_a : 0.f;
      const float inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
      const int64_t orow_a = static_cast<int64_t>(pz.seq) * p.rows + row_a;
      const int64_t orow_b = static_cast<int64_t>(pz.seq) * p.rows + row_b;
      for (int cb = 0; cb < kDv; cb += 64) {
        uint32_t o[32];
        if (pz.npg > 0) {
          tmem_ld16x64(tmem + quarter + kTmemO + cb, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int r = 0; r < 32; ++r) o[r] = 0u;
        }
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const int col = cb + 8 * q4 + c2;
          const float a0 = __uint_as_float(o[4 * q4]) * inv_a;
          const float a1 = __uint_as_float(o[4 * q4 + 1]) * inv_a;
          const float b0 = __uint_as_float(o[4 * q4 + 2]) * inv_b;
          const float b1 = __uint_as_float(o[4 * q4 + 3]) * inv_b;
          if (k_pieces == 1) {
            if (ok_a) *reinterpret_cast<uint32_t*>(p.out + orow_a * kDv + col) = pack_bf16x2(a0, a1);
            if (ok_b) *reinterpret_cast<uint32_t*>(p.out + orow_b * kDv + col) = pack_bf16x2(b0, b1);
          } else {
            if (ok_a)
              *reinterpret_cast<float2*>(p.part_o + (slot * p.rows + row_a) * kDv + col) =
                  make_float2(a0, a1);
            if (ok_b)
              *reinterpret_cast<float2*>(p.part_o + (slot * p.rows + row_b) * kDv + col) =
                  make_float2(b0, b1);
          }
        }
      }
      if ((lane & 3) == 0) {
        const float lse_a = l_a > 0.f ? (m_a + lg2_approx(l_a)) * 0.69314718055994531f : -INFINITY;
        const float lse_b = l_b > 0.f ? (m_b + lg2_approx(l_b)) * 0.69314718055994531f : -INFINITY;
        if (k_pieces == 1) {
          if (ok_a) p.lse[(static_cast<int64_t>(pz.seq) * p.h_q + hq_a) * p.s_q + jq_a] = lse_a;
          if (ok_b) p.lse[(static_cast<int64_t>(pz.seq) * p.h_q + hq_b) * p.s_q + jq_b] = lse_b;
        } else {
          if (ok_a) p.part_lse[slot * p.rows + row_a] = lse_a;
          if (ok_b) p.part_lse[slot * p.rows + row_b] = lse_b;
        }
      }
    }
  }

  // After an abort, MMAs this CTA issued may still be in flight: each issuing
  // thread waits for its own through a commit before tensor and shared memory
  // are released (the TMA producer has already let its copies land).
  if (*abort_flag) {
    if ((kWarpIssue || lane == 0) && (warp == kMmaWarp || warp == kPvWarp || warp == kQkOddWarp)) {
      // the lane that issued the MMAs commits (the elected one of a whole warp)
      uint64_t* db = &bar[C::kDrain0 + (warp - kMmaWarp)];
      if constexpr (kWarpIssue) __syncwarp();
      issue_commit<kWarpIssue>(db);
      mbar_wait_drain(db, 0, kWaitLimitNs);
    }
    if (threadIdx.x == 0) abort_grace();
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

cudaError_t launch_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_page,
                          const DecodeParams& p, int num_workers, cudaStream_t stream) {
  static std::atomic<bool> configured[64];  // per device: attribute set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(mla_decode_sm100_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<false>::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(mla_decode_sm100_kernel<false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<false>::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev].store(true, std::memory_order_release);
  }
  const int row_blocks = (p.rows + kRowsPerCta - 1) / kRowsPerCta;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_workers, row_blocks);
  cfg.blockDim = dim3(Cfg<false>::kThreads);
  cfg.dynamicSmemBytes = Cfg<false>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.gather_rows != nullptr)
    e = cudaLaunchKernelEx(&cfg, mla_decode_sm100_kernel<false, true>, tm_q, tm_page, p);
  else
    e = cudaLaunchKernelEx(&cfg, mla_decode_sm100_kernel<false>, tm_q, tm_page, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_decode_fp8(const CUtensorMap& tm_q, const CUtensorMap& tm_page8,
                              const DecodeParams& p, int num_workers, cudaStream_t stream) {
  static std::atomic<bool> configured[64];  // per device: attribute set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(mla_decode_sm100_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<true>::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev].store(true, std::memory_order_release);
  }
  const int row_blocks = (p.rows + kRowsPerCta - 1) / kRowsPerCta;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_workers, row_blocks);
  cfg.blockDim = dim3(Cfg<true>::kThreads);
  cfg.dynamicSmemBytes = Cfg<true>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, mla_decode_sm100_kernel<true>, tm_q, tm_page8, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla

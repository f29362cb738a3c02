// Absorbed MLA decode on the sm_100a tensor cores (tcgen05 + TMEM + TMA), one CTA pair per worker.
//
// The path (« L'attention latente : compresser le cache », « Ce que DeepSeek fait de plus »;
// « Résumé technique : GQLA … », « Chemin MQA-Absorbé »): every head scores the cached rows
// [c_j ; k_r,j] with its absorbed query, softmaxes, and accumulates P·c. Shapes fixed here:
// H = 128 heads, d_c = 512, d_r = 64, one new token per sequence, bf16 storage, fp32 accumulation.
//
// Why a pair: the fp32 accumulator O = 128 heads x 512 latent columns fills all 512 TMEM columns of
// one SM, leaving no room for the scores. So the two CTAs of a cluster split the work by operand:
//   CTA 0 ("score CTA") keeps Q̃ [128 x 576] bf16 in TMEM (288 columns) as the A operand and
//         computes S = Q̃ · [c;k_r]ᵀ for 64-position tiles into three TMEM buffers; its softmax
//         warps turn S into bf16 P and write P straight into CTA 1's shared memory (DSMEM).
//   CTA 1 ("output CTA") holds O in TMEM and issues O += P · C for each tile; its warps rescale
//         O rows when the running maximum moved (lazily: only past 2^8) and run the epilogue.
// No FLOP is done twice. Each CTA TMA-loads the rows it needs (the second read hits L2).
// Work: the tiles of all sequences are laid end to end and cut into one contiguous range per
// pair; a sequence cut between pairs is written as fp32 partials and merged afterwards.
// Every wait is bounded in time; on expiry the kernel records MLA_ERR_TIMEOUT and drains.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace sm100 {

// Optional per-role cycle counters (build with -DMLA_DECODE_PROFILE; absent otherwise).
#ifdef MLA_DECODE_PROFILE
__device__ long long g_prof[148][2][12][16];
#define PROF_DECL() long long prof_[14] = {0}; const long long prof_t0_ = clock64()
#define PROF_MARK(v) const long long v = clock64()
#define PROF_ADD(i, from) (prof_[i] += clock64() - (from))
#define PROF_SAVE(its) do { if (pair < 148) { for (int k_ = 0; k_ < 14; ++k_) g_prof[pair][rank][warp][k_] = prof_[k_]; \
    g_prof[pair][rank][warp][14] = clock64() - prof_t0_; g_prof[pair][rank][warp][15] = (its); } } while (0)
#else
#define PROF_DECL() do {} while (0)
#define PROF_MARK(v) do {} while (0)
#define PROF_ADD(i, from) do {} while (0)
#define PROF_SAVE(its) do {} while (0)
#endif

constexpr int kH = 128, kDC = 512, kDR = 64, kRow = kDC + kDR;
constexpr int kTile = 64;                              // positions per tile = one cache page
constexpr int kChunkBytes = 64 * 128;                  // one TMA box: 64 rows x 64 bf16
constexpr int kKChunks = kRow / 64;                    // 9 chunks per tile on the score CTA
constexpr int kVChunks = kDC / 64;                     // 8 chunks per tile on the output CTA
constexpr int kGroupChunks = 3;                       // score CTA: a ring of 3-chunk groups (24 KB),
constexpr int kGroupsPerTile = kKChunks / kGroupChunks;// 3 per tile, each released as soon as its
constexpr int kRing = 7;                               // 12 MMAs are done
constexpr int kGroupBytes = kGroupChunks * kChunkBytes;// 24576
constexpr int kPrefetchAhead = 3;                      // tiles fetched into L2 ahead of the ring loads
constexpr int kQGroups = 6;                            // a sequence's Q̃ travels the ring first: 18 boxes of
                                                       // 64 heads x 64 columns in 6 groups
constexpr int kVStages = 2;                            // output CTA: whole-tile stages
constexpr int kVStageBytes = kVChunks * kChunkBytes;   // 65536
constexpr int kPSlots = 4;                             // P tiles in flight to the output CTA
constexpr int kStaging = 2;                            // P tiles assembled on the score CTA
constexpr int kPBytes = kH * kTile * 2;                // 16384: P tile, bf16, 128-byte swizzle
constexpr int kPSlotStride = 17408;                    // P, then rescale factor per row, then 4 flags
constexpr int kPCopyBytes = kPBytes + kH * 4 + 16;     // 16912: one bulk copy per tile
constexpr int kSBufs = 3;
constexpr int kQCols = kRow / 2;                       // 288 TMEM columns hold Q̃ as bf16 pairs
constexpr int kSCol0 = kQCols;                         // S buffers at 288, 352, 416
constexpr int kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;                   // lazy rescale threshold (log2 units)
constexpr int kThreads = 384;                          // 4 control warps + 8 softmax / epilogue warps
constexpr int kGroup = 256;                            // threads of the softmax / epilogue warps
constexpr uint64_t kTimeoutNs = 2000000000ull;

// shared memory map (offsets from a 1024-byte aligned base)
//   score CTA:  K group ring [7] | P staging [2]  | row-maximum and row-sum exchange
//   output CTA: V stages [2] | P slots [4]        | 1/l per row | mailbox
constexpr int kOffK = 0;
constexpr int kOffStaging = kRing * kGroupBytes;                       // 172032
constexpr int kOffV = 0;
constexpr int kOffPSlots = kVStages * kVStageBytes;                    // 131072
constexpr int kRegion0 = kOffStaging + kStaging * kPSlotStride;       // 206848
constexpr int kRegion1 = kOffPSlots + kPSlots * kPSlotStride;         // 200704
constexpr int kRegion = kRegion0 > kRegion1 ? kRegion0 : kRegion1;
constexpr int kOffStats = kRegion;                     // float [128] 1/l            (output CTA)
constexpr int kOffXmax = kOffStats + kH * 4;           // float [2][2][128] partial maxima (score CTA)
constexpr int kOffXsum = kOffXmax + 2 * 2 * kH * 4;    // float [2][128] partial sums     (score CTA)
constexpr int kOffMail = kOffXsum + 2 * kH * 4;        // int [4] request to the correction warps
constexpr int kOffBar = kOffMail + 16;
// Barriers. Score CTA: K_*, S_*, Q_FULL, P_EMPTY, STATS_EMPTY. Output CTA: V_*, P_FULL, REQ*,
// RS_READY, SEG_DONE, O_FREE, STATS_FULL. Arrivals from the other CTA reach P_EMPTY, STATS_EMPTY
// (score CTA) and P_FULL, STATS_FULL (output CTA).
enum Bar : int {
  K_FULL = 0, K_EMPTY = K_FULL + kRing, S_FULL = K_EMPTY + kRing, S_EMPTY = S_FULL + kSBufs,
  Q_FULL = S_EMPTY + kSBufs, P_EMPTY = Q_FULL + 1, P_WRITTEN = P_EMPTY + kPSlots,
  STG_FREE = P_WRITTEN + kStaging, STATS_EMPTY = STG_FREE + kStaging,
  V_FULL = STATS_EMPTY + 1, V_EMPTY = V_FULL + kVStages, P_FULL = V_EMPTY + kVStages,
  REQ = P_FULL + kPSlots, REQ_DONE = REQ + 1, RS_READY = REQ_DONE + 1, SEG_DONE = RS_READY + 1,
  O_FREE = SEG_DONE + 1, STATS_FULL = O_FREE + 1, NUM_BARS = STATS_FULL + 1
};
enum Mail : int { MAIL_RESCALE = 1, MAIL_EPILOGUE = 2, MAIL_STOP = 3 };
constexpr int kOffTmemSlot = kOffBar + NUM_BARS * 8;
constexpr int kOffAbort = kOffTmemSlot + 8;
constexpr int kOffWork = kOffAbort + 8;                // long long start, end, off_b, b
constexpr int kSmemUsed = kOffWork + 32;
constexpr int kSmemBytes = kSmemUsed + 1024;           // + alignment slack of the dynamic base
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert((kOffBar % 8) == 0 && (kOffWork % 8) == 0, "alignment");

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 64, false);   // S = Q̃ · Kᵀ   (K-major B)
constexpr uint32_t kIdescO = ptx::idesc_bf16_f32(128, 256, true);   // O += P · C   (MN-major B)

struct Params {
  const __nv_bfloat16* q_abs;  // [B, 128, 576]
  const int32_t* block_table;
  int max_pages;
  int num_pages;
  const int32_t* seqlens;
  int B;
  int max_tiles;               // max_pages: a sequence never reads past its table row
  __nv_bfloat16* o_lat;        // [B, 128, 512]
  float* lse;                  // [B, 128]
  float* part_o;               // [2 * pairs, 128, 512]
  float* part_lse;             // [2 * pairs, 128]
  float sm_scale_log2;         // sm_scale * log2(e)
};

// ---- work split -----------------------------------------------------------------------------------
__device__ __forceinline__ int tiles_of(int L, int max_tiles) { return L > 0 ? min((L + kTile - 1) / kTile, max_tiles) : 0; }

// Walks the segments (sequence, tile range) of one pair's contiguous range of the global tile list.
struct SegIter {
  long long cur, end, off_b;
  int b;
  __device__ bool next(const int32_t* seqlens, int B, int max_tiles, int& bo, int& t_lo, int& t_hi, int& tiles_b) {
    while (cur < end && b < B) {
      const int tb = tiles_of(seqlens[b], max_tiles);
      if (cur >= off_b + tb) {
        off_b += tb;
        ++b;
        continue;
      }
      bo = b;
      t_lo = (int)(cur - off_b);
      t_hi = (int)min((long long)tb, end - off_b);
      tiles_b = tb;
      cur = off_b + t_hi;
      return true;
    }
    return false;
  }
};

// One warp: total tiles T, this pair's range [pair*T/P, (pair+1)*T/P), and the sequence holding its
// first tile. Lane l scans sequences [l*per, (l+1)*per).
__device__ void plan_range(const int32_t* seqlens, int B, int max_tiles, int pair, int npairs, long long* out) {
  const int lane = threadIdx.x & 31;
  const int per = (B + 31) / 32;
  const int b0 = min(B, lane * per), b1 = min(B, b0 + per);
  long long local = 0;
  for (int b = b0; b < b1; ++b) {
    const int L = seqlens[b];
    if (L < 1 || (L + kTile - 1) / kTile > max_tiles) report(MLA_ERR_DEVICE_CHECK);
    local += tiles_of(L, max_tiles);
  }
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const long long T = __shfl_sync(0xffffffffu, incl, 31);
  const long long excl = incl - local;
  const long long start = (long long)pair * T / npairs;
  const long long end = (long long)(pair + 1) * T / npairs;
  if (start < end && start >= excl && start < incl) {
    long long off = excl;
    for (int b = b0; b < b1; ++b) {
      const int tb = tiles_of(seqlens[b], max_tiles);
      if (start < off + tb) {
        out[0] = start; out[1] = end; out[2] = off; out[3] = b;
        break;
      }
      off += tb;
    }
  }
  if (lane == 0 && start >= end) { out[0] = 0; out[1] = 0; out[2] = 0; out[3] = B; }
}

// ---- bounded waits ---------------------------------------------------------------------------------
__device__ __forceinline__ void raise_abort(uint32_t abort_addr) {
  *reinterpret_cast<volatile int*>(__cvta_shared_to_generic(abort_addr)) = 1;
  const uint32_t peer = ptx::map_to_cta(abort_addr, ptx::cluster_ctarank() ^ 1u);
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1) : "memory");
}

// Slow path of wait_bar: polls until the phase completes. Returns false (and makes both CTAs
// abort) after kTimeoutNs, or at once when an abort was raised and `stop_on_abort` is set.
__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, uint32_t abort_addr, bool cluster_scope,
                                           bool stop_on_abort) {
  const volatile int* abort_flag = reinterpret_cast<const volatile int*>(__cvta_shared_to_generic(abort_addr));
  uint64_t t0 = 0;
  for (uint32_t n = 0;; ++n) {
    const bool ok = cluster_scope ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity);
    if (ok) return true;
    if ((n & 15u) == 15u) {
      if (stop_on_abort && *abort_flag) return false;
      const uint64_t now = ptx::globaltimer();
      if (t0 == 0) t0 = now;
      else if (now - t0 > kTimeoutNs) {
        report(MLA_ERR_TIMEOUT);
        raise_abort(abort_addr);
        return false;
      }
    }
  }
}
// Waits for the phase of `parity` to complete; the first probe is inline (a wait that is already
// satisfied costs one mbarrier round trip, not a call).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, uint32_t abort_addr, bool cluster_scope,
                                         bool stop_on_abort = true) {
  const bool ok = cluster_scope ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity);
  return ok || wait_bar_slow(bar, parity, abort_addr, cluster_scope, stop_on_abort);
}
// Warp-uniform version: every lane polls, the warp proceeds only if all lanes saw completion.
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, uint32_t abort_addr, bool cluster_scope) {
  const bool ok = wait_bar(bar, parity, abort_addr, cluster_scope);
  return __all_sync(0xffffffffu, ok);
}

// ---- the kernel ------------------------------------------------------------------------------------
// Warp roles.  Score CTA: 0 TMA producer (+ L2 prefetch ahead) | 1 S-MMA issuer for even tiles, and
// lane 0 of warp 2 for odd tiles (one issuing thread cannot keep the tensor core busy at N = 64) |
// 2 TMEM | 3 copier (one bulk copy of each finished P tile into the output CTA) | 4-11 softmax
// (warps 4-7 columns 0-31 of a tile, warps 8-11 columns 32-63).
// Output CTA: 0 TMA producer | 1 O-MMA issuer | 2 TMEM, then receiver (returns the score CTA's
// staging buffers as P tiles land) | 4-11 correction and epilogue (warps 4-7 latent columns 0-255,
// warps 8-11 columns 256-511).
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope,
              const __grid_constant__ CUtensorMap tm_q, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t rank = ptx::cluster_ctarank();
  const int pair = (int)ptx::cluster_id_x();
  const int npairs = (int)ptx::num_clusters_x();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return base + kOffBar + 8u * (uint32_t)i; };
  const uint32_t abort_addr = base + kOffAbort;
  long long* work = reinterpret_cast<long long*>(gbase + kOffWork);

  if (threadIdx.x == 0) {
    // arrival counts: TMA producers and tcgen05.commit arrive once; thread groups one by one
    for (int i = 0; i < kRing; ++i) { ptx::mbar_init(bar(K_FULL + i), 1); ptx::mbar_init(bar(K_EMPTY + i), 1); }
    for (int i = 0; i < kSBufs; ++i) { ptx::mbar_init(bar(S_FULL + i), 1); ptx::mbar_init(bar(S_EMPTY + i), kGroup); }
    ptx::mbar_init(bar(Q_FULL), kGroup);
    for (int i = 0; i < kPSlots; ++i) { ptx::mbar_init(bar(P_EMPTY + i), 1); ptx::mbar_init(bar(P_FULL + i), 1); }
    for (int i = 0; i < kStaging; ++i) { ptx::mbar_init(bar(P_WRITTEN + i), kGroup); ptx::mbar_init(bar(STG_FREE + i), 1); }
    ptx::mbar_init(bar(STATS_EMPTY), kGroup);
    for (int i = 0; i < kVStages; ++i) { ptx::mbar_init(bar(V_FULL + i), 1); ptx::mbar_init(bar(V_EMPTY + i), 1); }
    ptx::mbar_init(bar(REQ), 1);
    ptx::mbar_init(bar(REQ_DONE), kGroup);
    ptx::mbar_init(bar(RS_READY), 1);
    ptx::mbar_init(bar(SEG_DONE), 1);
    ptx::mbar_init(bar(O_FREE), kGroup);
    ptx::mbar_init(bar(STATS_FULL), kH);
    *reinterpret_cast<volatile int*>(gbase + kOffAbort) = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_lat);
    ptx::prefetch_tmap(&tm_rope);
    ptx::prefetch_tmap(&tm_q);
  }
  if (warp == 2) {
    ptx::tmem_alloc(base + kOffTmemSlot, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 3) plan_range(p.seqlens, p.B, p.max_tiles, pair, npairs, work);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();      // the peer's barriers are initialised before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + kOffTmemSlot);
  SegIter segs{work[0], work[1], work[2], (int)work[3]};
  int b, t_lo, t_hi, tiles_b;

  if (rank == 0) {
    // ============================== score CTA ==============================
    if (warp == 0) {
      if (lane == 0) {   // ---- TMA producer: [c (8 chunks) ; k_r (1 chunk)] of each tile
        uint32_t it = 0;
        bool ok = true;
        // a second walk over the same tiles, kPrefetchAhead ahead, pulls them into L2 (and the
        // next sequence's query block when it starts)
        SegIter ahead = segs;
        int ab = -1, at = 0, a_hi = 0, ax = 0;
        auto prefetch_next = [&]() {
          if (at >= a_hi) {
            if (!ahead.next(p.seqlens, p.B, p.max_tiles, ab, at, a_hi, ax)) { ab = -1; return; }
          }
          int pg = p.block_table[(long long)ab * p.max_pages + at];
          if (pg >= 0 && pg < p.num_pages) {
            for (int j = 0; j < kVChunks; ++j) ptx::tma_prefetch_2d(&tm_lat, 64 * j, pg * kTile);
            ptx::tma_prefetch_2d(&tm_rope, 0, pg * kTile);
          }
          ++at;
        };
        for (int k = 0; k < kPrefetchAhead; ++k) prefetch_next();
        uint32_t gi = 0;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          // the sequence's absorbed query first: box (column block cb, head half rh)
          for (int qg = 0; qg < kQGroups && ok; ++qg, ++gi) {
            const uint32_t s = gi % kRing;
            if (!(ok = wait_bar(bar(K_EMPTY + s), ((gi / kRing) & 1u) ^ 1u, abort_addr, false))) break;
            ptx::mbar_arrive_expect_tx(bar(K_FULL + s), kGroupBytes);
            for (int j = 0; j < kGroupChunks; ++j) {
              const int qc = qg * kGroupChunks + j;
              ptx::tma_load_2d(base + kOffK + s * kGroupBytes + j * kChunkBytes, &tm_q, 64 * (qc >> 1), b * kH + 64 * (qc & 1), bar(K_FULL + s));
            }
          }
          for (int t = t_lo; t < t_hi && ok; ++t, ++it) {
            if (ab >= 0 || at < a_hi) prefetch_next();
            int page = p.block_table[(long long)b * p.max_pages + t];   // issued before the wait
            for (int q = 0; q < kGroupsPerTile && ok; ++q, ++gi) {
              const uint32_t s = gi % kRing;
              if (!(ok = wait_bar(bar(K_EMPTY + s), ((gi / kRing) & 1u) ^ 1u, abort_addr, false))) break;
              if (q == 0 && (page < 0 || page >= p.num_pages)) { report(MLA_ERR_DEVICE_CHECK); page = p.num_pages; }  // off the map: TMA fills zeros
              const uint32_t dst = base + kOffK + s * kGroupBytes;
              ptx::mbar_arrive_expect_tx(bar(K_FULL + s), kGroupBytes);
              for (int j = 0; j < kGroupChunks; ++j) {
                const int c = q * kGroupChunks + j;
                if (c < kVChunks) ptx::tma_load_2d(dst + j * kChunkBytes, &tm_lat, 64 * c, page * kTile, bar(K_FULL + s));
                else ptx::tma_load_2d(dst + j * kChunkBytes, &tm_rope, 0, page * kTile, bar(K_FULL + s));
              }
            }
          }
        }
        // loads still in flight must land before the CTA may exit
        const uint32_t ng = gi;
        for (uint32_t k = (ng > (uint32_t)kRing ? ng - kRing : 0); k < ng; ++k)
          wait_bar(bar(K_FULL + k % kRing), (k / kRing) & 1u, abort_addr, false, false);
      }
    } else if (warp == 3) {
      if (lane == 0) {   // ---- copier: each P tile the softmax warps finished goes to the output CTA
        const uint32_t slot_remote0 = ptx::map_to_cta(base + kOffPSlots, 1);
        uint32_t it = 0;
        bool ok = true;
        PROF_DECL();
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          for (int t = t_lo; t < t_hi; ++t, ++it) {
            const uint32_t stg = it % kStaging, slot = it % kPSlots;
            PROF_MARK(c0);
            if (!(ok = wait_bar(bar(P_WRITTEN + stg), (it / kStaging) & 1u, abort_addr, false))) break;
            PROF_ADD(0, c0);
            PROF_MARK(c1);
            // the slot on the output CTA is free once its MMAs of tile it - kPSlots are done
            if (!(ok = wait_bar(bar(P_EMPTY + slot), ((it / kPSlots) & 1u) ^ 1u, abort_addr, true))) break;
            PROF_ADD(1, c1);
            PROF_MARK(c2);
            const uint32_t full = ptx::map_to_cta(bar(P_FULL + slot), 1);
            ptx::mbar_arrive_expect_tx_remote(bar(P_FULL + slot), 1, kPCopyBytes);
            ptx::bulk_copy_to_cta(slot_remote0 + slot * kPSlotStride, base + kOffStaging + stg * kPSlotStride, kPCopyBytes, full);
            PROF_ADD(2, c2);
          }
        }
        PROF_SAVE(it);
        // before leaving: every copy has landed and every slot came back
        for (uint32_t k = (it > (uint32_t)kPSlots ? it - kPSlots : 0); k < it; ++k)
          wait_bar(bar(P_EMPTY + k % kPSlots), (k / kPSlots) & 1u, abort_addr, true, false);
        for (uint32_t k = (it > (uint32_t)kStaging ? it - kStaging : 0); k < it; ++k)
          wait_bar(bar(STG_FREE + k % kStaging), (k / kStaging) & 1u, abort_addr, true, false);
      }
    } else if (warp == 1 || warp == 2) {
      if (lane == 0) {   // ---- S-MMA issuers: S = Q̃ · [c ; k_r]ᵀ, K = 576 in 36 steps of 16
        const uint32_t parity = warp == 1 ? 0u : 1u;
        const uint64_t k_desc = ptx::smem_desc_sw128(base + kOffK, 16, 1024);
        uint32_t it = 0, seg = 0, gq = 0;
        bool ok = true;
        PROF_DECL();
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          PROF_MARK(q0);
          if (!(ok = wait_bar(bar(Q_FULL), seg & 1u, abort_addr, false))) break;
          PROF_ADD(4, q0);
          ++seg;
          gq += kQGroups;
          for (int t = t_lo; t < t_hi && ok; ++t, ++it, gq += kGroupsPerTile) {
            if ((it & 1u) != parity) continue;
            PROF_MARK(c0);
            const uint32_t sb = it % kSBufs;
            const uint32_t g0 = gq;
            // probe, then block on whichever is not there yet
            const bool se = ptx::mbar_try_wait(bar(S_EMPTY + sb), ((it / kSBufs) & 1u) ^ 1u);
            if (!se && !(ok = wait_bar(bar(S_EMPTY + sb), ((it / kSBufs) & 1u) ^ 1u, abort_addr, false))) break;
            const uint32_t d = tmem + kSCol0 + 64u * sb;
            PROF_ADD(0, c0);
#pragma unroll
            for (int q = 0; q < kGroupsPerTile; ++q) {
              const uint32_t gi = g0 + q, s = gi % kRing;
              PROF_MARK(c1);
              if (!(ok = wait_bar(bar(K_FULL + s), (gi / kRing) & 1u, abort_addr, false))) break;
              PROF_ADD(1, c1);
              PROF_MARK(c2);
              ptx::tc_fence_after();
              const uint64_t gd = k_desc + (uint64_t)(s * (kGroupBytes >> 4));
#pragma unroll
              for (int j = 0; j < kGroupChunks; ++j) {
                // chunk at +8 KB; K-steps of 16 at +32 bytes inside the 128-byte swizzle row
                const uint64_t bd = gd + (uint64_t)(j * (kChunkBytes >> 4));
                const uint32_t a = tmem + 32u * (q * kGroupChunks + j);
#pragma unroll
                for (int k = 0; k < 4; ++k) ptx::mma_ts(d, a + 8u * k, bd + 2 * k, kIdescS, (q | j | k) ? 1u : 0u);
              }
              ptx::mma_commit(bar(K_EMPTY + s));
              PROF_ADD(2, c2);
            }
            if (!ok) break;
            ptx::mma_commit(bar(S_FULL + sb));
          }
        }
        PROF_SAVE(it);
      }
    } else if (warp >= 4) {
      // ---- softmax: thread = (head h = TMEM lane, column half g of the tile)
      const int g = (warp - 4) >> 2;
      const int h = ((warp & 3) << 5) | lane;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t stats_remote = ptx::map_to_cta(base + kOffStats, 1);
      float* xmax = reinterpret_cast<float*>(gbase + kOffXmax);
      float* xsum = reinterpret_cast<float*>(gbase + kOffXsum);
      const float scale2 = p.sm_scale_log2;
      uint32_t it = 0, seg = 0, gq = 0;
      bool ok = true;
      PROF_DECL();
      while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
        const int L = p.seqlens[b];
        PROF_MARK(q0);
        // Q̃ of this sequence into TMEM columns [0, 288), from the 6 ring groups that carry it (the
        // previous segment's S MMAs are done: their last result was read below). Half g fills
        // column blocks [5g, 5 + 4g) of 64 values (32 TMEM columns).
        {
          bool qok = true;
          for (int qg = 0; qg < kQGroups; ++qg)
            qok = qok && wait_bar_warp(bar(K_FULL + (gq + qg) % kRing), ((gq + qg) / kRing) & 1u, abort_addr, false);
          if (qok) {
            const int r = h & 63, rh = h >> 6;
#pragma unroll 1
            for (int cb = g ? 5 : 0; cb < (g ? 9 : 5); ++cb) {
              const int qc = 2 * cb + rh, qg = qc / kGroupChunks, j = qc % kGroupChunks;
              const uint32_t row = base + kOffK + ((gq + qg) % kRing) * kGroupBytes + j * kChunkBytes + r * 128;
              uint32_t v[32];
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const uint4 x = ptx::ld_shared_v4(row + ((uint32_t)(k ^ (r & 7)) << 4));
                v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
              }
              ptx::tmem_st32(tmem + lane_off + 32u * cb, v);
            }
            ptx::tmem_wait_st();
          }
          // the query groups go back to the producer once every thread has read its part
          if (ptx::named_bar_or(4, kGroup, !qok)) { ok = false; break; }
          if (threadIdx.x == 128)
            for (int qg = 0; qg < kQGroups; ++qg) ptx::mbar_arrive(bar(K_EMPTY + (gq + qg) % kRing));
          gq += kQGroups;
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(Q_FULL));
        }
        PROF_ADD(7, q0);
        int nb = -1;
        {
          SegIter peek = segs;
          int x0, x1, x2;
          if (!peek.next(p.seqlens, p.B, p.max_tiles, nb, x0, x1, x2)) nb = -1;
        }
        float m = -INFINITY, l = 0.f;
        gq += kGroupsPerTile * (t_hi - t_lo);
        for (int t = t_lo; t < t_hi; ++t, ++it) {
          const uint32_t s = it % kSBufs, stg = it % kStaging;
          if (nb >= 0 && t == max(t_lo, t_hi - 3)) {   // the next segment's query row into L2
            const char* nq = reinterpret_cast<const char*>(p.q_abs + ((size_t)nb * kH + h) * kRow);
            for (int k = g ? 5 : 0; k < (g ? 9 : 5); ++k) ptx::prefetch_l2(nq + 128 * k);
          }
          // probe this tile's staging buffer now; the answer is used after the softmax arithmetic
          bool stg_free = ptx::mbar_test_wait_cluster(bar(STG_FREE + stg), ((it / kStaging) & 1u) ^ 1u);
          PROF_MARK(c0);
          bool good = wait_bar_warp(bar(S_FULL + s), (it / kSBufs) & 1u, abort_addr, false);
          PROF_ADD(0, c0);
          PROF_MARK(c1);
          uint32_t sr[32];
          const int valid = min(kTile, L - t * kTile) - 32 * g;     // valid columns of this half
          float pm = -INFINITY;
          if (good) {
            ptx::tc_fence_after();
            ptx::tmem_ld32(tmem + lane_off + kSCol0 + 64u * s + 32u * g, sr);
            ptx::tmem_wait_ld();
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar(S_EMPTY + s));
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < valid) mx[j & 3] = fmaxf(mx[j & 3], __uint_as_float(sr[j]));
            pm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            xmax[((it & 1) * 2 + g) * kH + h] = pm;
          }
          PROF_ADD(1, c1);
          PROF_MARK(c2);
          // all 256 threads meet here every tile and agree whether to stop
          if (ptx::named_bar_or(1, kGroup, !good)) { ok = false; break; }
          PROF_ADD(2, c2);
          PROF_MARK(c3);
          const float m_tile = fmaxf(pm, xmax[((it & 1) * 2 + (g ^ 1)) * kH + h]) * scale2;
          float alpha = 1.f;
          if (m_tile > m + kRescaleLog2) {
            alpha = (m == -INFINITY) ? 0.f : ptx::ex2_approx(m - m_tile);
            l *= alpha;
            m = m_tile;
          }
          uint32_t pk[16];
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float e0 = (j < valid) ? ptx::ex2_approx(fmaf(__uint_as_float(sr[j]), scale2, -m)) : 0.f;
            const float e1 = (j + 1 < valid) ? ptx::ex2_approx(fmaf(__uint_as_float(sr[j + 1]), scale2, -m)) : 0.f;
            ls[(j >> 1) & 3] += e0 + e1;
            pk[j / 2] = ptx::pack_bf16x2(e0, e1);
          }
          l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
          PROF_ADD(3, c3);
          PROF_MARK(c4);
          // this tile's staging buffer must have been copied out (tile it - kStaging)
          if (!__all_sync(0xffffffffu, stg_free) &&
              !wait_bar_warp(bar(STG_FREE + stg), ((it / kStaging) & 1u) ^ 1u, abort_addr, true))
            continue;
          PROF_ADD(4, c4);
          PROF_MARK(c5);
          const uint32_t st0 = base + kOffStaging + stg * kPSlotStride;
          const uint32_t row = st0 + (uint32_t)(h >> 3) * 1024u + (uint32_t)(h & 7) * 128u;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int c = 4 * g + k;
            ptx::st_shared_v4(row + ((uint32_t)(c ^ (h & 7)) << 4), pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          }
          if (g == 0) {
            reinterpret_cast<float*>(gbase + kOffStaging + stg * kPSlotStride + kPBytes)[h] = alpha;
            const bool rescaled = __any_sync(0xffffffffu, alpha != 1.f);
            if (lane == 0)
              reinterpret_cast<int*>(gbase + kOffStaging + stg * kPSlotStride + kPBytes + kH * 4)[warp & 3] = rescaled ? 1 : 0;
          }
          // visible to the bulk copy (async proxy), then handed to the copier
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(bar(P_WRITTEN + stg));
          PROF_ADD(5, c5);
        }
        if (!ok) break;
        // segment end: combine the two halves' row sums; 1/l to the output CTA, lse to memory
        xsum[g * kH + h] = l;
        if (ptx::named_bar_or(2, kGroup, false)) { ok = false; break; }
        l = xsum[h] + xsum[kH + h];
        bool fail = false;
        if (g == 0) {
          if (!wait_bar_warp(bar(STATS_EMPTY), (seg & 1u) ^ 1u, abort_addr, true)) {
            fail = true;
          } else {
            const bool partial = !(t_lo == 0 && t_hi == tiles_b);
            const float lse = (m + log2f(l)) * 0.69314718055994531f;
            if (partial) p.part_lse[((size_t)pair * 2 + (seg > 0)) * kH + h] = lse;
            else p.lse[(size_t)b * kH + h] = lse;
            ptx::st_cluster_f32(stats_remote + h * 4u, 1.f / l);
            ptx::mbar_arrive_remote(bar(STATS_FULL), 1);
          }
        }
        // both halves leave together if either failed (the next segment meets at named barriers)
        if (ptx::named_bar_or(3, kGroup, fail)) { ok = false; break; }
        ++seg;
      }
      PROF_SAVE(it);
      // before leaving: the output CTA's last release of the stats must have landed here
      if (g == 0 && seg > 0) wait_bar(bar(STATS_EMPTY), (seg - 1) & 1u, abort_addr, true, false);
    }
  } else {
    // ============================== output CTA ==============================
    if (warp == 2) {
      if (lane == 0) {   // ---- receiver: as each P tile lands, the score CTA may reuse that staging buffer
        uint32_t it = 0;
        bool ok = true;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          for (int t = t_lo; t < t_hi; ++t, ++it) {
            if (!(ok = wait_bar(bar(P_FULL + it % kPSlots), (it / kPSlots) & 1u, abort_addr, true))) break;
            ptx::mbar_arrive_remote(bar(STG_FREE + it % kStaging), 0);
          }
        }
      }
    } else if (warp == 0) {
      if (lane == 0) {   // ---- TMA producer: latent rows c of each tile
        uint32_t it = 0;
        bool ok = true;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          for (int t = t_lo; t < t_hi && ok; ++t, ++it) {
            const uint32_t s = it % kVStages;
            int page = p.block_table[(long long)b * p.max_pages + t];   // issued before the wait
            if (!(ok = wait_bar(bar(V_EMPTY + s), ((it / kVStages) & 1u) ^ 1u, abort_addr, false))) break;
            if (page < 0 || page >= p.num_pages) page = p.num_pages;   // reported by the score CTA
            const uint32_t dst = base + kOffV + s * kVStageBytes;
            ptx::mbar_arrive_expect_tx(bar(V_FULL + s), kVStageBytes);
            for (int j = 0; j < kVChunks; ++j) ptx::tma_load_2d(dst + j * kChunkBytes, &tm_lat, 64 * j, page * kTile, bar(V_FULL + s));
          }
        }
        for (uint32_t k = (it > (uint32_t)kVStages ? it - kVStages : 0); k < it; ++k)
          wait_bar(bar(V_FULL + k % kVStages), (k / kVStages) & 1u, abort_addr, false, false);
      }
    } else if (warp == 1) {
      // ---- MMA issuer (lane 0) with the warp's help for masking: O += P · C, K = 64 positions in
      // 4 steps of 16, N = 512 in 2 halves
      const uint64_t v_desc0 = ptx::smem_desc_sw128(base + kOffV, kChunkBytes, 1024);
      const uint64_t p_desc0 = ptx::smem_desc_sw128(base + kOffPSlots, 16, 1024);
      volatile int* mail = reinterpret_cast<volatile int*>(gbase + kOffMail);
      uint32_t it = 0, seg = 0, nresc = 0;
      bool ok = true;
      PROF_DECL();
      while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
        const int L = p.seqlens[b];
        // the previous segment's epilogue has read O out of TMEM
        PROF_MARK(f0);
        if (!(ok = wait_bar_warp(bar(O_FREE), (seg & 1u) ^ 1u, abort_addr, false))) break;
        PROF_ADD(4, f0);
        for (int t = t_lo; t < t_hi; ++t, ++it) {
          const uint32_t slot = it % kPSlots, s = it % kVStages;
          PROF_MARK(c0);
          if (!(ok = wait_bar_warp(bar(P_FULL + slot), (it / kPSlots) & 1u, abort_addr, true))) break;
          PROF_ADD(0, c0);
          const volatile int* flags = reinterpret_cast<const volatile int*>(gbase + kOffPSlots + slot * kPSlotStride + kPBytes + kH * 4);
          const bool resc = (t > t_lo) && (flags[0] | flags[1] | flags[2] | flags[3]);
          if (resc) {
            // some rows' maximum moved: the correction warps rescale O once the MMAs so far are done
            if (lane == 0) {
              ptx::mma_commit(bar(RS_READY));
              mail[0] = MAIL_RESCALE;
              mail[1] = (int)slot;
              ptx::mbar_arrive(bar(REQ));
            }
            if (!(ok = wait_bar_warp(bar(REQ_DONE), nresc & 1u, abort_addr, false))) break;
            ++nresc;
          }
          PROF_MARK(c2);
          if (!(ok = wait_bar_warp(bar(V_FULL + s), (it / kVStages) & 1u, abort_addr, false))) break;
          PROF_ADD(1, c2);
          PROF_MARK(c3);
          // the last page of a sequence: skip whole 16-row steps past its end and zero the rows of
          // the last step that lie past it (a pool row there may hold anything, and 0 * NaN = NaN)
          int nk = kTile / 16;
          if (t == tiles_b - 1) {
            const int valid = L - t * kTile;
            nk = (valid + 15) / 16;
            const int zr = nk * 16 - valid;
            if (zr > 0) {
              uint8_t* vst = gbase + kOffV + s * kVStageBytes;
              for (int i = lane; i < zr * kVChunks * 8; i += 32) {
                const int r = valid + i / (kVChunks * 8), rest = i % (kVChunks * 8);
                reinterpret_cast<uint4*>(vst + (rest / 8) * kChunkBytes + r * 128)[rest % 8] = make_uint4(0, 0, 0, 0);
              }
              ptx::fence_proxy_async_smem();
              __syncwarp();
            }
          }
          if (lane == 0) {
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_after();
            const uint64_t pd = p_desc0 + (uint64_t)(slot * (kPSlotStride >> 4));
            const uint64_t vd = v_desc0 + (uint64_t)(s * (kVStageBytes >> 4));
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              if (kk < nk) {
                const uint32_t acc = (t > t_lo || kk > 0) ? 1u : 0u;
                ptx::mma_ss(tmem, pd + 2 * kk, vd + 128 * kk, kIdescO, acc);
                ptx::mma_ss(tmem + 256, pd + 2 * kk, vd + 2048 + 128 * kk, kIdescO, acc);
              }
            }
            ptx::mma_commit(bar(V_EMPTY + s));
            ptx::mma_commit_mc(bar(P_EMPTY + slot), (uint16_t)0x1);
          }
          __syncwarp();
          PROF_ADD(2, c3);
        }
        if (!ok) break;
        // segment complete once its MMAs are: hand O to the epilogue
        if (lane == 0) {
          ptx::mma_commit(bar(SEG_DONE));
          mail[0] = MAIL_EPILOGUE;
          mail[1] = (int)seg;
          ptx::mbar_arrive(bar(REQ));
        }
        ++seg;
      }
      if (lane == 0) PROF_SAVE(it);
      if (lane == 0) {
        // let the correction warps leave (after the last epilogue has freed O)
        if (seg > 0) wait_bar(bar(O_FREE), (seg - 1) & 1u, abort_addr, false, false);
        mail[0] = MAIL_STOP;
        ptx::mbar_arrive(bar(REQ));
      }
    } else if (warp >= 4) {
      // ---- correction + epilogue: thread = (head h = TMEM lane, latent half g). Serves the
      // requests of the MMA warp in order: rescale O rows, or write out a finished segment.
      const int g = (warp - 4) >> 2;
      const int h = ((warp & 3) << 5) | lane;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t col0 = 256u * g;
      const volatile float* stats_s = reinterpret_cast<const volatile float*>(gbase + kOffStats);
      const volatile int* mail = reinterpret_cast<const volatile int*>(gbase + kOffMail);
      uint32_t nreq = 0, nresc = 0, seg = 0;
      while (true) {
        if (!wait_bar_warp(bar(REQ), nreq & 1u, abort_addr, false)) break;
        ++nreq;
        const int kind = mail[0], arg = mail[1];
        if (kind == MAIL_STOP) break;
        if (kind == MAIL_RESCALE) {
          if (!wait_bar_warp(bar(RS_READY), nresc & 1u, abort_addr, false)) break;
          ++nresc;
          ptx::tc_fence_after();
          const float alpha = reinterpret_cast<const volatile float*>(gbase + kOffPSlots + arg * kPSlotStride + kPBytes)[h];
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
            for (int c = 0; c < kDC / 2; c += 32) {
              uint32_t r[32];
              ptx::tmem_ld32(tmem + lane_off + col0 + c, r);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
              ptx::tmem_st32(tmem + lane_off + col0 + c, r);
            }
            ptx::tmem_wait_st();
          }
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(REQ_DONE));
          continue;
        }
        // MAIL_EPILOGUE: O / l  ->  o_lat (bf16) or an fp32 partial
        if (!segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) break;
        if (!wait_bar_warp(bar(SEG_DONE), seg & 1u, abort_addr, false)) break;
        if (!wait_bar_warp(bar(STATS_FULL), seg & 1u, abort_addr, true)) break;
        ptx::tc_fence_after();
        const float inv_l = stats_s[h];
        const bool partial = !(t_lo == 0 && t_hi == tiles_b);
        if (partial) {
          float* dst = p.part_o + (((size_t)pair * 2 + (seg > 0)) * kH + h) * kDC + col0;
#pragma unroll 1
          for (int c = 0; c < kDC / 2; c += 32) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_off + col0 + c, r);
            ptx::tmem_wait_ld();
            float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              d4[k] = make_float4(__uint_as_float(r[4 * k]) * inv_l, __uint_as_float(r[4 * k + 1]) * inv_l,
                                  __uint_as_float(r[4 * k + 2]) * inv_l, __uint_as_float(r[4 * k + 3]) * inv_l);
          }
        } else {
          __nv_bfloat16* dst = p.o_lat + ((size_t)b * kH + h) * kDC + col0;
#pragma unroll 1
          for (int c = 0; c < kDC / 2; c += 32) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_off + col0 + c, r);
            ptx::tmem_wait_ld();
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              d4[k] = make_uint4(ptx::pack_bf16x2(__uint_as_float(r[8 * k]) * inv_l, __uint_as_float(r[8 * k + 1]) * inv_l),
                                 ptx::pack_bf16x2(__uint_as_float(r[8 * k + 2]) * inv_l, __uint_as_float(r[8 * k + 3]) * inv_l),
                                 ptx::pack_bf16x2(__uint_as_float(r[8 * k + 4]) * inv_l, __uint_as_float(r[8 * k + 5]) * inv_l),
                                 ptx::pack_bf16x2(__uint_as_float(r[8 * k + 6]) * inv_l, __uint_as_float(r[8 * k + 7]) * inv_l));
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(O_FREE));
        ptx::mbar_arrive_remote(bar(STATS_EMPTY), 0);
        ++seg;
      }
    }
  }

  // teardown: TMEM back, then leave together so no remote access can target an exited CTA
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  ptx::cluster_sync();
}

// ---- merge of split sequences ------------------------------------------------------------------------
// pair p covers global tiles [p*T/P, (p+1)*T/P); the pair holding tile x is floor(((x+1)*P - 1) / T).
__device__ __forceinline__ int pair_of(long long x, long long T, int P) { return (int)(((x + 1) * P - 1) / T); }

__global__ void __launch_bounds__(256)
merge_kernel(const int32_t* __restrict__ seqlens, int B, int max_tiles, int npairs, const float* __restrict__ part_o,
             const float* __restrict__ part_lse, __nv_bfloat16* __restrict__ o_lat, float* __restrict__ lse) {
  __shared__ long long sh[3];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    const int per = (B + 31) / 32;
    const int b0 = min(B, lane * per), b1 = min(B, b0 + per);
    long long local = 0, before = 0;
    for (int x = b0; x < b1; ++x) {
      const int tb = tiles_of(seqlens[x], max_tiles);
      if (x < b) before += tb;
      local += tb;
    }
    long long incl = local, incl_b = before;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, incl, o);
      const long long w = __shfl_up_sync(0xffffffffu, incl_b, o);
      if (lane >= o) { incl += v; incl_b += w; }
    }
    if (lane == 31) { sh[0] = incl; sh[1] = incl_b; sh[2] = tiles_of(seqlens[b], max_tiles); }
  }
  __syncthreads();
  const long long T = sh[0], off = sh[1], tb = sh[2];
  if (tb == 0 || T == 0) return;
  const int p0 = pair_of(off, T, npairs), p1 = pair_of(off + tb - 1, T, npairs);
  if (p0 == p1) return;                       // written whole by one pair
  // one head per warp; lanes cover 16 columns each. A pair with an empty range wrote nothing.
  const int h = blockIdx.y * 8 + warp;
  auto slot = [&](int q) -> int {
    const long long start_q = (long long)q * T / npairs;
    if ((long long)(q + 1) * T / npairs <= start_q) return -1;
    return q * 2 + (start_q < off ? 1 : 0);
  };
  float mx = -INFINITY;
  for (int q0 = p0; q0 <= p1; q0 += 32) {     // the partials' lse values, one lane each
    const int q = q0 + lane;
    const int idx = q <= p1 ? slot(q) : -1;
    mx = fmaxf(mx, warp_max(idx >= 0 ? part_lse[(size_t)idx * kH + h] : -INFINITY));
  }
  float tot = 0.f;
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
#pragma unroll 2
  for (int q = p0; q <= p1; ++q) {
    const int idx = slot(q);
    if (idx < 0) continue;
    const float wgt = exp2f((part_lse[(size_t)idx * kH + h] - mx) * 1.4426950408889634f);
    tot += wgt;
    const float4* src = reinterpret_cast<const float4*>(part_o + ((size_t)idx * kH + h) * kDC + lane * 16);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = src[k];
      acc[4 * k] = fmaf(wgt, v.x, acc[4 * k]);
      acc[4 * k + 1] = fmaf(wgt, v.y, acc[4 * k + 1]);
      acc[4 * k + 2] = fmaf(wgt, v.z, acc[4 * k + 2]);
      acc[4 * k + 3] = fmaf(wgt, v.w, acc[4 * k + 3]);
    }
  }
  const float inv = 1.f / tot;
  uint4* dst = reinterpret_cast<uint4*>(o_lat + ((size_t)b * kH + h) * kDC + lane * 16);
  dst[0] = make_uint4(ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv), ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv),
                      ptx::pack_bf16x2(acc[4] * inv, acc[5] * inv), ptx::pack_bf16x2(acc[6] * inv, acc[7] * inv));
  dst[1] = make_uint4(ptx::pack_bf16x2(acc[8] * inv, acc[9] * inv), ptx::pack_bf16x2(acc[10] * inv, acc[11] * inv),
                      ptx::pack_bf16x2(acc[12] * inv, acc[13] * inv), ptx::pack_bf16x2(acc[14] * inv, acc[15] * inv));
  if (lane == 0) lse[(size_t)b * kH + h] = mx + logf(tot);
}

// ---- host side -----------------------------------------------------------------------------------------
inline bool decode_supported(const mla_dims_t* d, int32_t dtype, int32_t B, int32_t s_q) {
  return dtype == MLA_BF16 && d->H == kH && d->d_c == kDC && d->d_r == kDR && s_q == 1 && B >= 1;
}

inline int max_pairs(int num_sms) { return num_sms / 2; }

inline size_t decode_workspace_bytes(const mla_dims_t* d, int32_t dtype, int32_t B, int32_t s_q, int num_sms) {
  if (!decode_supported(d, dtype, B, s_q)) return 0;
  const size_t slots = (size_t)2 * max_pairs(num_sms);
  return slots * kH * kDC * sizeof(float) + slots * kH * sizeof(float) + 256;
}

inline bool make_tmap(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t stride_elems) {
  return tmap::make_bf16_sw128(m, base, cols, rows, stride_elems, kTile);
}

inline int active_pairs(int num_sms) {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev]) return cached[dev];
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * max_pairs(num_sms));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  if (cudaOccupancyMaxActiveClusters(&n, decode_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = max_pairs(num_sms);
  }
  cached[dev] = std::min(n, max_pairs(num_sms));
  return cached[dev];
}

inline int launch_decode(const mla_dims_t* d, int32_t B, int32_t s_q, const void* q_abs, const mla_latent_cache_t* cache,
                         const int32_t* block_table, int32_t max_pages, const int32_t* seqlens, void* o_lat, float* lse,
                         void* workspace, size_t ws_bytes, int num_sms, cudaStream_t st) {
  (void)s_q;
  if (!workspace || ws_bytes < decode_workspace_bytes(d, MLA_BF16, B, 1, num_sms)) return MLA_ERR_WORKSPACE;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
      return MLA_ERR_CUDA;
    attr_done[dev] = true;
  }
  CUtensorMap tm_lat, tm_rope;
  const int64_t rows = (int64_t)cache->num_pages * kTile;
  if (!make_tmap(&tm_lat, cache->latent, kDC, rows, cache->latent_stride)) return MLA_ERR_INVALID_ARG;
  if (!make_tmap(&tm_rope, cache->rope, kDR, rows, cache->rope_stride)) return MLA_ERR_INVALID_ARG;
  CUtensorMap tm_q;   // q_abs as [B*128 heads, 576]: boxes of 64 heads x 64 columns
  if (!make_tmap(&tm_q, q_abs, kRow, (int64_t)B * kH, kRow)) return MLA_ERR_INVALID_ARG;
  const int P = active_pairs(num_sms);
  Params prm;
  prm.q_abs = reinterpret_cast<const __nv_bfloat16*>(q_abs);
  prm.block_table = block_table;
  prm.max_pages = max_pages;
  prm.num_pages = cache->num_pages;
  prm.seqlens = seqlens;
  prm.B = B;
  prm.max_tiles = max_pages;
  prm.o_lat = reinterpret_cast<__nv_bfloat16*>(o_lat);
  prm.lse = lse;
  prm.part_o = reinterpret_cast<float*>(workspace);
  prm.part_lse = prm.part_o + (size_t)2 * max_pairs(num_sms) * kH * kDC;
  prm.sm_scale_log2 = d->sm_scale * 1.4426950408889634f;
  launch(decode_kernel, dim3(2 * P), dim3(kThreads), kSmemBytes, st, tm_lat, tm_rope, tm_q, prm);
  launch(merge_kernel, dim3(B, kH / 8), dim3(256), 0, st, seqlens, (int)B, (int)max_pages, P, (const float*)prm.part_o,
         (const float*)prm.part_lse, prm.o_lat, lse);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla

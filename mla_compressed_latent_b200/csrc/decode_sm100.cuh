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

namespace mla {
namespace sm100 {

constexpr int kH = 128, kDC = 512, kDR = 64, kRow = kDC + kDR;
constexpr int kTile = 64;                              // positions per tile = one cache page
constexpr int kChunkBytes = 64 * 128;                  // one TMA box: 64 rows x 64 bf16
constexpr int kKChunks = kRow / 64;                    // 9
constexpr int kVChunks = kDC / 64;                     // 8
constexpr int kKStages = 3;
constexpr int kKStageBytes = kKChunks * kChunkBytes;   // 73728
constexpr int kVStages = 2;
constexpr int kVStageBytes = kVChunks * kChunkBytes;   // 65536
constexpr int kPSlots = 2;
constexpr int kPSlotBytes = kH * kTile * 2;            // 16384
constexpr int kSBufs = 3;
constexpr int kQCols = kRow / 2;                       // 288 TMEM columns hold Q̃ as bf16 pairs
constexpr int kSCol0 = kQCols;                         // S buffers at 288, 352, 416
constexpr int kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;                   // lazy rescale threshold (log2 units)
constexpr int kThreads = 256;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// shared memory map (offsets from a 1024-byte aligned base; same map in both CTAs)
constexpr int kOffStage = 0;                           // CTA 0: K stages; CTA 1: V stages, P slots
constexpr int kOffP = kVStages * kVStageBytes;
constexpr int kStageRegion = kKStages * kKStageBytes;
static_assert(kOffP + kPSlots * kPSlotBytes <= kStageRegion, "CTA 1 buffers exceed the stage region");
constexpr int kOffAlpha = kStageRegion;                // float [kPSlots][128]   (CTA 1)
constexpr int kOffStats = kOffAlpha + kPSlots * kH * 4;// float [128] 1/l        (CTA 1)
constexpr int kOffBar = kOffStats + kH * 4;
enum Bar : int {
  K_FULL = 0, K_EMPTY = K_FULL + kKStages, S_FULL = K_EMPTY + kKStages, S_EMPTY = S_FULL + kSBufs,
  Q_FULL = S_EMPTY + kSBufs, P_EMPTY = Q_FULL + 1, STATS_EMPTY = P_EMPTY + kPSlots,
  V_FULL = STATS_EMPTY + 1, V_EMPTY = V_FULL + kVStages, P_FULL = V_EMPTY + kVStages,
  CORR_DONE = P_FULL + kPSlots, O_DONE = CORR_DONE + kPSlots, O_FREE = O_DONE + 2,
  STATS_FULL = O_FREE + 1, NUM_BARS = STATS_FULL + 1
};
constexpr int kOffTmemSlot = kOffBar + NUM_BARS * 8;
constexpr int kOffAbort = kOffTmemSlot + 8;
constexpr int kOffWork = kOffAbort + 8;                // long long start, end, off_b; int b
constexpr int kSmemUsed = kOffWork + 32;
constexpr int kSmemBytes = kSmemUsed + 1024;           // + alignment slack of the dynamic base
static_assert(kSmemBytes <= 232448, "shared memory budget");

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
  // the lane whose sequences contain tile `start` finds it
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

// Waits for the phase of `parity` to complete. Returns false (and makes both CTAs abort) after
// kTimeoutNs, or at once when an abort was raised and `stop_on_abort` is set.
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, uint32_t abort_addr, bool cluster_scope,
                                      bool stop_on_abort = true) {
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
// Warp-uniform version: every lane polls, the warp proceeds only if all lanes saw completion.
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, uint32_t abort_addr, bool cluster_scope) {
  const bool ok = wait_bar(bar, parity, abort_addr, cluster_scope);
  return __all_sync(0xffffffffu, ok);
}

// ---- the kernel ------------------------------------------------------------------------------------
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope, const Params p) {
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
    // arrival counts: tcgen05.commit and TMA producers arrive once; thread groups of 128 arrive
    // one by one
    for (int i = 0; i < kKStages; ++i) { ptx::mbar_init(bar(K_FULL + i), 1); ptx::mbar_init(bar(K_EMPTY + i), 1); }
    for (int i = 0; i < kSBufs; ++i) { ptx::mbar_init(bar(S_FULL + i), 1); ptx::mbar_init(bar(S_EMPTY + i), 128); }
    ptx::mbar_init(bar(Q_FULL), 128);
    for (int i = 0; i < kPSlots; ++i) {
      ptx::mbar_init(bar(P_EMPTY + i), 1);
      ptx::mbar_init(bar(P_FULL + i), 128);
      ptx::mbar_init(bar(CORR_DONE + i), 128);
    }
    ptx::mbar_init(bar(STATS_EMPTY), 128);
    for (int i = 0; i < kVStages; ++i) { ptx::mbar_init(bar(V_FULL + i), 1); ptx::mbar_init(bar(V_EMPTY + i), 1); }
    ptx::mbar_init(bar(O_DONE), 1);
    ptx::mbar_init(bar(O_DONE + 1), 1);
    ptx::mbar_init(bar(O_FREE), 128);
    ptx::mbar_init(bar(STATS_FULL), 128);
    *reinterpret_cast<volatile int*>(gbase + kOffAbort) = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_lat);
    ptx::prefetch_tmap(&tm_rope);
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
      if (lane == 0) {   // ---- TMA producer: [c ; k_r] rows of each tile
        uint32_t it = 0;
        bool ok = true;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          for (int t = t_lo; t < t_hi && ok; ++t, ++it) {
            const uint32_t s = it % kKStages;
            if (!(ok = wait_bar(bar(K_EMPTY + s), ((it / kKStages) & 1u) ^ 1u, abort_addr, false))) break;
            int page = p.block_table[(long long)b * p.max_pages + t];
            if (page < 0 || page >= p.num_pages) { report(MLA_ERR_DEVICE_CHECK); page = p.num_pages; }  // out of the map: TMA fills zeros
            const uint32_t dst = base + kOffStage + s * kKStageBytes;
            ptx::mbar_arrive_expect_tx(bar(K_FULL + s), kKStageBytes);
            for (int j = 0; j < kVChunks; ++j) ptx::tma_load_2d(dst + j * kChunkBytes, &tm_lat, 64 * j, page * kTile, bar(K_FULL + s));
            ptx::tma_load_2d(dst + kVChunks * kChunkBytes, &tm_rope, 0, page * kTile, bar(K_FULL + s));
          }
        }
        // loads still in flight must land before the CTA may exit
        for (uint32_t k = (it > kKStages ? it - kKStages : 0); k < it; ++k)
          wait_bar(bar(K_FULL + k % kKStages), (k / kKStages) & 1u, abort_addr, false, false);
      }
    } else if (warp == 1) {
      if (lane == 0) {   // ---- MMA issuer: S = Q̃ · [c ; k_r]ᵀ, K = 576 in 36 steps of 16
        uint32_t it = 0, seg = 0;
        bool ok = true;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          if (!(ok = wait_bar(bar(Q_FULL), seg & 1u, abort_addr, false))) break;
          ++seg;
          for (int t = t_lo; t < t_hi; ++t, ++it) {
            const uint32_t s = it % kKStages, sb = it % kSBufs;
            if (!(ok = wait_bar(bar(K_FULL + s), (it / kKStages) & 1u, abort_addr, false))) break;
            if (!(ok = wait_bar(bar(S_EMPTY + sb), ((it / kSBufs) & 1u) ^ 1u, abort_addr, false))) break;
            ptx::tc_fence_after();
            const uint32_t kst = base + kOffStage + s * kKStageBytes;
            const uint32_t d = tmem + kSCol0 + 64u * sb;
#pragma unroll 4
            for (int k = 0; k < kRow / 16; ++k) {
              const uint64_t bdesc = ptx::smem_desc_sw128(kst + (k >> 2) * kChunkBytes + (k & 3) * 32, 16, 1024);
              ptx::mma_ts(d, tmem + 8u * k, bdesc, kIdescS, k > 0);
            }
            ptx::mma_commit(bar(S_FULL + sb));
            ptx::mma_commit(bar(K_EMPTY + s));
          }
        }
      }
    } else if (warp >= 4) {
      // ---- softmax warpgroup: thread = head h = TMEM lane
      const int h = threadIdx.x - 128;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t p_slot0 = ptx::map_to_cta(base + kOffP, 1);
      const uint32_t alpha0 = ptx::map_to_cta(base + kOffAlpha, 1);
      const uint32_t stats0 = ptx::map_to_cta(base + kOffStats, 1);
      const float scale2 = p.sm_scale_log2;
      uint32_t it = 0, seg = 0;
      bool ok = true;
      while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
        const int L = p.seqlens[b];
        // Q̃ of this sequence into TMEM columns [0, 288): the S MMAs of the previous segment are
        // complete (their last result was read below)
        const uint4* qsrc = reinterpret_cast<const uint4*>(p.q_abs + ((size_t)b * kH + h) * kRow);
#pragma unroll 1
        for (int c = 0; c < kQCols; c += 32) {
          uint32_t r[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 v = __ldg(qsrc + (c / 4) + k);
            r[4 * k] = v.x; r[4 * k + 1] = v.y; r[4 * k + 2] = v.z; r[4 * k + 3] = v.w;
          }
          ptx::tmem_st32(tmem + lane_off + c, r);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(Q_FULL));

        float m = -INFINITY, l = 0.f;
        for (int t = t_lo; t < t_hi; ++t, ++it) {
          const uint32_t sb = it % kSBufs, slot = it % kPSlots;
          if (!(ok = wait_bar_warp(bar(S_FULL + sb), (it / kSBufs) & 1u, abort_addr, false))) break;
          ptx::tc_fence_after();
          uint32_t sr[64];
          ptx::tmem_ld32(tmem + lane_off + kSCol0 + 64u * sb, *reinterpret_cast<uint32_t(*)[32]>(sr));
          ptx::tmem_ld32(tmem + lane_off + kSCol0 + 64u * sb + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
          ptx::tmem_wait_ld();
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(S_EMPTY + sb));

          const int valid = min(kTile, L - t * kTile);
          float mt = -INFINITY;
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (j < valid) mt = fmaxf(mt, __uint_as_float(sr[j]));
          const float m_tile = mt * scale2;
          float alpha = 1.f;
          if (m_tile > m + kRescaleLog2) {
            alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_tile);
            l *= alpha;
            m = m_tile;
          }
          uint32_t pk[32];
          float lsum = 0.f;
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            const float e0 = (j < valid) ? exp2f(fmaf(__uint_as_float(sr[j]), scale2, -m)) : 0.f;
            const float e1 = (j + 1 < valid) ? exp2f(fmaf(__uint_as_float(sr[j + 1]), scale2, -m)) : 0.f;
            lsum += e0 + e1;
            pk[j / 2] = ptx::pack_bf16x2(e0, e1);
          }
          l += lsum;
          // P slot must be free (the MMAs that read it have completed)
          if (!(ok = wait_bar_warp(bar(P_EMPTY + slot), ((it / kPSlots) & 1u) ^ 1u, abort_addr, true))) break;
          const uint32_t row = p_slot0 + slot * kPSlotBytes + (uint32_t)(h >> 3) * 1024u + (uint32_t)(h & 7) * 128u;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            ptx::st_cluster_v4(row + ((uint32_t)(c ^ (h & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          ptx::st_cluster_f32(alpha0 + (slot * kH + h) * 4u, alpha);
          asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
          ptx::mbar_arrive_remote(bar(P_FULL + slot), 1);
        }
        if (!ok) break;
        // segment end: 1/l to the output CTA, lse to global memory
        if (!(ok = wait_bar_warp(bar(STATS_EMPTY), (seg & 1u) ^ 1u, abort_addr, true))) break;
        const bool partial = !(t_lo == 0 && t_hi == tiles_b);
        const float lse = (m + log2f(l)) * 0.69314718055994531f;
        if (partial) p.part_lse[((size_t)pair * 2 + (seg > 0)) * kH + h] = lse;
        else p.lse[(size_t)b * kH + h] = lse;
        ptx::st_cluster_f32(stats0 + h * 4u, 1.f / l);
        ptx::fence_acq_rel_cluster();
        ptx::mbar_arrive_remote(bar(STATS_FULL), 1);
        ++seg;
      }
      // before leaving: the output CTA's last releases of the P slots and of the stats must have
      // landed in this CTA's barriers
      for (uint32_t k = (it > kPSlots ? it - kPSlots : 0); k < it; ++k)
        wait_bar(bar(P_EMPTY + k % kPSlots), (k / kPSlots) & 1u, abort_addr, true, false);
      if (seg > 0) wait_bar(bar(STATS_EMPTY), (seg - 1) & 1u, abort_addr, true, false);
    }
  } else {
    // ============================== output CTA ==============================
    if (warp == 0) {
      if (lane == 0) {   // ---- TMA producer: latent rows c of each tile
        uint32_t it = 0;
        bool ok = true;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          for (int t = t_lo; t < t_hi && ok; ++t, ++it) {
            const uint32_t s = it % kVStages;
            if (!(ok = wait_bar(bar(V_EMPTY + s), ((it / kVStages) & 1u) ^ 1u, abort_addr, false))) break;
            int page = p.block_table[(long long)b * p.max_pages + t];
            if (page < 0 || page >= p.num_pages) page = p.num_pages;   // reported by the score CTA
            const uint32_t dst = base + kOffStage + s * kVStageBytes;
            ptx::mbar_arrive_expect_tx(bar(V_FULL + s), kVStageBytes);
            for (int j = 0; j < kVChunks; ++j) ptx::tma_load_2d(dst + j * kChunkBytes, &tm_lat, 64 * j, page * kTile, bar(V_FULL + s));
          }
        }
        for (uint32_t k = (it > kVStages ? it - kVStages : 0); k < it; ++k)
          wait_bar(bar(V_FULL + k % kVStages), (k / kVStages) & 1u, abort_addr, false, false);
      }
    } else if (warp == 1) {
      if (lane == 0) {   // ---- MMA issuer: O += P · C, K = 64 positions in 4 steps, N = 512 in 2 halves
        uint32_t it = 0, seg = 0;
        bool ok = true;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          if (!(ok = wait_bar(bar(O_FREE), (seg & 1u) ^ 1u, abort_addr, false))) break;
          ++seg;
          for (int t = t_lo; t < t_hi; ++t, ++it) {
            const uint32_t slot = it % kPSlots, s = it % kVStages;
            if (!(ok = wait_bar(bar(CORR_DONE + slot), (it / kPSlots) & 1u, abort_addr, false))) break;
            if (!(ok = wait_bar(bar(V_FULL + s), (it / kVStages) & 1u, abort_addr, false))) break;
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_after();
            const uint32_t pa = base + kOffP + slot * kPSlotBytes;
            const uint32_t vs = base + kOffStage + s * kVStageBytes;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t adesc = ptx::smem_desc_sw128(pa + kk * 32, 16, 1024);
#pragma unroll
              for (int nh = 0; nh < 2; ++nh) {
                const uint64_t bdesc = ptx::smem_desc_sw128(vs + nh * 4 * kChunkBytes + kk * 2048, kChunkBytes, 1024);
                ptx::mma_ss(tmem + 256u * nh, adesc, bdesc, kIdescO, (t > t_lo || kk > 0) ? 1u : 0u);
              }
            }
            ptx::mma_commit(bar(V_EMPTY + s));
            ptx::mma_commit_mc(bar(P_EMPTY + slot), (uint16_t)0x1);
            ptx::mma_commit(bar(O_DONE + (it & 1u)));
          }
        }
      }
    } else if (warp >= 4) {
      // ---- correction + epilogue warpgroup: thread = head h = TMEM lane
      const int h = threadIdx.x - 128;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const float* alpha_s = reinterpret_cast<const float*>(gbase + kOffAlpha);
      const volatile float* stats_s = reinterpret_cast<const volatile float*>(gbase + kOffStats);
      uint32_t it = 0, seg = 0;
      bool ok = true;
      while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
        for (int t = t_lo; t < t_hi; ++t, ++it) {
          const uint32_t slot = it % kPSlots;
          if (!(ok = wait_bar_warp(bar(P_FULL + slot), (it / kPSlots) & 1u, abort_addr, true))) break;
          const float alpha = alpha_s[slot * kH + h];
          const bool need = (t > t_lo) && (alpha != 1.f);
          if (__any_sync(0xffffffffu, need)) {
            // rows whose running maximum moved: O *= alpha once the previous tile's MMAs are done
            if (!(ok = wait_bar_warp(bar(O_DONE + ((it - 1) & 1u)), ((it - 1) >> 1) & 1u, abort_addr, false))) break;
            ptx::tc_fence_after();
            const float a = need ? alpha : 1.f;
#pragma unroll 1
            for (int c = 0; c < kDC; c += 32) {
              uint32_t r[32];
              ptx::tmem_ld32(tmem + lane_off + c, r);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * a);
              ptx::tmem_st32(tmem + lane_off + c, r);
            }
            ptx::tmem_wait_st();
          }
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(CORR_DONE + slot));
        }
        if (!ok) break;
        // epilogue: O / l  ->  o_lat (bf16) or an fp32 partial
        if (!(ok = wait_bar_warp(bar(O_DONE + ((it - 1) & 1u)), ((it - 1) >> 1) & 1u, abort_addr, false))) break;
        if (!(ok = wait_bar_warp(bar(STATS_FULL), seg & 1u, abort_addr, true))) break;
        ptx::tc_fence_after();
        const float inv_l = stats_s[h];
        const bool partial = !(t_lo == 0 && t_hi == tiles_b);
        if (partial) {
          float* dst = p.part_o + (((size_t)pair * 2 + (seg > 0)) * kH + h) * kDC;
#pragma unroll 1
          for (int c = 0; c < kDC; c += 32) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_off + c, r);
            ptx::tmem_wait_ld();
            float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              d4[k] = make_float4(__uint_as_float(r[4 * k]) * inv_l, __uint_as_float(r[4 * k + 1]) * inv_l,
                                  __uint_as_float(r[4 * k + 2]) * inv_l, __uint_as_float(r[4 * k + 3]) * inv_l);
          }
        } else {
          __nv_bfloat16* dst = p.o_lat + ((size_t)b * kH + h) * kDC;
#pragma unroll 1
          for (int c = 0; c < kDC; c += 32) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_off + c, r);
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
  // heads of this block: 32 per blockIdx.y, 4 per warp; lanes cover 16 columns each
  for (int hh = 0; hh < 4; ++hh) {
    const int h = blockIdx.y * 32 + warp * 4 + hh;
    float mx = -INFINITY;
    for (int q = p0; q <= p1; ++q) {
      const long long start_q = (long long)q * T / npairs;
      if ((long long)(q + 1) * T / npairs <= start_q) continue;   // a pair with an empty range wrote nothing
      const int idx = q * 2 + (start_q < off ? 1 : 0);
      mx = fmaxf(mx, part_lse[(size_t)idx * kH + h]);
    }
    float tot = 0.f;
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    for (int q = p0; q <= p1; ++q) {
      const long long start_q = (long long)q * T / npairs;
      if ((long long)(q + 1) * T / npairs <= start_q) continue;
      const int idx = q * 2 + (start_q < off ? 1 : 0);
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

// The tensor-map encoder is a driver entry point; it is resolved at run time through the runtime
// so that the library does not link against libcuda (and loads on machines without a driver).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

inline bool make_tmap(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t stride_elems) {
  const EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)stride_elems * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kTile};
  const cuuint32_t estr[2] = {1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
  launch(decode_kernel, dim3(2 * P), dim3(kThreads), kSmemBytes, st, tm_lat, tm_rope, prm);
  launch(merge_kernel, dim3(B, kH / 32), dim3(256), 0, st, seqlens, (int)B, (int)max_pages, P, (const float*)prm.part_o,
         (const float*)prm.part_lse, prm.o_lat, lse);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla

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
//         computes S = Q̃ · [c;k_r]ᵀ for 64-position tiles into three TMEM buffers.
//   CTA 1 ("output CTA") holds O in TMEM and issues O += P · C for each tile.
// The score CTA's eight row warps turn S into bf16 P: two sets of four warps take alternate tiles, a
// thread holding a whole row of a tile, so the two warps of an SM sub-partition work on different
// tiles and their exponentials overlap the other's hand-off; each tile's P crosses to the output CTA
// as one bulk DSMEM copy. The output CTA's row warps rescale their rows of O when a running maximum
// moved (lazily: only past 2^8) and run the epilogue. No FLOP is done twice; each CTA TMA-loads the
// rows it needs (the second read hits L2).
// Work: the tiles of all sequences are laid end to end and cut into one contiguous range per
// pair; a sequence cut between pairs is written as fp32 partials and merged afterwards. When the
// batch has no more sequences than pairs and they are close in length, each pair takes one whole
// sequence instead.
// Every wait is bounded in time; on expiry the kernel records MLA_ERR_TIMEOUT and drains.
#pragma once

#include <cooperative_groups.h>
#include <cuda.h>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace sm100 {

constexpr int kH = 128, kDC = 512, kDR = 64, kRow = kDC + kDR;
constexpr int kTile = 64;                              // positions per tile = one cache page
constexpr int kChunkBytes = 64 * 128;                  // one TMA box: 64 rows x 64 bf16
constexpr int kKChunks = kRow / 64;                    // 9 chunks per tile on the score CTA
constexpr int kVChunks = kDC / 64;                     // 8 chunks per tile on the output CTA
constexpr int kGroupChunks = 3;                       // score CTA: a ring of 3-chunk groups (24 KB),
constexpr int kGroupsPerTile = kKChunks / kGroupChunks;// 3 per tile, each released as soon as its
constexpr int kRing = 8;                               // 12 MMAs are done
constexpr int kGroupBytes = kGroupChunks * kChunkBytes;// 24576
constexpr int kQGroups = 6;                            // a sequence's Q̃ travels the ring first: 18 boxes of
                                                       // 64 heads x 64 columns in 6 groups
constexpr int kVStages = 2;                            // output CTA: whole-tile stages
constexpr int kVStageBytes = kVChunks * kChunkBytes;   // 65536
constexpr int kSBufs = 3;
constexpr int kQCols = kRow / 2;                       // 288 TMEM columns hold Q̃ as bf16 pairs
constexpr int kSCol0 = kQCols;                         // S buffers at 288, 352, 416
constexpr int kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;                   // lazy rescale threshold (log2 units)
constexpr int kThreads = 384;                          // 4 control warps + 8 row warps
constexpr int kGroup = 256;                            // threads of the row warps (4-11)
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Per-tile geometry of the row warps (4..11): warp w owns rows [32 q + 16 u, +16) with q = w % 4 (its
// TMEM lane quarter, which only sub-partition q can reach) and u = (w - 4) / 4; lane t holds rows
// +t/4 and +t/4+8, columns 8j + 2 (t % 4) + {0, 1} (the tcgen05 16x256b shape). Two softmax warps per
// sub-partition: one alone is bound by its own latency, two keep the exponential unit near its rate.
constexpr int kPBytes = kH * kTile * 2;                // 16384: a P tile, bf16, K-major 128-byte swizzle
// Rescale factors alpha: per row, 1 unless the row's running maximum moved at this tile.
// staging buffer (score CTA) and P slot (output CTA) alike: P [128 rows] | alpha [128]
constexpr int kAlphaOff = kPBytes;
constexpr int kCopyBytes = kPBytes + kH * 4;           // 16896: one bulk copy per tile
constexpr int kStgStride = kCopyBytes;
constexpr int kSlotStride = 17408;                     // a multiple of 1024 (the swizzle repeat)
constexpr int kPSlots = 4;                             // P tiles in flight on the output CTA
constexpr int kStaging = 2;                            // P tiles assembled on the score CTA
static_assert(kCopyBytes <= kSlotStride && kSlotStride % 1024 == 0 && kCopyBytes % 16 == 0, "P slot layout");

// shared memory map (offsets from a 1024-byte aligned base)
//   score CTA:  K group ring [8] | staging [2]
//   output CTA: V stages [2] | P slots [4] | epilogue transpose buffers [8 x 2 KB]
//   both:       1/l per row (two segments) | barriers | TMEM address | abort flag | work range
constexpr int kOffK = 0;
constexpr int kOffStaging = kRing * kGroupBytes;                       // 196608
constexpr int kRegion0 = kOffStaging + kStaging * kStgStride;         // 230400
constexpr int kOffV = 0;
constexpr int kOffPSlots = kVStages * kVStageBytes;                    // 131072
constexpr int kOffEpi = kOffPSlots + kPSlots * kSlotStride;           // 200704
constexpr int kEpiWarpBytes = 2048;
constexpr int kRegion1 = kOffEpi + 8 * kEpiWarpBytes;                 // 217088
constexpr int kRegion = kRegion0 > kRegion1 ? kRegion0 : kRegion1;
// float [128] per row. Output CTA: 1/l (one buffer is enough: the score CTA writes a segment's values
// only after the output CTA released the previous segment's, STATS_EMPTY). Score CTA: the running
// maximum after the latest tile, handed from one softmax set to the other; at a segment end, set 1's
// partial row sums.
constexpr int kOffStats = kRegion;
constexpr int kOffBar = kOffStats + kH * 4;
// Barriers. Score CTA: K_*, S_*, Q_FULL, P_EMPTY, P_WRITTEN, STG_FREE, STATS_EMPTY. Output CTA:
// V_*, P_FULL, P_LOCAL, P_EMPTY, STATS_FULL. P_EMPTY[slot] completes in both CTAs when the O MMAs
// of the slot's tile are done (one multicast commit). Arrivals from the other CTA reach P_EMPTY,
// STG_FREE, STATS_EMPTY (score CTA) and P_FULL, STATS_FULL (output CTA).
enum Bar : int {
  K_FULL = 0, K_EMPTY = K_FULL + kRing, S_FULL = K_EMPTY + kRing, S_EMPTY = S_FULL + kSBufs,
  Q_FULL = S_EMPTY + kSBufs, P_EMPTY = Q_FULL + 1, P_WRITTEN = P_EMPTY + kPSlots,
  STG_FREE = P_WRITTEN + kStaging, STATS_EMPTY = STG_FREE + kStaging,
  DEC_FULL = STATS_EMPTY + 1, V_FULL = DEC_FULL + 1, V_EMPTY = V_FULL + kVStages, P_FULL = V_EMPTY + kVStages,
  P_LOCAL = P_FULL + kPSlots, STATS_FULL = P_LOCAL + kPSlots, NUM_BARS = STATS_FULL + 1
};
constexpr int kOffTmemSlot = kOffBar + NUM_BARS * 8;
constexpr int kOffAbort = kOffTmemSlot + 8;
constexpr int kOffWork = kOffAbort + 8;                // long long start, end, off_b, b, total tiles, whole
constexpr int kSmemUsed = kOffWork + 48;
constexpr int kSmemBytes = kSmemUsed + 1024;           // + alignment slack of the dynamic base
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert((kOffBar % 8) == 0 && (kOffWork % 8) == 0 && (kOffEpi % 1024) == 0 && (kOffStaging % 16) == 0, "alignment");

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 64, false);   // S = Q̃ · Kᵀ   (K-major B)
constexpr uint32_t kIdescO = ptx::idesc_bf16_f32(128, 256, true);   // O += P · C   (MN-major B)

struct Params {
  const __nv_bfloat16* q_abs;  // [B, s_q, 128, 576]
  const int32_t* block_table;
  int max_pages;
  int num_pages;
  const int32_t* seqlens;
  int B;
  int s_q;                     // new tokens per sequence (the pairs form groups of s_q, one token each)
  int max_tiles;               // max_pages: a sequence never reads past its table row
  __nv_bfloat16* o_lat;        // [B, s_q, 128, 512]
  float* lse;                  // [B, s_q, 128]
  float* part_o;               // [2 * pairs, 128, 512]
  float* part_lse;             // [2 * pairs, 128]
  float sm_scale_log2;         // sm_scale * log2(e)
  // 1: launched cooperatively; the kernel then merges cut sequences itself after a grid-wide barrier
  // (taken only when something was cut) and no merge kernel follows
  int merge_in_kernel;
  // 1: launched without any merge because the host's copy of seqlens cut no sequence; a cut found
  // here from the device's seqlens is then reported (its parts would stay unmerged)
  int expect_whole;
};

// ---- work split -----------------------------------------------------------------------------------
__host__ __device__ __forceinline__ int tiles_of(int L, int max_tiles) { return L > 0 ? min((L + kTile - 1) / kTile, max_tiles) : 0; }

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

// The work split. The pairs form G = P / s_q groups of s_q pairs; pair p is token p % s_q of group
// p / s_q, and the s_q pairs of a group walk the same tiles together (each page is read from DRAM
// once and from L2 by the group's other pairs). Default: the tiles of all sequences laid end to end
// and cut into one contiguous range per group (balanced to a tile), group g taking [g*T/G, (g+1)*T/G).
// A sequence cut between groups costs its pairs a segment switch, fp32 partials and the merge; so
// when there are no more sequences than groups and the longest is within kSplitSlack tiles of the
// balanced share, each group takes one whole sequence instead (group g takes sequence g; nothing is
// cut). Both the decode and the merge kernel decide it the same way from seqlens.
constexpr int kSplitSlack = 12;
__host__ __device__ __forceinline__ bool whole_sequences(int B, int npairs, long long T, int max_tb) {
  return B <= npairs && (long long)max_tb <= (T + npairs - 1) / npairs + kSplitSlack;
}

// One warp: total tiles T, this pair's range, and the sequence holding its first tile. Lane l scans
// sequences [l*per, (l+1)*per).
__device__ void plan_range(const int32_t* seqlens, int B, int s_q, int max_tiles, int pair, int npairs, long long* out) {
  const int lane = threadIdx.x & 31;
  const int per = (B + 31) / 32;
  const int b0 = min(B, lane * per), b1 = min(B, b0 + per);
  long long local = 0;
  int max_tb = 0;
  for (int b = b0; b < b1; ++b) {
    const int L = seqlens[b];
    if (L < s_q || (L + kTile - 1) / kTile > max_tiles) report(MLA_ERR_DEVICE_CHECK);
    const int tb = tiles_of(L, max_tiles);
    local += tb;
    max_tb = max(max_tb, tb);
  }
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
    max_tb = max(max_tb, __shfl_xor_sync(0xffffffffu, max_tb, o));
  }
  const long long T = __shfl_sync(0xffffffffu, incl, 31);
  const long long excl = incl - local;
  const int G = npairs / s_q, grp = pair / s_q;
  if (lane == 0) { out[4] = T; out[5] = (G > 0 && whole_sequences(B, G, T, max_tb)) ? 1 : 0; }
  if (grp >= G) {   // left over when s_q does not divide the pairs: no work
    if (lane == 0) { out[0] = 0; out[1] = 0; out[2] = 0; out[3] = B; }
    return;
  }
  if (whole_sequences(B, G, T, max_tb)) {
    // group g: sequence g whole
    if (grp >= B) {
      if (lane == 0) { out[0] = 0; out[1] = 0; out[2] = 0; out[3] = B; }
    } else if (grp >= b0 && grp < b1) {
      long long off = excl;
      for (int b = b0; b < grp; ++b) off += tiles_of(seqlens[b], max_tiles);
      out[0] = off; out[1] = off + tiles_of(seqlens[grp], max_tiles); out[2] = off; out[3] = grp;
    }
    return;
  }
  const long long start = (long long)grp * T / G;
  const long long end = (long long)(grp + 1) * T / G;
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

// ---- merge of split sequences ------------------------------------------------------------------------
// group g covers global tiles [g*T/G, (g+1)*T/G); the group holding tile x is floor(((x+1)*G - 1) / T).
__device__ __forceinline__ int pair_of(long long x, long long T, int P) { return (int)(((x + 1) * P - 1) / T); }

// One warp combines the parts of new token v (= b * s_q + tok) and head h, if its sequence was cut:
// the parts come from pair (group, tok) of the groups that covered the sequence's tiles. T = total
// tiles, G = groups; lane l holds sequences [b0, b1) for the prefix of tiles before b.
__device__ __forceinline__ void merge_token_head(const int32_t* __restrict__ seqlens, int s_q, int max_tiles, int G,
                                                 long long T, int b0, int b1, int v, int h,
                                                 const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                                 __nv_bfloat16* __restrict__ o_lat, float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int b = v / s_q, tok = v % s_q;
  long long before = 0;
  for (int x = b0; x < min(b1, b); ++x) before += tiles_of(__ldg(seqlens + x), max_tiles);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  const long long off = before, tb = tiles_of(__ldg(seqlens + b), max_tiles);
  if (tb == 0) return;
  const int p0 = pair_of(off, T, G), p1 = pair_of(off + tb - 1, T, G);   // groups
  if (p0 == p1) return;                       // written whole by one group
  // a group with an empty range wrote nothing; the others' parts in order, lane q holds group p0 + q's lse
  auto slot = [&](int q) -> int {
    const long long start_q = (long long)q * T / G;
    if ((long long)(q + 1) * T / G <= start_q) return -1;
    return (q * s_q + tok) * 2 + (start_q < off ? 1 : 0);
  };
  float mx = -INFINITY;
  for (int q0 = p0; q0 <= p1; q0 += 32) {
    const int q = q0 + lane;
    const int idx = q <= p1 ? slot(q) : -1;
    mx = fmaxf(mx, warp_max(idx >= 0 ? part_lse[(size_t)idx * kH + h] : -INFINITY));
  }
  float tot = 0.f;
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
  // lane covers columns [4 lane + 128 k, +4) for k < 4: every load instruction reads 512 contiguous bytes
  for (int q = p0; q <= p1; q += 2) {
    const int i0 = slot(q), i1 = q + 1 <= p1 ? slot(q + 1) : -1;
    float4 x0[4], x1[4];
    const float w0 = i0 >= 0 ? exp2f((part_lse[(size_t)i0 * kH + h] - mx) * 1.4426950408889634f) : 0.f;
    const float w1 = i1 >= 0 ? exp2f((part_lse[(size_t)i1 * kH + h] - mx) * 1.4426950408889634f) : 0.f;
    const float4* s0 = reinterpret_cast<const float4*>(part_o + ((size_t)max(i0, 0) * kH + h) * kDC) + lane;
    const float4* s1 = reinterpret_cast<const float4*>(part_o + ((size_t)max(i1, 0) * kH + h) * kDC) + lane;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x0[k] = i0 >= 0 ? s0[32 * k] : make_float4(0.f, 0.f, 0.f, 0.f);
      x1[k] = i1 >= 0 ? s1[32 * k] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tot += w0 + w1;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[4 * k] += w0 * x0[k].x + w1 * x1[k].x;
      acc[4 * k + 1] += w0 * x0[k].y + w1 * x1[k].y;
      acc[4 * k + 2] += w0 * x0[k].z + w1 * x1[k].z;
      acc[4 * k + 3] += w0 * x0[k].w + w1 * x1[k].w;
    }
  }
  const float inv = 1.f / tot;
  uint2* dst = reinterpret_cast<uint2*>(o_lat + ((size_t)v * kH + h) * kDC) + lane;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    dst[32 * k] = make_uint2(ptx::pack_bf16x2(acc[4 * k] * inv, acc[4 * k + 1] * inv),
                             ptx::pack_bf16x2(acc[4 * k + 2] * inv, acc[4 * k + 3] * inv));
  if (lane == 0) lse[(size_t)v * kH + h] = mx + logf(tot);
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
// Warp roles.  Score CTA: 0 TMA producer | 1 S-MMA issuer for even tiles, warp 2 for odd tiles (each
// warp waits as a whole and one elected lane issues) | 2 TMEM | 3 copier (one bulk
// copy per tile into the output CTA) | 4-11 row warps: softmax of their 16 rows each; all of them
// copy Q̃ into TMEM at a segment start.
// Output CTA: 0 TMA producer | 1 O-MMA issuer | 2 TMEM, then receiver (returns the score CTA's
// staging buffers as tiles land) | 4-11 row warps: rescale of their own rows of O when a running
// maximum moved, and the epilogue.
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
    for (int i = 0; i < kSBufs; ++i) { ptx::mbar_init(bar(S_FULL + i), 1); ptx::mbar_init(bar(S_EMPTY + i), kH); }
    ptx::mbar_init(bar(Q_FULL), kGroup);
    for (int i = 0; i < kPSlots; ++i) {
      ptx::mbar_init(bar(P_EMPTY + i), 1);
      ptx::mbar_init(bar(P_FULL + i), 1);
      ptx::mbar_init(bar(P_LOCAL + i), kGroup);
    }
    for (int i = 0; i < kStaging; ++i) { ptx::mbar_init(bar(P_WRITTEN + i), kH); ptx::mbar_init(bar(STG_FREE + i), 1); }
    ptx::mbar_init(bar(DEC_FULL), kH);   // one set's 128 row threads, once per tile
    ptx::mbar_init(bar(STATS_EMPTY), kGroup);
    for (int i = 0; i < kVStages; ++i) { ptx::mbar_init(bar(V_FULL + i), 1); ptx::mbar_init(bar(V_EMPTY + i), 1); }
    ptx::mbar_init(bar(STATS_FULL), kH);   // one arrival per row (set 0 of the score CTA)
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
  // nothing above touched global memory; from here on the previous kernel's results are needed
  grid_dependency_wait();
  if (warp == 3) plan_range(p.seqlens, p.B, p.s_q, p.max_tiles, pair, npairs, work);
  ptx::tc_fence_before();
  __syncthreads();
  // (allow_dependents() only at the end: the merge that follows would park its blocks on these SMs)
  ptx::cluster_sync();      // the peer's barriers are initialised before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + kOffTmemSlot);
  SegIter segs{work[0], work[1], work[2], (int)work[3]};
  int b, t_lo, t_hi, tiles_b;
  // row-warp geometry (warps 4-11)
  const int qd = warp & 3, sub = (warp - 4) >> 2;
  const int r0 = 32 * qd + 16 * sub + (lane >> 2);                       // and r0 + 8
  const uint32_t s_lane = (uint32_t)(32 * qd + 16 * sub) << 16;          // TMEM lane field of the warp
  const float scale2 = p.sm_scale_log2;
  // this pair's new token: row block v = b * s_q + tok of the queries and outputs; it sees the
  // first seqlens[b] - s_q + 1 + tok positions of its sequence
  const int tok = pair % p.s_q;
  auto vrow = [&](int bb) -> long long { return (long long)bb * p.s_q + tok; };
  auto vlen = [&](int bb) -> int { return p.seqlens[bb] - (p.s_q - 1 - tok); };

  if (rank == 0) {
    // ============================== score CTA ==============================
    if (warp == 0) {
      if (lane == 0) {   // ---- TMA producer: [c (8 chunks) ; k_r (1 chunk)] of each tile
        uint32_t it = 0;
        bool ok = true;
        uint32_t gi = 0;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          // the sequence's absorbed query first: box (column block cb, head half rh)
          for (int qg = 0; qg < kQGroups && ok; ++qg, ++gi) {
            const uint32_t s = gi % kRing;
            if (!(ok = wait_bar(bar(K_EMPTY + s), ((gi / kRing) & 1u) ^ 1u, abort_addr, false))) break;
            ptx::mbar_arrive_expect_tx(bar(K_FULL + s), kGroupBytes);
            for (int j = 0; j < kGroupChunks; ++j) {
              const int qc = qg * kGroupChunks + j;
              ptx::tma_load_2d(base + kOffK + s * kGroupBytes + j * kChunkBytes, &tm_q, 64 * (qc >> 1), (int)vrow(b) * kH + 64 * (qc & 1), bar(K_FULL + s));
            }
          }
          for (int t = t_lo; t < t_hi && ok; ++t, ++it) {
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
      if (lane == 0) {   // ---- copier: each finished staging buffer goes to the output CTA's slot
        const uint32_t slot_remote0 = ptx::map_to_cta(base + kOffPSlots, 1);
        uint32_t it = 0;
        bool ok = true;
        while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
          for (int t = t_lo; t < t_hi; ++t, ++it) {
            const uint32_t stg = it % kStaging, slot = it % kPSlots;
            if (!(ok = wait_bar(bar(P_WRITTEN + stg), (it / kStaging) & 1u, abort_addr, false))) break;
            // the slot is free once the output CTA's MMAs of tile it - kPSlots are done
            if (!(ok = wait_bar(bar(P_EMPTY + slot), ((it / kPSlots) & 1u) ^ 1u, abort_addr, true))) break;
            const uint32_t full = ptx::map_to_cta(bar(P_FULL + slot), 1);
            const uint32_t src = base + kOffStaging + stg * kStgStride, dst = slot_remote0 + slot * kSlotStride;
            ptx::mbar_arrive_expect_tx_remote(bar(P_FULL + slot), 1, kCopyBytes);
            ptx::bulk_copy_to_cta(dst, src, kCopyBytes, full);
          }
        }
        // before leaving: every copy has landed and every slot came back
        for (uint32_t k = (it > (uint32_t)kPSlots ? it - kPSlots : 0); k < it; ++k)
          wait_bar(bar(P_EMPTY + k % kPSlots), (k / kPSlots) & 1u, abort_addr, true, false);
        for (uint32_t k = (it > (uint32_t)kStaging ? it - kStaging : 0); k < it; ++k)
          wait_bar(bar(STG_FREE + k % kStaging), (k / kStaging) & 1u, abort_addr, true, false);
      }
    } else if (warp == 1 || warp == 2) {
      // ---- S-MMA issuers: S = Q̃ · [c ; k_r]ᵀ, K = 576 in 36 steps of 16. The whole warp runs the
      // loop and waits; one elected lane issues each group's 12 MMAs and their commits.
      const uint32_t parity = warp == 1 ? 0u : 1u;
      const uint64_t k_desc = ptx::smem_desc_sw128(base + kOffK, 16, 1024);
      uint32_t it = 0, seg = 0, gq = 0;
      bool ok = true;
      while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
        if (!(ok = wait_bar_warp(bar(Q_FULL), seg & 1u, abort_addr, false))) break;
        if (parity == 0 && lane == 0)   // every row-warp thread has copied its part of the query out of the ring
          for (int qg = 0; qg < kQGroups; ++qg) ptx::mbar_arrive(bar(K_EMPTY + (gq + qg) % kRing));
        __syncwarp();
        ++seg;
        gq += kQGroups;
        for (int t = t_lo; t < t_hi && ok; ++t, ++it, gq += kGroupsPerTile) {
          if ((it & 1u) != parity) continue;
          const uint32_t sb = it % kSBufs;
          const uint32_t g0 = gq;
          if (!(ok = wait_bar_warp(bar(S_EMPTY + sb), ((it / kSBufs) & 1u) ^ 1u, abort_addr, false))) break;
          const uint32_t d = tmem + kSCol0 + 64u * sb;
#pragma unroll
          for (int q = 0; q < kGroupsPerTile; ++q) {
            const uint32_t gi = g0 + q, s = gi % kRing;
            if (!(ok = wait_bar_warp(bar(K_FULL + s), (gi / kRing) & 1u, abort_addr, false))) break;
            if (ptx::elect_one()) {
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
              if (q == kGroupsPerTile - 1) ptx::mma_commit(bar(S_FULL + sb));
            }
            __syncwarp();
          }
        }
      }
    } else if (warp >= 4) {
      // ---- row warps: two sets of four warps take alternate tiles (set = it % 2); in a set, thread =
      // one head row of its warp's TMEM lane quarter, the whole 64-position row of S in registers
      // (32x32b loads), so a row's maximum and sum need no shuffle. The lazy running maximum m of a
      // row moves only when a tile's maximum exceeds it by 2^kRescaleLog2; each tile's decision (m
      // after the tile) is published for the next tile, which the other set processes. Each set keeps
      // its own partial row sums, combined at the segment end.
      const int set = (warp - 4) >> 2;                    // also the Q̃ column half this warp copies
      const int row = ((warp & 3) << 5) | lane;           // head = TMEM lane
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t stats_remote = ptx::map_to_cta(base + kOffStats, 1);
      float* dec = reinterpret_cast<float*>(gbase + kOffStats);   // [128]: m after the latest tile
      uint32_t it = 0, seg = 0, gq = 0;
      bool ok = true;
      while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
        const int L = vlen(b);
        // Q̃ of this sequence into TMEM columns [0, 288), from the 6 ring groups that carry it (every
        // S MMA of the previous segment is done: the row warps met after its last result). Set g
        // fills column blocks [5g, 5 + 4g) of 64 values (32 TMEM columns).
        {
          bool qok = true;
          for (int qg = 0; qg < kQGroups; ++qg)
            qok = qok && wait_bar_warp(bar(K_FULL + (gq + qg) % kRing), ((gq + qg) / kRing) & 1u, abort_addr, false);
          ok = ok && qok;   // after a failure every row warp still meets the others at the segment end
          const int r = row & 63, rh = row >> 6;
#pragma unroll 1
          for (int cb = set ? 5 : 0; cb < (set ? 9 : 5) && ok; ++cb) {
            const int qc = 2 * cb + rh, qg = qc / kGroupChunks, j = qc % kGroupChunks;
            const uint32_t srow = base + kOffK + ((gq + qg) % kRing) * kGroupBytes + j * kChunkBytes + r * 128;
            uint32_t v[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint4 x = ptx::ld_shared_v4(srow + ((uint32_t)(k ^ (r & 7)) << 4));
              v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
            }
            ptx::tmem_st32(tmem + lane_off + 32u * cb, v);
          }
          ptx::tmem_wait_st();
          // Q_FULL completes once every thread has stored its part in TMEM; the S-MMA issuer of even
          // tiles then hands the query groups back to the producer
          gq += kQGroups;
          ptx::tc_fence_before();
          if (ok) ptx::mbar_arrive(bar(Q_FULL));
        }
        int nb = -1;
        {
          SegIter peek = segs;
          int x0, x1, x2;
          if (!peek.next(p.seqlens, p.B, p.max_tiles, nb, x0, x1, x2)) nb = -1;
        }
        gq += kGroupsPerTile * (t_hi - t_lo);
        float m_own = -INFINITY, l_own = 0.f;   // this set's running maximum and partial row sum
        for (int t = t_lo; t < t_hi; ++t, ++it) {
          if ((it & 1u) != (uint32_t)set || !ok) continue;   // the other set's tile (or give up: meet below)
          const uint32_t sb = it % kSBufs, stg = it % kStaging;
          if (nb >= 0 && t == max(t_lo, t_hi - 3)) {   // the next segment's query row into L2
            const char* nq = reinterpret_cast<const char*>(p.q_abs + ((size_t)vrow(nb) * kH + row) * kRow);
            for (int k = set ? 5 : 0; k < (set ? 9 : 5); ++k) ptx::prefetch_l2(nq + 128 * k);
          }
          // probe this tile's staging buffer now; the answer is used after the arithmetic
          const bool stg_free = ptx::mbar_test_wait_cluster(bar(STG_FREE + stg), ((it / kStaging) & 1u) ^ 1u);
          if (!wait_bar_warp(bar(S_FULL + sb), (it / kSBufs) & 1u, abort_addr, false)) { ok = false; continue; }
          uint32_t v[64];
          {
            uint32_t (&v0)[32] = *reinterpret_cast<uint32_t(*)[32]>(v);
            uint32_t (&v1)[32] = *reinterpret_cast<uint32_t(*)[32]>(v + 32);
            ptx::tc_fence_after();
            ptx::tmem_ld32(tmem + lane_off + kSCol0 + 64u * sb, v0);
            ptx::tmem_ld32(tmem + lane_off + kSCol0 + 64u * sb + 32u, v1);
            ptx::tmem_wait_ld_regs(v0);
            ptx::tmem_wait_ld_regs(v1);
          }
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(S_EMPTY + sb));
          const int valid = L - t * kTile;
          // the tile's maximum over its visible positions
          float a4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (valid >= kTile || j < valid) a4[j & 3] = fmaxf(a4[j & 3], __uint_as_float(v[j]));
          const float mt = fmaxf(fmaxf(a4[0], a4[1]), fmaxf(a4[2], a4[3])) * scale2;
          // m after the previous tile (the other set's decision), then this tile's
          float m_prev = -INFINITY;
          if (t > t_lo) {   // phase it - 1 of DEC_FULL: the previous tile's decision (one slot: each
                            // tile's set reads its predecessor's value before writing its own)
            if (!wait_bar_warp(bar(DEC_FULL), (it - 1) & 1u, abort_addr, true)) { ok = false; continue; }
            m_prev = dec[row];
          }
          float al = 1.f, m_new = m_prev;
          if (mt > m_prev + kRescaleLog2) {
            al = (m_prev == -INFINITY) ? 0.f : ptx::ex2_approx(m_prev - mt);
            m_new = mt;
          }
          dec[row] = m_new;
          ptx::mbar_arrive(bar(DEC_FULL));
          if (m_new != m_own) {   // this set's partial sum to the new maximum
            l_own = (m_own == -INFINITY) ? 0.f : l_own * ptx::ex2_approx(m_own - m_new);
            m_own = m_new;
          }
          // exponentials, their sum, bf16 pairs
          uint32_t pk[32];
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            const bool in0 = valid >= kTile || j < valid, in1 = valid >= kTile || j + 1 < valid;
            const float x0 = fmaf(__uint_as_float(v[j]), scale2, -m_new);
            const float x1 = fmaf(__uint_as_float(v[j + 1]), scale2, -m_new);
            const float e0 = in0 ? ptx::ex2_approx(x0) : 0.f;
            const float e1 = in1 ? ptx::ex2_approx(x1) : 0.f;
            ls[(j >> 1) & 3] += e0 + e1;
            pk[j >> 1] = ptx::pack_bf16x2(e0, e1);
          }
          l_own += (ls[0] + ls[1]) + (ls[2] + ls[3]);
          // this tile's staging buffer must have been copied out (this set's tile two before)
          if (!__all_sync(0xffffffffu, stg_free) &&
              !wait_bar_warp(bar(STG_FREE + stg), ((it / kStaging) & 1u) ^ 1u, abort_addr, true)) {
            ok = false;
            continue;
          }
          // P row into the K-major, 128-byte swizzled tile (row r at (r / 8) * 1024 + (r % 8) * 128,
          // 16-byte chunk c at (c ^ (r % 8)) * 16), and its rescale factor
          const uint32_t st0 = base + kOffStaging + stg * kStgStride;
          const uint32_t prow = st0 + (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            ptx::st_shared_v4(prow + (((uint32_t)c ^ (uint32_t)(row & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                              pk[4 * c + 3]);
          reinterpret_cast<float*>(gbase + kOffStaging + stg * kStgStride + kAlphaOff)[row] = al;
          // visible to the bulk copy (async proxy), then handed to the copier
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(bar(P_WRITTEN + stg));
        }
        // segment end: the two sets' partial sums combined at the maximum after the segment's last
        // tile (the set that did not process that tile reads its decision), set 1's sums handed to set
        // 0 through the same slot. All row warps meet here (and agree whether to go on); after it,
        // every S MMA of the segment is known to be done.
        float m_fin = -INFINITY;
        if (ok && t_hi > t_lo) {
          const uint32_t last = it - 1;
          if ((last & 1u) == (uint32_t)set) m_fin = m_own;
          else if (wait_bar_warp(bar(DEC_FULL), last & 1u, abort_addr, true)) m_fin = dec[row];
          else ok = false;
        }
        const float l_fin = (m_own == -INFINITY) ? 0.f : l_own * ptx::ex2_approx(m_own - m_fin);
        if (ptx::named_bar_or(2, kGroup, !ok)) { ok = false; break; }
        if (set == 1) dec[row] = l_fin;
        ptx::named_bar_sync(2, kGroup);
        if (set == 0) {
          const float l = l_fin + dec[row];
          if (!wait_bar_warp(bar(STATS_EMPTY), (seg & 1u) ^ 1u, abort_addr, true)) ok = false;
          if (ok) {
            const bool partial = !(t_lo == 0 && t_hi == tiles_b);
            float* lse_dst = partial ? p.part_lse + ((size_t)pair * 2 + (seg > 0)) * kH : p.lse + (size_t)vrow(b) * kH;
            // a segment with no visible position (a token's masked last tile alone) has l = 0:
            // lse -inf and a zero part, which the merge weighs by 0
            lse_dst[row] = (m_fin + log2f(l)) * 0.69314718055994531f;
            ptx::st_cluster_f32(stats_remote + row * 4u, l > 0.f ? 1.f / l : 0.f);
            ptx::mbar_arrive_remote(bar(STATS_FULL), 1);
          }
        }
        ++seg;
      }
      // before leaving: the output CTA's last release of the stats must have landed here
      if (set == 0 && seg > 0) wait_bar(bar(STATS_EMPTY), (seg - 1) & 1u, abort_addr, true, false);
    }
  } else {
    // ============================== output CTA ==============================
    if (warp == 2) {
      if (lane == 0) {   // ---- receiver: as each tile lands, the score CTA may reuse that staging buffer
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
      // ---- MMA issuer (an elected lane) with the warp's help for masking: O += P · C, K = 64 positions in
      // 4 steps of 16, N = 512 in 2 halves. A tile's P is complete (and O rescaled for it) once the
      // row warps arrived on P_LOCAL.
      const uint64_t v_desc0 = ptx::smem_desc_sw128(base + kOffV, kChunkBytes, 1024);
      const uint64_t p_desc0 = ptx::smem_desc_sw128(base + kOffPSlots, 16, 1024);
      uint32_t it = 0;
      bool ok = true;
      while (ok && segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
        const int L = vlen(b);
        for (int t = t_lo; t < t_hi; ++t, ++it) {
          const uint32_t slot = it % kPSlots, s = it % kVStages;
          if (!(ok = wait_bar_warp(bar(P_LOCAL + slot), (it / kPSlots) & 1u, abort_addr, false))) break;
          if (!(ok = wait_bar_warp(bar(V_FULL + s), (it / kVStages) & 1u, abort_addr, false))) break;
          // a tile past the token's last visible position (the last page of a sequence, or with
          // several new tokens the one before it): skip whole 16-row steps past the end and zero the
          // rows of the last step that lie past it (a pool row there may hold anything, and
          // 0 * NaN = NaN). At least one step runs, so that a segment's first tile always sets O.
          int nk = kTile / 16;
          if (L - t * kTile < kTile) {
            const int valid = max(0, L - t * kTile);
            nk = max(1, (valid + 15) / 16);
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
          if (ptx::elect_one()) {
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_after();
            const uint64_t pd = p_desc0 + (uint64_t)(slot * (kSlotStride >> 4));
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
            ptx::mma_commit_mc(bar(P_EMPTY + slot), (uint16_t)0x3);
          }
          __syncwarp();
        }
      }
    } else if (warp >= 4) {
      // ---- row warps: rescale of the warp's own 16 rows of O before a tile whose P was computed
      // against a larger maximum, and the segment epilogue
      const int g = (warp - 4) >> 2;                      // epilogue: head h, latent half g
      const int h = ((warp & 3) << 5) | lane;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t col0 = 256u * g;
      float* stats = reinterpret_cast<float*>(gbase + kOffStats);
      uint32_t it = 0, seg = 0;
      bool ok = true;
      while (segs.next(p.seqlens, p.B, p.max_tiles, b, t_lo, t_hi, tiles_b)) {
        for (int t = t_lo; t < t_hi; ++t, ++it) {
          if (!ok) continue;   // after a failure: skip to the segment end, where all row warps meet
          const uint32_t slot = it % kPSlots;
          if (!wait_bar_warp(bar(P_FULL + slot), (it / kPSlots) & 1u, abort_addr, true)) { ok = false; continue; }
          const float* alpha_s = reinterpret_cast<const float*>(gbase + kOffPSlots + slot * kSlotStride + kAlphaOff);
          const float al0 = alpha_s[r0], al1 = alpha_s[r0 + 8];
          // O rows of this warp computed against an older maximum: scale them once the MMAs of the
          // previous tile are done (16x256b: rows r0, r0 + 8, 8 columns per 256-bit chunk). The slot's
          // phase before that one (tile it - 1 - kPSlots) completed before tile it - 1's P_FULL, so the
          // parity test cannot mistake it.
          if (t > t_lo && __any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
            const uint32_t pt = it - 1;
            if (!wait_bar_warp(bar(P_EMPTY + pt % kPSlots), (pt / kPSlots) & 1u, abort_addr, false)) { ok = false; continue; }
            ptx::tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < kDC; c += 64) {
              uint32_t r[32];
              ptx::tmem_ld_16x256b_x8(tmem + s_lane + c, r);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                r[4 * j] = __float_as_uint(__uint_as_float(r[4 * j]) * al0);
                r[4 * j + 1] = __float_as_uint(__uint_as_float(r[4 * j + 1]) * al0);
                r[4 * j + 2] = __float_as_uint(__uint_as_float(r[4 * j + 2]) * al1);
                r[4 * j + 3] = __float_as_uint(__uint_as_float(r[4 * j + 3]) * al1);
              }
              ptx::tmem_st_16x256b_x8(tmem + s_lane + c, r);
            }
            ptx::tmem_wait_st();
          }
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(P_LOCAL + slot));
        }
        // segment end: O / l out, 1/l from the score CTA
        if (ok && !wait_bar_warp(bar(P_EMPTY + (it - 1) % kPSlots), ((it - 1) / kPSlots) & 1u, abort_addr, false)) ok = false;
        if (ok && !wait_bar_warp(bar(STATS_FULL), seg & 1u, abort_addr, true)) ok = false;
        // every row warp meets here once per segment and agrees whether to go on
        if (ptx::named_bar_or(1, kGroup, !ok)) break;
        ptx::tc_fence_after();
        const float inv_l = stats[h];
        const bool partial = !(t_lo == 0 && t_hi == tiles_b);
        // 32 columns of the warp's 32 rows at a time: each thread (row) scales its values and puts
        // them in the warp's buffer as one 64-byte row (16-byte chunks XOR-swizzled by row / 2, so
        // both phases are free of bank conflicts); read back as (row 8i + lane / 4, chunk lane % 4),
        // every 16-byte store instruction writes eight 64-byte row pieces.
        const uint32_t ebuf = base + kOffEpi + (uint32_t)(warp - 4) * kEpiWarpBytes;
        const uint32_t wrow = ebuf + (uint32_t)lane * 64u;
        const uint32_t sw = (uint32_t)(lane >> 1) & 3u;
        const int c4 = lane & 3, rsub = lane >> 2;
        const int row0 = (warp & 3) * 32;
        auto flush = [&](char* dst0, size_t row_bytes) {   // the buffer's 32 rows to dst0 + row * row_bytes
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int rr = 8 * i + rsub;
            const uint4 v = ptx::ld_shared_v4(ebuf + rr * 64u + (((uint32_t)c4 ^ (((uint32_t)rr >> 1) & 3u)) << 4));
            *reinterpret_cast<uint4*>(dst0 + (size_t)(row0 + rr) * row_bytes + c4 * 16) = v;
          }
          __syncwarp();
        };
#pragma unroll 1
        for (int c = 0; c < kDC / 2; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld32(tmem + lane_off + col0 + c, r);
          ptx::tmem_wait_ld();
          if (partial) {
            float* dst = p.part_o + ((size_t)pair * 2 + (seg > 0)) * kH * kDC + col0 + c;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int j = 16 * half + 4 * k;
                ptx::st_shared_v4(wrow + ((k ^ sw) << 4), __float_as_uint(__uint_as_float(r[j]) * inv_l),
                                  __float_as_uint(__uint_as_float(r[j + 1]) * inv_l),
                                  __float_as_uint(__uint_as_float(r[j + 2]) * inv_l),
                                  __float_as_uint(__uint_as_float(r[j + 3]) * inv_l));
              }
              flush(reinterpret_cast<char*>(dst + 16 * half), kDC * sizeof(float));
            }
          } else {
            __nv_bfloat16* dst = p.o_lat + (size_t)vrow(b) * kH * kDC + col0 + c;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int j = 8 * k;
              ptx::st_shared_v4(wrow + ((k ^ sw) << 4),
                                ptx::pack_bf16x2(__uint_as_float(r[j]) * inv_l, __uint_as_float(r[j + 1]) * inv_l),
                                ptx::pack_bf16x2(__uint_as_float(r[j + 2]) * inv_l, __uint_as_float(r[j + 3]) * inv_l),
                                ptx::pack_bf16x2(__uint_as_float(r[j + 4]) * inv_l, __uint_as_float(r[j + 5]) * inv_l),
                                ptx::pack_bf16x2(__uint_as_float(r[j + 6]) * inv_l, __uint_as_float(r[j + 7]) * inv_l));
            }
            flush(reinterpret_cast<char*>(dst), kDC * sizeof(__nv_bfloat16));
          }
        }
        // O may be overwritten by the next segment's first MMA once every row warp arrived on its
        // P_LOCAL (after this point, in program order); the score CTA may write the next 1/l values
        ptx::tc_fence_before();
        ptx::mbar_arrive_remote(bar(STATS_EMPTY), 0);
        ++seg;
      }
    }
  }

  // teardown: TMEM back, then leave together so no remote access can target an exited CTA. The
  // merge kernel that follows (when there is one) may be scheduled from here on (it waits for this
  // grid's completion and its writes before reading anything), so its launch overlaps the last
  // CTAs' exit.
  ptx::tc_fence_before();
  __syncthreads();
  if (!p.merge_in_kernel) allow_dependents();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  ptx::cluster_sync();
  if (p.expect_whole && work[4] > 0 && work[5] == 0 && threadIdx.x == 0 && blockIdx.x == 0) report(MLA_ERR_DEVICE_CHECK);
  if (p.merge_in_kernel) {
    // Launched cooperatively: when a sequence was cut (the same decision in every CTA, from the same
    // totals) every CTA passes one grid-wide barrier, after which all parts are written and visible,
    // and the grid's warps take the (token, head) units in turn. Every path of the kernel arrives
    // here (all waits above are bounded), so the barrier always completes.
    if (work[4] > 0 && work[5] == 0) {
      cooperative_groups::this_grid().sync();
      const int per = (p.B + 31) / 32;
      const int b0 = min(p.B, lane * per), b1 = min(p.B, b0 + per);
      const int warps = kThreads / 32;
      const long long units = (long long)p.B * p.s_q * kH;
      for (long long u = (long long)blockIdx.x * warps + warp; u < units; u += (long long)gridDim.x * warps)
        merge_token_head(p.seqlens, p.s_q, p.max_tiles, npairs / p.s_q, work[4], b0, b1, (int)(u / kH), (int)(u % kH),
                         p.part_o, p.part_lse, p.o_lat, p.lse);
    }
    allow_dependents();
  }
}

// One warp per (sequence, head), 4 heads per block of 128 threads (about 1.4 waves at 48 registers).
// Each warp finds the sequence's tile range itself (no block barrier), then issues all its
// partial loads before combining them.
constexpr int kMergeHeads = 4;
constexpr int kMergeTokenBlocks = 8;   // blocks along the tokens; each strides over them
__global__ void __launch_bounds__(32 * kMergeHeads)
merge_kernel(const int32_t* __restrict__ seqlens, int B, int s_q, int max_tiles, int npairs, const float* __restrict__ part_o,
             const float* __restrict__ part_lse, __nv_bfloat16* __restrict__ o_lat, float* __restrict__ lse) {
  // blocks stride over the new tokens v = b * s_q + tok; a token's parts come from pair (group, tok) of
  // the groups that covered its sequence's tiles
  const int G = npairs / s_q;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dependency_wait();
  allow_dependents();
  // the total of tiles and the longest sequence decide the split, the same for every token: lane l
  // sums sequences [l*per, (l+1)*per)
  const int per = (B + 31) / 32;
  const int b0 = min(B, lane * per), b1 = min(B, b0 + per);
  long long local = 0;
  int max_tb = 0;
  for (int x = b0; x < b1; ++x) {
    const int tb = tiles_of(__ldg(seqlens + x), max_tiles);
    local += tb;
    max_tb = max(max_tb, tb);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    local += __shfl_xor_sync(0xffffffffu, local, o);
    max_tb = max(max_tb, __shfl_xor_sync(0xffffffffu, max_tb, o));
  }
  const long long T = local;
  if (T == 0 || G == 0 || whole_sequences(B, G, T, max_tb)) return;   // nothing was cut
  for (int v = blockIdx.x; v < B * s_q; v += gridDim.x)
    merge_token_head(seqlens, s_q, max_tiles, G, T, b0, b1, v, blockIdx.y * kMergeHeads + warp, part_o, part_lse, o_lat, lse);
}

// ---- host side -----------------------------------------------------------------------------------------
// s_q new tokens per sequence take s_q pairs each (one token per pair): at most kMaxTokens.
constexpr int kMaxTokens = 8;
inline bool decode_supported(const mla_dims_t* d, int32_t dtype, int32_t B, int32_t s_q) {
  return dtype == MLA_BF16 && d->H == kH && d->d_c == kDC && d->d_r == kDR && s_q >= 1 && s_q <= kMaxTokens &&
         B >= 1;
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

#ifdef MLA_TEST_HOOKS
// Test builds only: launch the decode and the merge kernel as two launches (the path taken when the
// runtime refuses the cooperative launch), so that a test keeps that path covered.
inline bool g_test_two_launches = false;
#endif

inline int launch_decode(const mla_dims_t* d, int32_t B, int32_t s_q, const void* q_abs, const mla_latent_cache_t* cache,
                         const int32_t* block_table, int32_t max_pages, const int32_t* seqlens, void* o_lat, float* lse,
                         void* workspace, size_t ws_bytes, int num_sms, const int32_t* seqlens_host, cudaStream_t st) {
  if (!workspace || ws_bytes < decode_workspace_bytes(d, MLA_BF16, B, s_q, num_sms)) return MLA_ERR_WORKSPACE;
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
  CUtensorMap tm_q;   // q_abs as [B*s_q*128 heads, 576]: boxes of 64 heads x 64 columns
  if (!make_tmap(&tm_q, q_abs, kRow, (int64_t)B * s_q * kH, kRow)) return MLA_ERR_INVALID_ARG;
  const int P = active_pairs(num_sms);
  if (P < s_q) return MLA_ERR_UNSUPPORTED;   // every token of a sequence needs a pair of its own
  Params prm;
  prm.q_abs = reinterpret_cast<const __nv_bfloat16*>(q_abs);
  prm.block_table = block_table;
  prm.max_pages = max_pages;
  prm.num_pages = cache->num_pages;
  prm.seqlens = seqlens;
  prm.B = B;
  prm.s_q = s_q;
  prm.max_tiles = max_pages;
  prm.o_lat = reinterpret_cast<__nv_bfloat16*>(o_lat);
  prm.lse = lse;
  prm.part_o = reinterpret_cast<float*>(workspace);
  prm.part_lse = prm.part_o + (size_t)2 * max_pairs(num_sms) * kH * kDC;
  prm.sm_scale_log2 = d->sm_scale * 1.4426950408889634f;
  prm.expect_whole = 0;
  if (seqlens_host) {
    // the host's copy of the lengths decides the split as the kernel will: when nothing is cut, the
    // decode goes as a plain launch (programmatic dependent launch, no merge at all)
    long long T = 0;
    int max_tb = 0;
    for (int b = 0; b < B; ++b) {
      const int tb = tiles_of(seqlens_host[b], max_pages);
      T += tb;
      max_tb = std::max(max_tb, tb);
    }
    if (T == 0 || whole_sequences(B, P / s_q, T, max_tb)) {
      prm.merge_in_kernel = 0;
      prm.expect_whole = 1;
      launch_pdl(decode_kernel, dim3(2 * P), dim3(kThreads), kSmemBytes, st, tm_lat, tm_rope, tm_q, prm);
      return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
    }
  }
  // First choice: one cooperative launch that merges cut sequences itself (no merge kernel, no
  // kernel boundary after the decode). If the runtime does not take a cooperative launch of this
  // clustered grid (with programmatic dependent launch, then without), the decode and the merge
  // kernel go as two launches. The outcome is remembered per device.
  static int coop_mode[64] = {0};   // 0 unknown, 1 cooperative + PDL, 2 cooperative, 3 two launches
  const int di = (dev >= 0 && dev < 64) ? dev : 0;
  bool forced = false;
#ifdef MLA_TEST_HOOKS
  forced = g_test_two_launches;
#endif
  for (int mode = forced ? 3 : (coop_mode[di] ? coop_mode[di] : 1); mode <= 3; ++mode) {
    if (mode == 3) {
      prm.merge_in_kernel = 0;
      launch_pdl(decode_kernel, dim3(2 * P), dim3(kThreads), kSmemBytes, st, tm_lat, tm_rope, tm_q, prm);
      launch_pdl(merge_kernel, dim3(std::min(B * s_q, kMergeTokenBlocks), kH / kMergeHeads), dim3(32 * kMergeHeads), 0,
                 st, seqlens, (int)B, (int)s_q, (int)max_pages, P, (const float*)prm.part_o,
                 (const float*)prm.part_lse, prm.o_lat, lse);
      if (!forced) coop_mode[di] = 3;
      break;
    }
    prm.merge_in_kernel = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = mode == 1 ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, decode_kernel, tm_lat, tm_rope, tm_q, prm) == cudaSuccess) {
      g_launches.fetch_add(1, std::memory_order_relaxed);
      coop_mode[di] = mode;
      break;
    }
    (void)cudaGetLastError();   // a configuration the runtime refused: nothing was launched
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace sm100
}  // namespace mla

// GQLA grouped decode on the sm_100a tensor cores (« Résumé technique : GQLA … », « Architecture »,
// « Chemin GQA »): the cache holds, per position, K_g and V_g for each of g groups (16 heads share
// a group) and one RoPE key shared by all heads. Shapes fixed here: 16 heads per group,
// D = d_v = 128, d_r = 64, one new token per sequence, bf16 storage, fp32 accumulation.
//
// The contraction is laid out with positions as the MMA's M: for a 128-position tile of one
// (sequence, group),
//   Sᵀ [128 positions x 16 heads] = [K_g ; k_r] (128 x 192, K-major) · [q ; q_r]ᵀ (192 x 16)
//   Oᵀ [128 d_v x 16 heads]      += V_gᵀ (MN-major: V_g read as stored) · Pᵀ (128 positions x 16)
// so both accumulators take 16 TMEM columns and one CTA does all of it. A thread of the four
// compute warps owns one TMEM lane: one position of S, one latent column of O. Per-head maxima
// and sums over the tile's positions are shuffle reductions plus one exchange through shared
// memory; the running maximum moves lazily (only past 2^8), then the head's column of O is scaled.
// Work: persistent CTAs over (sequence, group, split) units; splits are merged by the CUDA-core
// merge kernel. Every wait is bounded; on expiry the kernel records MLA_ERR_TIMEOUT and drains.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace gqla {

constexpr int kHG = 16;                  // heads per group
constexpr int kD = 128, kDV = 128, kDR = 64;
constexpr int kTile = 128;               // positions per tile = two pages
constexpr int kBox = 64 * 128;           // one TMA box: 64 rows x 64 bf16 (8 KB)
constexpr int kKRBytes = 6 * kBox;       // K (2 column chunks x 2 pages) + RoPE key (2 pages)
constexpr int kVBytes = 4 * kBox;        // V (2 column chunks x 2 pages)
constexpr int kKRStages = 2;             // [K_g ; k_r] tiles in flight (released by the tile's score MMAs)
constexpr int kVStages = 3;              // V_g tiles in flight (held one tile longer, until the output MMA)
constexpr int kQBytes = 3 * kHG * 128;   // [q (2 chunks) ; q_r (1 chunk)] x 16 heads, 128-byte swizzle
constexpr int kPBytes = 2 * kHG * 128;   // Pᵀ: 16 heads x 128 positions (2 chunks)
constexpr int kThreads = 256;            // 0 TMA, 1 MMA, 2 TMEM, 3 idle, 4-7 compute
constexpr float kRescaleLog2 = 8.0f;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// shared memory (from a 1024-aligned base)
constexpr int kOffKR = 0;
constexpr int kOffV = kOffKR + kKRStages * kKRBytes;    // 98304
constexpr int kOffQ = kOffV + kVStages * kVBytes;       // 196608
constexpr int kOffP = kOffQ + 2 * kQBytes;              // 208896
constexpr int kOffRed = kOffP + 2 * kPBytes;            // float [2][4][16] per-warp head maxima; [4][16] sums
constexpr int kOffInvFreq = kOffRed + 3 * 4 * kHG * 4;  // double [32]
constexpr int kOffBar = kOffInvFreq + 32 * 8;
enum Bar : int {
  KR_FULL = 0, KR_EMPTY = KR_FULL + kKRStages, V_FULL = KR_EMPTY + kKRStages, V_EMPTY = V_FULL + kVStages,
  S_FULL = V_EMPTY + kVStages, S_EMPTY = S_FULL + 2, P_READY = S_EMPTY + 2, P_FREE = P_READY + 2,
  Q_FULL = P_FREE + 2, Q_EMPTY = Q_FULL + 2, NUM_BARS = Q_EMPTY + 2
};
constexpr int kOffTmemSlot = kOffBar + NUM_BARS * 8;
constexpr int kOffAbort = kOffTmemSlot + 8;
constexpr int kSmemBytes = kOffAbort + 8 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0 && kOffBar % 8 == 0, "alignment");
constexpr uint32_t kTmemCols = 64;       // S buffers at 0 and 16, O at 32

struct Params {
  const __nv_bfloat16* q_nope;     // [B, H, 128]
  const __nv_bfloat16* q_rope;     // [B, H, 64], not yet rotated
  const int32_t* block_table;
  const int32_t* seqlens;
  int max_pages, num_pages, B, g, H;
  int nsplit, chunk;               // a unit covers tiles [split*chunk, (split+1)*chunk) of its sequence
  float sm_scale_log2, rope_base;
  __nv_bfloat16* out;              // [B, H, 128]
  float* lse;                      // [B, H]
  float* part_o;                   // [B*H*nsplit, 128] when nsplit > 1
  float* part_lse;                 // [B*H*nsplit]
};

// unit -> (sequence, group, split) and its tile range [t0, t1) (empty when past the sequence)
struct Unit {
  int b, gi, split, t0, t1, L;
};
__device__ __forceinline__ Unit unit_of(const Params& p, int u) {
  Unit x;
  x.split = u % p.nsplit;
  x.gi = (u / p.nsplit) % p.g;
  x.b = u / (p.nsplit * p.g);
  x.L = p.seqlens[x.b];
  const int tiles = (x.L + kTile - 1) / kTile;
  x.t0 = min(tiles, x.split * p.chunk);
  x.t1 = min(tiles, x.t0 + p.chunk);
  return x;
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t n = 0;; ++n) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((n & 15u) == 15u) {
      if (*abort_flag) return false;
      const uint64_t now = ptx::globaltimer();
      if (t0 == 0) t0 = now;
      else if (now - t0 > kTimeoutNs) {
        report(MLA_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag));
}

__global__ void __launch_bounds__(kThreads, 1)
gqla_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
            const __grid_constant__ CUtensorMap tm_r, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return base + kOffBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOffAbort);
  const int units = p.B * p.g * p.nsplit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKRStages; ++i) { ptx::mbar_init(bar(KR_FULL + i), 1); ptx::mbar_init(bar(KR_EMPTY + i), 1); }
    for (int i = 0; i < kVStages; ++i) { ptx::mbar_init(bar(V_FULL + i), 1); ptx::mbar_init(bar(V_EMPTY + i), 1); }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(S_FULL + i), 1); ptx::mbar_init(bar(S_EMPTY + i), 128);
      ptx::mbar_init(bar(P_READY + i), 128); ptx::mbar_init(bar(P_FREE + i), 1);
      ptx::mbar_init(bar(Q_FULL + i), 128); ptx::mbar_init(bar(Q_EMPTY + i), 1);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::prefetch_tmap(&tm_r);
  }
  if (warp == 2) { ptx::tmem_alloc(base + kOffTmemSlot, kTmemCols); ptx::tmem_relinquish(); }
  grid_dependency_wait();
  // a sequence must hold at least its new token: an empty one is reported (its outputs stay unwritten)
  for (int b = blockIdx.x * kThreads + threadIdx.x; b < p.B; b += gridDim.x * kThreads)
    if (p.seqlens[b] < 1) report(MLA_ERR_DEVICE_CHECK);
  ptx::tc_fence_before();
  __syncthreads();
  allow_dependents();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + kOffTmemSlot);

  if (warp == 0) {
    if (lane == 0) {   // ---- TMA producer: K_g, k_r and V_g of each tile, two pages per tile
      uint32_t i = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit x = unit_of(p, u);
        const int pages = (x.L + 63) / 64;
        for (int t = x.t0; t < x.t1 && ok; ++t, ++i) {
          const uint32_t s = i % kKRStages, ph = ((i / kKRStages) & 1u) ^ 1u;
          const uint32_t sv = i % kVStages, phv = ((i / kVStages) & 1u) ^ 1u;
          int pg[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int lp = 2 * t + j;
            // a page past the sequence's end reads as zeros (a row beyond the tensor map)
            if (lp < pages && lp >= p.max_pages) {   // longer than its table row: reported, read as zeros
              report(MLA_ERR_DEVICE_CHECK);
              pg[j] = p.num_pages;
              continue;
            }
            pg[j] = lp < pages ? p.block_table[(long long)x.b * p.max_pages + lp] : p.num_pages;
            if (lp < pages && (pg[j] < 0 || pg[j] >= p.num_pages)) {
              report(MLA_ERR_DEVICE_CHECK);
              pg[j] = p.num_pages;
            }
          }
          if (!(ok = wait_bar(bar(KR_EMPTY + s), ph, abort_flag))) break;
          const uint32_t kr = base + kOffKR + s * kKRBytes;
          ptx::mbar_arrive_expect_tx(bar(KR_FULL + s), kKRBytes);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            ptx::tma_load_2d(kr + j * kBox, &tm_k, x.gi * kD, pg[j] * 64, bar(KR_FULL + s));
            ptx::tma_load_2d(kr + 2 * kBox + j * kBox, &tm_k, x.gi * kD + 64, pg[j] * 64, bar(KR_FULL + s));
            ptx::tma_load_2d(kr + 4 * kBox + j * kBox, &tm_r, 0, pg[j] * 64, bar(KR_FULL + s));
          }
          if (!(ok = wait_bar(bar(V_EMPTY + sv), phv, abort_flag))) break;
          const uint32_t vv = base + kOffV + sv * kVBytes;
          ptx::mbar_arrive_expect_tx(bar(V_FULL + sv), kVBytes);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            ptx::tma_load_2d(vv + j * kBox, &tm_v, x.gi * kDV, pg[j] * 64, bar(V_FULL + sv));
            ptx::tma_load_2d(vv + 2 * kBox + j * kBox, &tm_v, x.gi * kDV + 64, pg[j] * 64, bar(V_FULL + sv));
          }
        }
      }
      // loads in flight land before the CTA may exit
      for (uint32_t k = (i > (uint32_t)kKRStages ? i - kKRStages : 0); k < i; ++k)
        wait_bar(bar(KR_FULL + k % kKRStages), (k / kKRStages) & 1u, abort_flag);
      for (uint32_t k = (i > (uint32_t)kVStages ? i - kVStages : 0); k < i; ++k)
        wait_bar(bar(V_FULL + k % kVStages), (k / kVStages) & 1u, abort_flag);
    }
  } else if (warp == 1) {
    // ---- MMA issuer (lane 0; the warp zeroes V rows past a sequence's end). Order within a unit: S
    // of tile i, then O of tile i - 1, so the softmax of a tile overlaps the next tile's scores.
    const uint32_t idesc_s = ptx::idesc_bf16_f32_ab(128, kHG, false, false);
    const uint32_t idesc_o = ptx::idesc_bf16_f32_ab(128, kHG, true, false);
    uint32_t i = 0, nu = 0;
    bool ok = true;
    int prev_first = 1, prev_valid = kTile;   // the pending O tile: first of its unit? valid rows
    auto issue_o = [&](uint32_t j) -> bool {
      const uint32_t s = j % kVStages, pb = j % 2;
      if (!wait_bar_warp(bar(P_READY + pb), (j / 2) & 1u, abort_flag)) return false;
      if (!wait_bar_warp(bar(V_FULL + s), (j / kVStages) & 1u, abort_flag)) return false;
      uint8_t* vst = gbase + kOffV + s * kVBytes;
      if (prev_valid < kTile) {   // V rows past the end may hold anything (0 * NaN = NaN): zero them
        const int zr = kTile - prev_valid;
        for (int q = lane; q < zr * 2 * 8; q += 32) {
          const int r = prev_valid + q / 16, rest = q % 16, c = rest / 8;   // chunk c, 16-byte piece
          reinterpret_cast<uint4*>(vst + c * 2 * kBox + r * 128)[rest % 8] = make_uint4(0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_after();
        // A = V_gᵀ: MN-major, 64-column chunks 16 KB apart (LBO), 8-position groups 1 KB apart
        const uint64_t ad = ptx::smem_desc_sw128(base + kOffV + s * kVBytes, 2 * kBox, 1024);
        const uint32_t pbase = base + kOffP + pb * kPBytes;
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
          const uint64_t bd = ptx::smem_desc_sw128(pbase + (k >> 2) * (kHG * 128), 16, 1024) + (uint64_t)(2 * (k & 3));
          ptx::mma_ss(tmem + 32, ad + (uint64_t)(k * (2048 >> 4)), bd, idesc_o, (prev_first && k == 0) ? 0u : 1u);
        }
        ptx::mma_commit(bar(V_EMPTY + s));
        ptx::mma_commit(bar(P_FREE + pb));
      }
      __syncwarp();
      return true;
    };
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++nu) {
      const Unit x = unit_of(p, u);
      const uint32_t qb = nu % 2;
      // every unit's query is waited for, in order, and its buffer handed back (after the unit's
      // score MMAs, or at once for a unit without tiles): the two buffers form a ring, so no wait
      // can take an older phase of the same parity for the one it wants
      if (!(ok = wait_bar_warp(bar(Q_FULL + qb), (nu / 2) & 1u, abort_flag))) break;
      if (x.t1 <= x.t0) {
        if (lane == 0) ptx::mbar_arrive(bar(Q_EMPTY + qb));
        continue;
      }
      for (int t = x.t0; t < x.t1; ++t, ++i) {
        const uint32_t s = i % kKRStages, sb = i % 2;
        if (!(ok = wait_bar_warp(bar(S_EMPTY + sb), ((i / 2) & 1u) ^ 1u, abort_flag))) break;
        if (!(ok = wait_bar_warp(bar(KR_FULL + s), (i / kKRStages) & 1u, abort_flag))) break;
        if (lane == 0) {
          ptx::tc_fence_after();
          const uint32_t kr = base + kOffKR + s * kKRBytes, qq = base + kOffQ + qb * kQBytes;
#pragma unroll
          for (int c = 0; c < 3; ++c) {
            const uint64_t ad = ptx::smem_desc_sw128(kr + c * 2 * kBox, 16, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(qq + c * kHG * 128, 16, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              ptx::mma_ss(tmem + 16u * sb, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc_s, (c | k) ? 1u : 0u);
          }
          ptx::mma_commit(bar(S_FULL + sb));
          ptx::mma_commit(bar(KR_EMPTY + s));
        }
        __syncwarp();
        if (t > x.t0 && !(ok = issue_o(i - 1))) break;
        prev_first = (t == x.t0);
        prev_valid = min(kTile, x.L - t * kTile);
      }
      // a unit's last O MMA goes before the next unit's scores: the compute warps prepare the next
      // query only after this unit's epilogue, which waits for it
      if (ok) ok = issue_o(i - 1);
      if (ok && lane == 0) ptx::mma_commit(bar(Q_EMPTY + qb));
    }
  } else if (warp >= 4) {
    // ---- compute warps: thread r = TMEM lane = a position of S and a latent column of O
    const int r = threadIdx.x - 128, w = warp - 4;
    const uint32_t lane_off = (uint32_t)(w * 32) << 16;
    float* red = reinterpret_cast<float*>(gbase + kOffRed);
    double* inv_freq = reinterpret_cast<double*>(gbase + kOffInvFreq);
    if (r < kDR / 2) inv_freq[r] = rope_inv_freq(r, kDR, p.rope_base);
    ptx::named_bar_sync(1, 128);
    // [q ; RoPE(q_r)] of a unit's 16 heads into a Q buffer (K-major, 128-byte swizzle)
    // (nq = the unit's position in this CTA's sequence; buffer nq % 2, its use nq / 2 of that buffer)
    auto prepare_q = [&](int u, uint32_t nq) -> bool {
      // the four warps pass units without tiles without meeting; they meet here, so a buffer's
      // arrivals for one unit never mix with those for the next
      ptx::named_bar_sync(1, 128);
      const uint32_t qb = nq % 2;
      if (!wait_bar_warp(bar(Q_EMPTY + qb), ((nq / 2) & 1u) ^ 1u, abort_flag)) return false;
      const Unit x = unit_of(p, u);
      const uint32_t qq = base + kOffQ + qb * kQBytes;
      const int pos = x.L - 1;
      for (int e = r; e < kHG * 16; e += 128) {   // q: 16 heads x 16 pieces of 16 bytes
        const int h = e / 16, c16 = e % 16;
        const uint4 v = *reinterpret_cast<const uint4*>(p.q_nope + ((size_t)x.b * p.H + x.gi * kHG + h) * kD + c16 * 8);
        ptx::st_shared_v4(qq + (c16 >> 3) * (kHG * 128) + (h >> 3) * 1024 + (h & 7) * 128 + (((c16 & 7) ^ (h & 7)) << 4),
                          v.x, v.y, v.z, v.w);
      }
      for (int e = r; e < kHG * (kDR / 2); e += 128) {   // q_r: 16 heads x 32 pairs, rotated
        const int h = e / (kDR / 2), q = e % (kDR / 2);
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(
            p.q_rope + ((size_t)x.b * p.H + x.gi * kHG + h) * kDR + 2 * q);
        float cs, sn;
        rope_cos_sin_at(pos, inv_freq[q], &cs, &sn);
        const float a = __low2float(v), bb = __high2float(v);
        const uint32_t packed = ptx::pack_bf16x2(a * cs - bb * sn, a * sn + bb * cs);
        ptx::st_shared_u32(qq + 2 * (kHG * 128) + (h >> 3) * 1024 + (h & 7) * 128 + ((((q >> 2) & 7) ^ (h & 7)) << 4) + (q & 3) * 4,
                           packed);
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(bar(Q_FULL + qb));
      return true;
    };
    uint32_t i = 0, nu = 0;
    bool ok = true;
    if ((int)blockIdx.x < units && !prepare_q(blockIdx.x, 0)) ok = false;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++nu) {
      const Unit x = unit_of(p, u);
      float m[kHG], lp[kHG];
#pragma unroll
      for (int h = 0; h < kHG; ++h) { m[h] = -INFINITY; lp[h] = 0.f; }
      for (int t = x.t0; t < x.t1; ++t, ++i) {
        const uint32_t sb = i % 2;
        bool good = ok && wait_bar_warp(bar(S_FULL + sb), (i / 2) & 1u, abort_flag);
        uint32_t sr[16];
        if (good) {
          ptx::tc_fence_after();
          ptx::tmem_ld16(tmem + lane_off + 16u * sb, sr);
          ptx::tmem_wait_ld();
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(S_EMPTY + sb));
        }
        const bool valid = t * kTile + r < x.L;
        float s[kHG], mx[kHG];
#pragma unroll
        for (int h = 0; h < kHG; ++h) {
          s[h] = (good && valid) ? __uint_as_float(sr[h]) * p.sm_scale_log2 : -INFINITY;
          mx[h] = s[h];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
          for (int h = 0; h < kHG; ++h) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
        float* rb = red + (i & 1u) * 4 * kHG;
        if (lane < kHG) {
          float v = mx[0];
#pragma unroll
          for (int h = 1; h < kHG; ++h) v = (lane == h) ? mx[h] : v;
          rb[w * kHG + lane] = v;
        }
        // the four warps meet once per tile and agree whether to go on
        if (ptx::named_bar_or(1, 128, !good)) { ok = false; break; }
        float al[kHG];
        bool moved = false;
#pragma unroll
        for (int h = 0; h < kHG; ++h) {
          const float tm = fmaxf(fmaxf(rb[h], rb[kHG + h]), fmaxf(rb[2 * kHG + h], rb[3 * kHG + h]));
          al[h] = 1.f;
          if (tm > m[h] + kRescaleLog2) {
            al[h] = (m[h] == -INFINITY) ? 0.f : ptx::ex2_approx(m[h] - tm);
            lp[h] *= al[h];
            m[h] = tm;
            moved = true;
          }
        }
        // Pᵀ into the tile's P buffer once the O MMA of tile i - 2 is done with it
        const uint32_t pb = i % 2;
        if (i >= 2 && !wait_bar_warp(bar(P_FREE + pb), ((i - 2) / 2) & 1u, abort_flag)) { ok = false; }
        const uint32_t pbase = base + kOffP + pb * kPBytes + (r >> 6) * (kHG * 128);
        const int rr = r & 63;
#pragma unroll
        for (int h = 0; h < kHG; ++h) {
          const float e = ptx::ex2_approx(s[h] - m[h]);   // -inf (masked) gives 0
          lp[h] += e;
          const __nv_bfloat16 bv = __float2bfloat16_rn(e);
          *reinterpret_cast<__nv_bfloat16*>(gbase + (pbase - base) + (h >> 3) * 1024 + (h & 7) * 128 +
                                            ((((rr >> 3) & 7) ^ (h & 7)) << 4) + (rr & 7) * 2) = bv;
        }
        ptx::fence_proxy_async_smem();
        // a head's running maximum moved: scale its column of O once the previous tile's O MMA is done
        if (ok && t > x.t0 && moved) {
          if (!wait_bar_warp(bar(P_FREE + ((i - 1) % 2)), ((i - 1) / 2) & 1u, abort_flag)) {
            ok = false;
          } else {
            ptx::tc_fence_after();
            uint32_t o[16];
            ptx::tmem_ld16(tmem + lane_off + 32u, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < kHG; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * al[h]);
            ptx::tmem_st16(tmem + lane_off + 32u, o);
            ptx::tmem_wait_st();
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(P_READY + pb));
      }
      if (!ok) break;
      // the next unit's query while this unit's last O MMA runs
      if (u + (int)gridDim.x < units && !prepare_q(u + gridDim.x, nu + 1)) ok = false;
      if (x.t1 <= x.t0) {   // nothing of this sequence here: an empty part
        if (p.nsplit > 1 && r < kHG)
          p.part_lse[((size_t)x.b * p.H + x.gi * kHG + r) * p.nsplit + x.split] = -INFINITY;
        continue;
      }
      // epilogue: row sums over the 128 positions, then Oᵀ / l (thread r = latent column r)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int h = 0; h < kHG; ++h) lp[h] += __shfl_xor_sync(0xffffffffu, lp[h], o);
      float* sb = red + 2 * 4 * kHG;
      if (lane < kHG) {
        float v = lp[0];
#pragma unroll
        for (int h = 1; h < kHG; ++h) v = (lane == h) ? lp[h] : v;
        sb[w * kHG + lane] = v;
      }
      const uint32_t last = i - 1;
      bool fin = wait_bar_warp(bar(P_FREE + (last % 2)), (last / 2) & 1u, abort_flag);
      if (ptx::named_bar_or(1, 128, !fin)) { ok = false; break; }
      ptx::tc_fence_after();
      uint32_t o[16];
      ptx::tmem_ld16(tmem + lane_off + 32u, o);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
#pragma unroll
      for (int h = 0; h < kHG; ++h) {
        const float l = (sb[h] + sb[kHG + h]) + (sb[2 * kHG + h] + sb[3 * kHG + h]);
        const size_t head = (size_t)x.b * p.H + x.gi * kHG + h;
        const float v = __uint_as_float(o[h]) / l;
        if (p.nsplit > 1) {
          p.part_o[(head * p.nsplit + x.split) * kDV + r] = v;
          if (r == 0) p.part_lse[head * p.nsplit + x.split] = (m[h] + log2f(l)) * 0.69314718055994531f;
        } else {
          p.out[head * kDV + r] = __float2bfloat16_rn(v);
          if (r == 0) p.lse[head] = (m[h] + log2f(l)) * 0.69314718055994531f;
        }
      }
      // the sums buffer is rewritten at the next unit's end, after that unit's per-tile meetings
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host ------------------------------------------------------------------------------------------
inline bool supported(const mla_dims_t* d, int32_t dtype, int32_t s_q) {
  return dtype == MLA_BF16 && s_q == 1 && d->g > 0 && d->H == d->g * kHG && d->D == kD && d->d_v == kDV &&
         d->d_r == kDR && d->page_size == 64;
}

struct Split { int nsplit, chunk; };
inline Split plan(int B, int g, int max_pages, int num_sms) {
  const int tiles = (max_pages + 1) / 2;
  int ns = (6 * num_sms + B * g - 1) / (B * g);
  ns = std::max(1, std::min(ns, tiles));
  const int chunk = (tiles + ns - 1) / ns;
  return {(tiles + chunk - 1) / chunk, chunk};
}

inline size_t workspace_bytes(const mla_dims_t* d, int32_t B, int32_t max_pages, int num_sms) {
  const Split sp = plan(B, d->g, max_pages, num_sms);
  if (sp.nsplit <= 1) return 0;
  const size_t slots = (size_t)B * d->H * sp.nsplit;
  return slots * kDV * sizeof(float) + slots * sizeof(float) + 256;
}

inline int launch_gqla(const mla_dims_t* d, int32_t B, const void* q_nope, const void* q_rope,
                       const mla_gqa_cache_t* cache, const int32_t* block_table, int32_t max_pages,
                       const int32_t* seqlens, void* out, float* lse, void* workspace, size_t ws_bytes, int num_sms,
                       cudaStream_t st) {
  const Split sp = plan(B, d->g, max_pages, num_sms);
  Params prm{};
  if (sp.nsplit > 1) {
    const size_t slots = (size_t)B * d->H * sp.nsplit;
    if (!workspace || ws_bytes < slots * kDV * sizeof(float) + slots * sizeof(float)) return MLA_ERR_WORKSPACE;
    prm.part_o = reinterpret_cast<float*>(workspace);
    prm.part_lse = prm.part_o + slots * kDV;
  }
  const int64_t rows = (int64_t)cache->num_pages * 64;
  CUtensorMap tm_k, tm_v, tm_r;
  if (!tmap::make_bf16_sw128(&tm_k, cache->k, (int64_t)d->g * kD, rows, cache->k_stride, 64) ||
      !tmap::make_bf16_sw128(&tm_v, cache->v, (int64_t)d->g * kDV, rows, cache->v_stride, 64) ||
      !tmap::make_bf16_sw128(&tm_r, cache->rope, kDR, rows, cache->rope_stride, 64))
    return MLA_ERR_INVALID_ARG;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev]) {
    if (cudaFuncSetAttribute(gqla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
      return MLA_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_done[dev] = true;
  }
  prm.q_nope = reinterpret_cast<const __nv_bfloat16*>(q_nope);
  prm.q_rope = reinterpret_cast<const __nv_bfloat16*>(q_rope);
  prm.block_table = block_table;
  prm.seqlens = seqlens;
  prm.max_pages = max_pages;
  prm.num_pages = cache->num_pages;
  prm.B = B;
  prm.g = d->g;
  prm.H = d->H;
  prm.nsplit = sp.nsplit;
  prm.chunk = sp.chunk;
  prm.sm_scale_log2 = d->sm_scale * 1.4426950408889634f;
  prm.rope_base = d->rope_base;
  prm.out = reinterpret_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  const int units = B * d->g * sp.nsplit;
  mla::launch_pdl(gqla_kernel, dim3(std::min(units, num_sms)), dim3(kThreads), (size_t)kSmemBytes, st, tm_k, tm_v, tm_r,
                  prm);
  if (sp.nsplit > 1)
    mla::launch(simt::merge_splits_kernel<__nv_bfloat16>, dim3(B * d->H), dim3(128), 0, st,
                (const float*)prm.part_o, (const float*)prm.part_lse, sp.nsplit, kDV,
                reinterpret_cast<__nv_bfloat16*>(out), (int64_t)kDV, lse);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace gqla
}  // namespace mla

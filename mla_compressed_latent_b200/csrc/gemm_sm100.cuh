// Per-head "activations times weights" GEMM on the sm_100a tensor cores, for the projections of a
// decode step: query absorption (q_nope · W_UK[h]), the output projection (o_lat · W_UV[h]) and the
// cache-append projection (x · [W_DKV | W_KR], split over K). At decode batch sizes all three are
// bound by reading the weights once, so the kernel streams weight tiles with TMA into a ring of
// shared-memory stages and keeps one tcgen05 MMA chain fed from it.
//
//   Y[tok, h, m] = sum_k X[tok, h, k] · W[h, k, m]
// is computed transposed, D[m, tok] = A[m, k] · B[tok, k], with A = W[h]ᵀ (the weights' row-major
// [k, m] layout is MN-major for A, so they are read as stored) and B = X[:, h, :] (K-major). One
// CTA owns one head, 128 output features (MMA M) and up to 128 tokens (MMA N), and a range of K in
// chunks of 64. The fp32 accumulator lives in TMEM; four epilogue warps read it back (one TMEM lane
// = one output feature) and write bf16 rows or fp32 split-K partial sums.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace gemm {

constexpr int kBM = 128;         // output features per CTA (MMA M)
constexpr int kBK = 64;          // K per stage: one 128-byte swizzle row of bf16
constexpr int kMaxStages = 8;           // a CTA streaming a long K keeps up to 8 chunks (192 KB) in flight
constexpr int kThreads = 256;    // warp 0 TMA producer, 1 MMA issuer, 2 TMEM owner, 4-7 epilogue
constexpr int kABytes = kBK * 128 * 2;   // two boxes of 64 k-rows x 64 features
constexpr int kBarBytes = 1024;          // barriers, TMEM address slot, RoPE inverse frequencies
constexpr int kInvFreqOff = 512;         // double [d_r / 2 <= 64] inside the barrier area
constexpr uint64_t kTimeoutNs = 2000000000ull;

struct Params {
  int M, K;                // output features per head, reduction length per head (K % 64 == 0)
  int n_tok;               // rows of X
  int chunks_per_split;    // K chunks (of 64) per blockIdx.z
  int tn;                  // tokens per CTA = MMA N: 32, 64 or 128
  int stages;              // ring depth, 1..kMaxStages
  // mode 0: bf16 Y[tok * y_tok_stride + h * y_head_stride + m]
  // mode 1: fp32 part[(split * n_tok + tok) * M + m]   (one head)
  int mode;
  __nv_bfloat16* y;
  int64_t y_tok_stride, y_head_stride;
  float* part;
  // Optional rotated tail (query absorption): the m-tile-0 CTA of head h also writes
  // Y[tok, h, M + 2i], Y[tok, h, M + 2i + 1] = RoPE of rope_in[tok, h, 2i .. 2i + 1] at the token's
  // position seqlens[tok / s_q] - s_q + tok % s_q.
  const __nv_bfloat16* rope_in;
  int d_r, H, s_q;
  const int32_t* seqlens;
  float rope_base;
  // Optional second problem in the same launch (mode 0, no rotated tail): the CTAs past the first
  // problem's H * m_tiles take the m-tiles of a second weight [K, M2] on the same tokens and write
  // y2[tok * y2_tok_stride + m]. M2 = 0: none.
  int M2;
  __nv_bfloat16* y2;
  int64_t y2_tok_stride;
  // Layouts: a_kmajor = the weights are stored [H, M, K] (K contiguous: W[h] transposed), read
  // K-major; x_shared = X is [n_tok, K], one row per token shared by every head.
  int a_kmajor, x_shared;
  // set by run(): every output row start is 16-byte aligned (base and strides), so the epilogue may
  // store 16-byte pieces
  int vec_out;
  // set by run(): the grid of CTAs (x = head * CTAs per head [+ the second problem's m-tiles],
  // y = token block, z = K split)
  int gx, gy, gz;
  // 1: the weights are not written by the kernel launched before this one on the stream, so a CTA
  // issues its first weight tiles before it waits for that kernel (everything else after)
  int w_early;
  // m-tiles (128 output features each) per CTA, 1..4: a head's tiles side by side in TMEM, fed by
  // one token box per K chunk (1 with a second problem or K-major weights)
  int m_sub;
};

__host__ __device__ constexpr int stage_bytes(int tn, int msub = 1) { return msub * kABytes + tn * 128; }
__host__ __device__ constexpr int smem_bytes(int tn, int stages, int msub = 1) {
  return 1024 + kBarBytes + stages * stage_bytes(tn, msub);
}

#ifdef MLA_TEST_HOOKS
// Test builds only: with g_test_stall set, each CTA's MMA issuer first waits for a barrier phase that
// nothing completes, with a 10 ms limit, so that the bounded-wait path (status, abort, drain) runs.
__device__ int g_test_stall;
#endif

// Waits for the phase of `parity`. Gives up (false) after limit_ns, recording MLA_ERR_TIMEOUT, or as
// soon as *abort is set (when abort is given).
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, const volatile int* abort = nullptr,
                                     uint64_t limit_ns = kTimeoutNs) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t n = 0;; ++n) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((n & 15u) == 15u) {
      if (abort && *abort) return false;
      const uint64_t now = ptx::globaltimer();
      if (t0 == 0) t0 = now;
      else if (now - t0 > limit_ns) { report(MLA_ERR_TIMEOUT); return false; }
    }
  }
}

// Tile (bx, by, bz): x = head * m_tiles + m_tile (then, with kTwo, the second problem's m-tiles),
// y = token block, z = K split. The tensor maps stay kernel parameters (TMA reads them from parameter
// space); the body is instantiated once with a single weight map, and once with a second one.
template <bool kTwo>
__device__ __forceinline__ void head_gemm_body(const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                                               const CUtensorMap& tm_w2, const Params p, const int bx,
                                               const int by, const int bz) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (p.M + kBM - 1) / kBM;
  const int msub = kTwo ? 1 : max(1, p.m_sub);
  const int cph = (m_tiles + msub - 1) / msub;      // CTAs per head
  const bool second = kTwo && bx >= p.H * cph;      // a CTA of the second problem
  const int h = second ? 0 : bx / cph;
  const int mc = second ? 0 : bx % cph;             // the CTA's place among its head's CTAs
  const int mt = second ? bx - p.H * cph : mc * msub;   // its first m-tile
  const int M = second ? p.M2 : p.M;
  const CUtensorMap* tw = second ? &tm_w2 : &tm_w;
  const int tok0 = by * p.tn;
  const int split = bz;
  const int kc0 = split * p.chunks_per_split;
  const int nk = max(0, min(p.K / kBK, kc0 + p.chunks_per_split) - kc0);
  const int S = p.stages;
  const uint32_t full0 = base, empty0 = base + 8u * kMaxStages, done = base + 16u * kMaxStages;
  const uint32_t slot = done + 8u;
  volatile int* abort = reinterpret_cast<volatile int*>(smem_raw + (done + 16u - raw));   // the issuer gave up
  const uint32_t ring = base + kBarBytes;
  const uint32_t sbytes = (uint32_t)stage_bytes(p.tn, msub);
  const uint32_t xoff = (uint32_t)(msub * kABytes);   // the token box after the weight boxes
  const uint32_t acc_cols = (uint32_t)(msub * p.tn);   // m-subtile j's accumulator: columns [j*tn, (j+1)*tn)
  const uint32_t tmem_cols = acc_cols <= 32 ? 32u : acc_cols <= 64 ? 64u : acc_cols <= 128 ? 128u : acc_cols <= 256 ? 256u : 512u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { ptx::mbar_init(full0 + 8u * s, 1); ptx::mbar_init(empty0 + 8u * s, 1); }
    ptx::mbar_init(done, 1);
    *abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(tw);
    ptx::prefetch_tmap(&tm_x);
  }
  if (warp == 2) { ptx::tmem_alloc(slot, tmem_cols); ptx::tmem_relinquish(); }
  // the rotated tail's inverse frequencies (one per pair) depend on no input: into shared memory now
  const bool rope_tail = p.rope_in != nullptr && !second;
  double* inv_freq = reinterpret_cast<double*>(smem_raw + (base + kInvFreqOff - raw));
  if (rope_tail && warp >= 4 && (int)threadIdx.x - 128 < p.d_r / 2)
    inv_freq[threadIdx.x - 128] = rope_inv_freq((int)threadIdx.x - 128, p.d_r, p.rope_base);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + (slot - raw));

  // per m-subtile, the two weight boxes (64 k x 64 features each) of K chunk i into stage st (a tile
  // past M reads the fill value: features are the inner coordinate of the MN-major weight map)
  auto load_w = [&](int i, uint32_t st, uint32_t fb) {
    const int kk = (kc0 + i) * kBK;
    for (int j = 0; j < msub; ++j) {
      const int m0 = (mt + j) * kBM;
      const uint32_t sj = st + (uint32_t)j * kABytes;
      if (p.a_kmajor) {   // rows m of W[h]ᵀ: two boxes of 64 rows x 64 k
        ptx::tma_load_2d(sj, tw, kk, h * M + m0, fb);
        ptx::tma_load_2d(sj + kABytes / 2, tw, kk, h * M + m0 + 64, fb);
      } else {
        ptx::tma_load_2d(sj, tw, m0, h * p.K + kk, fb);
        ptx::tma_load_2d(sj + kABytes / 2, tw, m0 + 64, h * p.K + kk, fb);
      }
    }
  };
  // Weights that no earlier kernel of the stream writes fill the ring's first two stages while that
  // kernel finishes; the token rows (and everything else) wait for it. (Two, not the whole ring: a
  // token box issued behind every stage's weights would hold back the first MMA.)
  const int pre = p.w_early ? min(min(nk, S), 2) : 0;
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < pre; ++i) {
      ptx::mbar_arrive_expect_tx(full0 + 8u * i, sbytes);
      load_w(i, ring + i * sbytes, full0 + 8u * i);
    }
  }
  grid_dependency_wait();   // the inputs may come from the previous kernel of the stream
  allow_dependents();

  if (warp == 0 && lane == 0) {
    // ---- TMA producer: per K chunk two weight boxes and one token box (64 tokens x 64 k)
    int i = 0;
    for (; i < nk; ++i) {
      const int s = i % S;
      const uint32_t st = ring + s * sbytes;
      if (i >= pre) {   // a pre-issued stage is on its first use: free
        if (!wait(empty0 + 8u * s, ((i / S) & 1u) ^ 1u, abort)) break;
        ptx::mbar_arrive_expect_tx(full0 + 8u * s, sbytes);
        load_w(i, st, full0 + 8u * s);
      }
      const int kk = (kc0 + i) * kBK;
      ptx::tma_load_2d(st + xoff, &tm_x, p.x_shared ? kk : h * p.K + kk, tok0, full0 + 8u * s);
    }
    // every load issued must land before the CTA may exit (waited for even after a give-up)
    for (int k = (i > S ? i - S : 0); k < i; ++k) wait(full0 + 8u * (k % S), (k / S) & 1u);
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer: M = 128, N = tn, four K = 16 steps per chunk (one thread: with two to four K
    // chunks per CTA at decode batch sizes, a warp-wide wait costs more than the issue rate gains)
    const uint32_t idesc = ptx::idesc_bf16_f32_ab(kBM, p.tn, !p.a_kmajor, false);
    bool live = true;
#ifdef MLA_TEST_HOOKS
    // phase 0 of `done` completes only through this warp's own commit below: nothing else can end the wait
    if (g_test_stall) live = wait(done, 0u, nullptr, 10000000ull);
#endif
    for (int i = 0; i < nk && live; ++i) {
      const int s = i % S;
      if (!wait(full0 + 8u * s, (i / S) & 1u)) { live = false; break; }
      {
        ptx::tc_fence_after();
        const uint32_t st = ring + s * sbytes;
        // A, MN-major: 8-row K groups 1024 B apart (SBO), the two 64-feature halves one box apart (LBO);
        // a K step of 16 moves 16 rows = 2048 B. A, K-major: 8-feature groups 1024 B apart (the two
        // 64-row boxes are contiguous); a K step moves 32 B inside the swizzle row.
        // B, K-major: 8-token groups 1024 B apart; a K step of 16 moves 32 B inside the swizzle row.
        const uint64_t a_step = p.a_kmajor ? 2u : (uint64_t)(2048 >> 4);
        const uint64_t bd = ptx::smem_desc_sw128(st + xoff, 16, 1024);
        for (int j = 0; j < msub; ++j) {
          const uint32_t sj = st + (uint32_t)j * kABytes;
          const uint64_t ad = p.a_kmajor ? ptx::smem_desc_sw128(sj, 16, 1024) : ptx::smem_desc_sw128(sj, kABytes / 2, 1024);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_ss(tmem + (uint32_t)(j * p.tn), ad + (uint64_t)k * a_step, bd + (uint64_t)(2 * k), idesc,
                        (i | k) ? 1u : 0u);
        }
        ptx::mma_commit(empty0 + 8u * s);
      }
    }
    if (!live) *abort = 1;   // the producer stops waiting for stages that will not be freed
    ptx::mma_commit(done);
  } else if (warp >= 4 && rope_tail) {
    {
      const int row = threadIdx.x - 128;
      // the rotated tail does not depend on the GEMM: done while the main loop runs, the token
      // block's tokens dealt out over the head's CTAs (token j of the block goes to CTA j % cph)
      const int half = p.d_r / 2;
      const int my_tok = (p.tn - mc + cph - 1) / cph;
      auto token = [&](int j) { return tok0 + j * cph + mc; };
      auto out_row = [&](int tok) { return p.y + (int64_t)tok * p.y_tok_stride + (int64_t)h * p.y_head_stride + p.M; };
      if (p.vec_out && (half & 3) == 0) {
        // four pairs (16 bytes) per item, four items per thread per round, all loads issued first
        const int quads = half / 4, items = my_tok * quads;
        for (int i0 = row; i0 < items; i0 += 4 * 128) {
          uint4 v[4];
          int tok[4], pos[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + 128 * u;
            tok[u] = i < items ? token(i / quads) : p.n_tok;
            const bool live = tok[u] < p.n_tok;
            const int g = i % quads;
            v[u] = live ? *reinterpret_cast<const uint4*>(p.rope_in + ((int64_t)tok[u] * p.H + h) * p.d_r + 8 * g)
                        : make_uint4(0u, 0u, 0u, 0u);
            pos[u] = live ? p.seqlens[tok[u] / p.s_q] - p.s_q + tok[u] % p.s_q : 0;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (tok[u] >= p.n_tok) continue;
            const int g = (i0 + 128 * u) % quads;
            __nv_bfloat162* x2 = reinterpret_cast<__nv_bfloat162*>(&v[u]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float cs, sn;
              rope_cos_sin_at_sfu(pos[u], inv_freq[4 * g + e], &cs, &sn);
              const float x0 = __low2float(x2[e]), x1 = __high2float(x2[e]);
              x2[e] = __floats2bfloat162_rn(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
            }
            *reinterpret_cast<uint4*>(out_row(tok[u]) + 8 * g) = v[u];
          }
        }
      } else {
        // one pair per item, four items per thread per round
        for (int i0 = row; i0 < my_tok * half; i0 += 4 * 128) {
          __nv_bfloat162 r2[4];
          int tok[4], q[4], pos[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + 128 * u;
            tok[u] = token(i / half);
            q[u] = i % half;
            const bool live = i < my_tok * half && tok[u] < p.n_tok;
            if (!live) tok[u] = -1;
            r2[u] = live ? *reinterpret_cast<const __nv_bfloat162*>(p.rope_in + ((int64_t)tok[u] * p.H + h) * p.d_r + 2 * q[u])
                         : __floats2bfloat162_rn(0.f, 0.f);
            pos[u] = live ? p.seqlens[tok[u] / p.s_q] - p.s_q + tok[u] % p.s_q : 0;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (tok[u] < 0) continue;
            float cs, sn;
            rope_cos_sin_at_sfu(pos[u], inv_freq[q[u]], &cs, &sn);
            const float x0 = __low2float(r2[u]), x1 = __high2float(r2[u]);
            *reinterpret_cast<__nv_bfloat162*>(out_row(tok[u]) + 2 * q[u]) =
                __floats2bfloat162_rn(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
          }
        }
      }
    }
  }
  // ---- epilogue: thread = output feature (TMEM lane (warp % 4) * 32 + lane), 32 tokens (TMEM
  // columns) per load. Warps 4-7 take the even m-subtiles; with two or more, warps 0-3 (their roles
  // done) take the odd ones.
  if (warp >= 4 || msub > 1) {
    __syncwarp();
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const bool ok = __all_sync(0xffffffffu, wait(done, 0));
    ptx::tc_fence_after();
    const int jstep = msub > 1 ? 2 : 1;
    for (int j = warp >= 4 ? 0 : 1; j < msub && ok; j += jstep) {
      const int mj = mt + j;                        // the m-tile of subtile j
      if (mj * kBM >= M) break;
      const uint32_t col0 = (uint32_t)(j * p.tn);   // its accumulator's first TMEM column
      const int m = mj * kBM + row;
      if (p.vec_out) {
        // 32 features (the warp's TMEM lanes) x 32 tokens at a time: each thread puts its feature's
        // values in column `lane` of a [token][feature] tile in shared memory (the ring, free once the
        // accumulator is done: 4 KB per warp), then the warp stores the tile's token rows in 16-byte
        // pieces (features are contiguous in every output; M and the strides are multiples of 8).
        uint8_t* tile = smem_raw + (ring - raw) + (uint32_t)(warp ^ 4) * 4096u;
        const uint32_t tile_s = ring + (uint32_t)(warp ^ 4) * 4096u;
        const int f0 = mj * kBM + (warp & 3) * 32;   // the warp's first feature
        const bool f32_out = !second && p.mode != 0;
        for (int c = 0; c < p.tn && tok0 + c < p.n_tok; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld32(tmem + lane_off + col0 + (uint32_t)c, r);
          ptx::tmem_wait_ld();
          const int kn = min(32, p.n_tok - tok0 - c);
          if (f32_out) {
  #pragma unroll
            for (int k = 0; k < 32; ++k)
              reinterpret_cast<float*>(tile)[k * 32 + lane] = nk > 0 ? __uint_as_float(r[k]) : 0.f;
          } else {
  #pragma unroll
            for (int k = 0; k < 32; ++k)
              reinterpret_cast<__nv_bfloat16*>(tile)[k * 32 + lane] = __float2bfloat16_rn(nk > 0 ? __uint_as_float(r[k]) : 0.f);
          }
          __syncwarp();
          const int pieces = f32_out ? 8 : 4;   // 16-byte pieces per 32-feature token row
          for (int i = lane; i < 32 * pieces; i += 32) {
            const int t = i / pieces, f = f0 + (i % pieces) * (f32_out ? 4 : 8);
            if (t >= kn || f >= M) continue;
            const uint4 v = ptx::ld_shared_v4(tile_s + (uint32_t)i * 16u);
            const int tok = tok0 + c + t;
            void* dst = second ? (void*)(p.y2 + (int64_t)tok * p.y2_tok_stride + f)
                      : p.mode == 0 ? (void*)(p.y + (int64_t)tok * p.y_tok_stride + (int64_t)h * p.y_head_stride + f)
                                    : (void*)(p.part + ((int64_t)split * p.n_tok + tok) * p.M + f);
            *reinterpret_cast<uint4*>(dst) = v;
          }
          __syncwarp();
        }
      } else {   // any other output layout: one value per store
        for (int c = 0; c < p.tn && tok0 + c < p.n_tok; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld32(tmem + lane_off + col0 + (uint32_t)c, r);
          ptx::tmem_wait_ld();
          if (m >= M) continue;
          const int kn = min(32, p.n_tok - tok0 - c);
  #pragma unroll
          for (int k = 0; k < 32; ++k) {
            if (k >= kn) break;
            const int tok = tok0 + c + k;
            const float v = nk > 0 ? __uint_as_float(r[k]) : 0.f;
            if (second)
              p.y2[(int64_t)tok * p.y2_tok_stride + m] = __float2bfloat16_rn(v);
            else if (p.mode == 0)
              p.y[(int64_t)tok * p.y_tok_stride + (int64_t)h * p.y_head_stride + m] = __float2bfloat16_rn(v);
            else
              p.part[((int64_t)split * p.n_tok + tok) * p.M + m] = v;
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, tmem_cols);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
head_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, const Params p) {
  head_gemm_body<false>(tm_w, tm_x, tm_w, p, blockIdx.x, blockIdx.y, blockIdx.z);
}

__global__ void __launch_bounds__(kThreads, 1)
head_gemm2_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_w2, const Params p) {
  head_gemm_body<true>(tm_w, tm_x, tm_w2, p, blockIdx.x, blockIdx.y, blockIdx.z);
}

// ---- host ----------------------------------------------------------------------------------------
// Shapes the kernel takes: K a multiple of 64 (whole chunks), M a multiple of 8 (16-byte weight rows).
inline bool supported(int K, int M) { return K > 0 && K % kBK == 0 && M > 0 && M % 8 == 0; }
// The rotated tail of the absorbed query keeps one inverse frequency per pair in the barrier area.
inline bool supported_rope(int d_r) { return d_r > 0 && d_r <= 128; }

inline int tokens_per_cta(int n_tok) { return n_tok <= 32 ? 32 : (n_tok <= 64 ? 64 : 128); }

// Split of K for mode 1: at most one CTA per SM (a CTA streaming a long K fills an SM's shared
// memory, so one more would start a second wave), every split non-empty. Returns the number of splits.
inline int plan_splits(int M, int K, int n_tok, int num_sms, int max_splits) {
  const int chunks = K / kBK;
  const int base = ((M + kBM - 1) / kBM) * ((n_tok + tokens_per_cta(n_tok) - 1) / tokens_per_cta(n_tok));
  int ks = std::max(1, std::min({num_sms / base, chunks, max_splits}));
  const int per = (chunks + ks - 1) / ks;
  return (chunks + per - 1) / per;
}

struct Problem {
  const void* w;             // [H * K, M] row-major bf16 (W[h] = rows h*K .. h*K + K - 1)
  const void* x;             // [n_tok, H * K] row-major bf16
  int H, K, M, n_tok;
  int splits;                // 1 for mode 0
  const void* w2 = nullptr;  // optional second weight [K, M2] (H = 1, mode 0; output p.y2)
  int M2 = 0;
  int num_sms = 0;           // SMs of the device (0: unknown)
  bool a_kmajor = false;     // w is [H * M, K] (each head's weight transposed), read K-major
  bool x_shared = false;     // x is [n_tok, K], the same row for every head
  int m_per_cta = 1;         // m-tiles per CTA (1..4; more than 1 needs MN-major weights, no w2)
};

constexpr int kSmemMax = 232448;   // 227 KB per CTA

// One problem ready to launch: its parameters with every derived field set, and its tensor maps.
struct Prepared {
  Params p;
  CUtensorMap tm_w, tm_x, tm_w2;
  int ctas;
};

// Checks the problem and fills `out` (ring depth at most max_stages); MLA_OK, or an error status.
inline int prepare(const Problem& pr, Params p, int max_stages, Prepared* out) {
  if (!supported(pr.K, pr.M) || pr.n_tok <= 0 || pr.H <= 0 || pr.splits <= 0) return MLA_ERR_UNSUPPORTED;
  const bool two = pr.w2 != nullptr;
  if ((pr.a_kmajor || pr.x_shared) && (two || p.rope_in != nullptr)) return MLA_ERR_UNSUPPORTED;
  p.a_kmajor = pr.a_kmajor ? 1 : 0;
  p.x_shared = pr.x_shared ? 1 : 0;
  if (two && (pr.H != 1 || pr.splits != 1 || p.mode != 0 || p.rope_in != nullptr || !p.y2 || !supported(pr.K, pr.M2)))
    return MLA_ERR_UNSUPPORTED;
  p.M = pr.M;
  p.M2 = two ? pr.M2 : 0;
  {
    auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (p.mode == 0)
      p.vec_out = a16(p.y) && p.y_tok_stride % 8 == 0 && p.y_head_stride % 8 == 0 &&
                  (!two || (a16(p.y2) && p.y2_tok_stride % 8 == 0)) ? 1 : 0;
    else
      p.vec_out = a16(p.part) && pr.M % 4 == 0 ? 1 : 0;
  }
  p.K = pr.K;
  p.n_tok = pr.n_tok;
  p.H = pr.H;
  p.tn = tokens_per_cta(pr.n_tok);
  const int m_tiles = (pr.M + kBM - 1) / kBM;
  if (pr.m_per_cta < 1 || pr.m_per_cta > 4 || (pr.m_per_cta > 1 && (two || pr.a_kmajor))) return MLA_ERR_UNSUPPORTED;
  p.m_sub = std::min({pr.m_per_cta, m_tiles, 512 / p.tn});   // the accumulators fit TMEM's 512 columns
  const int chunks = pr.K / kBK;
  p.chunks_per_split = (chunks + pr.splits - 1) / pr.splits;
  p.stages = std::max(1, std::min({max_stages, kMaxStages, p.chunks_per_split,
                                   (kSmemMax - 2048) / stage_bytes(p.tn, p.m_sub)}));
  p.gx = pr.H * ((m_tiles + p.m_sub - 1) / p.m_sub) + (two ? (pr.M2 + kBM - 1) / kBM : 0);
  p.gy = (pr.n_tok + p.tn - 1) / p.tn;
  p.gz = pr.splits;
  out->ctas = p.gx * p.gy * p.gz;
  if (pr.a_kmajor) {
    if (!tmap::make_bf16_sw128(&out->tm_w, pr.w, pr.K, (int64_t)pr.H * pr.M, pr.K, kBK)) return MLA_ERR_INVALID_ARG;
  } else if (!tmap::make_bf16_sw128(&out->tm_w, pr.w, pr.M, (int64_t)pr.H * pr.K, pr.M, kBK)) {
    return MLA_ERR_INVALID_ARG;
  }
  out->tm_w2 = out->tm_w;
  if (two && !tmap::make_bf16_sw128(&out->tm_w2, pr.w2, pr.M2, pr.K, pr.M2, kBK)) return MLA_ERR_INVALID_ARG;
  const int64_t x_cols = pr.x_shared ? (int64_t)pr.K : (int64_t)pr.H * pr.K;
  if (!tmap::make_bf16_sw128(&out->tm_x, pr.x, x_cols, pr.n_tok, x_cols, p.tn)) return MLA_ERR_INVALID_ARG;
  out->p = p;
  return MLA_OK;
}

// The kernels' shared-memory limit, raised once per device.
inline int set_attributes() {
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && attr_done[dev]) return MLA_OK;
  if (cudaFuncSetAttribute(head_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) != cudaSuccess ||
      cudaFuncSetAttribute(head_gemm2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (dev >= 0 && dev < 64) attr_done[dev] = true;
  return MLA_OK;
}

// Launches on `st`; returns MLA_OK, or an error status with nothing launched.
inline int run(const Problem& pr, Params p, cudaStream_t st) {
  Prepared a;
  int rc = prepare(pr, p, kMaxStages, &a);
  if (rc) return rc;
  // more CTAs than SMs: a ring that lets two CTAs share an SM keeps the whole grid in one wave
  if (pr.num_sms > 0 && a.ctas > pr.num_sms)
    a.p.stages = std::max(1, std::min(a.p.stages, (kSmemMax / 2 - 2048) / stage_bytes(a.p.tn, a.p.m_sub)));
  if ((rc = set_attributes())) return rc;
  const dim3 grid(a.p.gx, a.p.gy, a.p.gz);
  const size_t smem = (size_t)smem_bytes(a.p.tn, a.p.stages, a.p.m_sub);
  if (pr.w2 != nullptr)
    mla::launch_pdl(head_gemm2_kernel, grid, dim3(kThreads), smem, st, a.tm_w, a.tm_x, a.tm_w2, a.p);
  else
    mla::launch_pdl(head_gemm_kernel, grid, dim3(kThreads), smem, st, a.tm_w, a.tm_x, a.p);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace gemm
}  // namespace mla

// CUDA-core kernels (fp32 arithmetic) for every step of one decode step: the fp32 workloads run
// on them, and so does every shape the tensor-core kernels do not cover.
#pragma once

#include "common.cuh"

namespace mla {
namespace simt {

// =============================================================================================
// Dense projection z = x · W, split over K: part[ks][n][col] = sum_{k in slice ks} x[n][k] W[k][col].
// One thread per output column, PROJ_TOK tokens per block; W rows are read coalesced.
// With out != nullptr (and one slice) the result is written in storage type instead.
// =============================================================================================
constexpr int PROJ_COLS = 128;
constexpr int PROJ_TOK = 8;
constexpr int PROJ_KT = 64;

template <typename T>
__global__ void __launch_bounds__(PROJ_COLS)
proj_partial_kernel(const T* __restrict__ x, int n_tok, int K, const T* __restrict__ W, int N,
                    int k_chunk, float* __restrict__ part, T* __restrict__ out) {
  __shared__ float xs[PROJ_TOK][PROJ_KT];
  const int col = blockIdx.x * PROJ_COLS + threadIdx.x;
  const int tok0 = blockIdx.y * PROJ_TOK;
  const int ks = blockIdx.z;
  const int k_lo = ks * k_chunk;
  const int k_hi = min(K, k_lo + k_chunk);
  float acc[PROJ_TOK];
#pragma unroll
  for (int t = 0; t < PROJ_TOK; ++t) acc[t] = 0.f;
  for (int kb = k_lo; kb < k_hi; kb += PROJ_KT) {
    for (int i = threadIdx.x; i < PROJ_TOK * PROJ_KT; i += blockDim.x) {
      const int tt = i / PROJ_KT, kk = i % PROJ_KT;
      const int tok = tok0 + tt, k = kb + kk;
      xs[tt][kk] = (tok < n_tok && k < k_hi) ? ld(x + (int64_t)tok * K + k) : 0.f;
    }
    __syncthreads();
    if (col < N) {
      const int kn = min(PROJ_KT, k_hi - kb);
      for (int kk = 0; kk < kn; ++kk) {
        const float w = ld(W + (int64_t)(kb + kk) * N + col);
#pragma unroll
        for (int t = 0; t < PROJ_TOK; ++t) acc[t] = fmaf(xs[t][kk], w, acc[t]);
      }
    }
    __syncthreads();
  }
  if (col >= N) return;
#pragma unroll
  for (int t = 0; t < PROJ_TOK; ++t) {
    const int tok = tok0 + t;
    if (tok >= n_tok) break;
    if (out) st(out + (int64_t)tok * N + col, acc[t]);
    else part[((int64_t)ks * n_tok + tok) * N + col] = acc[t];
  }
}

// Sum of the K slices of one output column: slice ks of the column is src[ks * step]; 32 loads
// are in flight together.
__device__ __forceinline__ float sum_slices(const float* src, int ksplit, int64_t step) {
  float s = 0.f;
  for (int ks = 0; ks < ksplit; ks += 32) {
    float v[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = (ks + k < ksplit) ? src[(ks + k) * step] : 0.f;
#pragma unroll
    for (int k = 0; k < 32; k += 4) s += (v[k] + v[k + 1]) + (v[k + 2] + v[k + 3]);
  }
  return s;
}

// =============================================================================================
// a1 epilogue: sum the K slices, RMSNorm the latent part, rotate the RoPE part, store the row.
// One block per new token. With groups > 0 (N % 4 == 0, 16-byte aligned slices; blockDim.x =
// L + 32 where L = groups * N/4 rounded up to a warp; dynamic shared memory (1 + groups) * N + d_r
// floats) the first groups * N/4 threads read the slices in 16-byte pieces: thread (g, q) sums
// columns 4q..4q+3 over slices g, g + groups, ... (all of its loads in flight together), and the
// groups' sums are then added in a fixed order; meanwhile the last warp finds the token's cache row
// and the rotation's cos/sin, so that no dependent load is left after the sums. With groups == 0 a
// thread per column sums that column's slices and the row is found afterwards. The latent row is
// written 16 bytes at a time. With latent_by_token the latent row of token tok goes to latent + tok *
// lat_stride (a plain buffer) instead of its cache slot; the RoPE key always goes to its cache slot.
// =============================================================================================
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int n = 4;
  static __device__ __forceinline__ void store(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int n = 8;
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* v) {
    uint4 u;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]), h3 = __floats2bfloat162_rn(v[6], v[7]);
    u.x = *reinterpret_cast<uint32_t*>(&h0);
    u.y = *reinterpret_cast<uint32_t*>(&h1);
    u.z = *reinterpret_cast<uint32_t*>(&h2);
    u.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(p) = u;
  }
};

// threads of the slice readers in the groups > 0 layout (the place-finding warp follows them)
__host__ __device__ inline int finish_readers(int N, int groups) { return (groups * (N / 4) + 31) / 32 * 32; }

template <typename T>
__global__ void append_finish_kernel(const float* __restrict__ part, int ksplit, int n_tok, int s_q,
                                     int d_c, int d_r, const T* __restrict__ gamma, float eps,
                                     float rope_base, const int32_t* __restrict__ seqlens,
                                     const int32_t* __restrict__ block_table, int max_pages,
                                     T* latent, int64_t lat_stride, T* rope, int64_t rope_stride,
                                     int num_pages, int latent_by_token, int groups) {
  extern __shared__ float z[];
  __shared__ float red[32];
  __shared__ long long s_row;   // the token's cache row; -1: none (reported)
  __shared__ int s_pos;
  grid_dependency_wait();   // launched with programmatic dependent launch after the projection
  allow_dependents();
  const int tok = blockIdx.x;
  const int b = tok / s_q, t = tok % s_q;
  const int N = d_c + d_r, half = d_r / 2;
  float* cs_sn = z + (1 + groups) * N;   // groups > 0: cos, sin of pair i at [2i], [2i + 1]
  if (groups > 0) {
    const int Q = N / 4, readers = finish_readers(N, groups);
    float* acc = z + N;   // [groups][N]
    if ((int)threadIdx.x >= readers) {
      // the place-finding warp: position, cache row, then the rotation of every pair
      const int lane = threadIdx.x - readers;
      int pos = 0;
      if (lane == 0) {
        long long row = -1;
        pos = seqlens[b] - s_q + t;
        if (pos < 0 || (pos >> 6) >= max_pages) report(MLA_ERR_DEVICE_CHECK);
        else row = cache_row(block_table + (int64_t)b * max_pages, pos, num_pages);
        s_row = row;
        s_pos = pos;
      }
      pos = __shfl_sync(0xffffffffu, pos, 0);
      for (int i = lane; i < half; i += 32) rope_cos_sin(pos, i, d_r, rope_base, &cs_sn[2 * i], &cs_sn[2 * i + 1]);
    } else if ((int)threadIdx.x < groups * Q) {
      const int q = threadIdx.x % Q, g = threadIdx.x / Q;
      const float4* src = reinterpret_cast<const float4*>(part + (int64_t)tok * N) + q;
      const int64_t step = (int64_t)n_tok * Q;   // one slice, in float4
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = g; s0 < ksplit; s0 += 8 * groups) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int sl = s0 + u * groups;
          v[u] = sl < ksplit ? __ldcg(src + sl * step) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) { a.x += v[u].x; a.y += v[u].y; a.z += v[u].z; a.w += v[u].w; }
      }
      reinterpret_cast<float4*>(acc + g * N)[q] = a;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      float v = 0.f;
      for (int g = 0; g < groups; ++g) v += acc[g * N + i];
      z[i] = v;
    }
  } else {
    // one column per thread, up to 32 slices' loads in flight per thread
    for (int i = threadIdx.x; i < N; i += blockDim.x)
      z[i] = sum_slices(part + (int64_t)tok * N + i, ksplit, (int64_t)n_tok * N);
    if (threadIdx.x == 0) {
      long long row = -1;
      const int pos = seqlens[b] - s_q + t;
      if (pos < 0 || (pos >> 6) >= max_pages) report(MLA_ERR_DEVICE_CHECK);
      else row = cache_row(block_table + (int64_t)b * max_pages, pos, num_pages);
      s_row = row;
      s_pos = pos;
    }
  }
  __syncthreads();
  float ss = 0.f;
  for (int i = threadIdx.x; i < d_c; i += blockDim.x) ss = fmaf(z[i], z[i], ss);
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)d_c + eps);
  const int64_t row = s_row;
  const int pos = s_pos;
  if (row < 0) return;
  T* lrow = latent + (latent_by_token ? (int64_t)tok : row) * lat_stride;
  constexpr int V = Vec16<T>::n;
  if (d_c % V == 0) {   // row starts are 16-byte aligned (aligned base, stride a multiple of 16 bytes)
    for (int i = threadIdx.x * V; i < d_c; i += blockDim.x * V) {
      float v[V];
#pragma unroll
      for (int u = 0; u < V; ++u) v[u] = z[i + u] * inv * (gamma ? ld(gamma + i + u) : 1.f);
      Vec16<T>::store(lrow + i, v);
    }
  } else {
    for (int i = threadIdx.x; i < d_c; i += blockDim.x) st(lrow + i, z[i] * inv * (gamma ? ld(gamma + i) : 1.f));
  }
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    float cs, sn;
    if (groups > 0) {
      cs = cs_sn[2 * i];
      sn = cs_sn[2 * i + 1];
    } else {
      rope_cos_sin(pos, i, d_r, rope_base, &cs, &sn);
    }
    const float a = z[d_c + 2 * i], bb = z[d_c + 2 * i + 1];
    st(rope + row * rope_stride + 2 * i, a * cs - bb * sn);
    st(rope + row * rope_stride + 2 * i + 1, a * sn + bb * cs);
  }
}

// =============================================================================================
// f3 epilogue of the expanded (GQA) cache append: token tok's expanded keys [g*D] and values
// [g*d_v], computed into plain buffers, copied into the cache rows of its position, 16 bytes at a
// time (row widths are multiples of 16 bytes). One block per new token.
// =============================================================================================
template <typename T>
__global__ void gqa_scatter_kernel(const T* __restrict__ kbuf, const T* __restrict__ vbuf, int s_q, int kw, int vw,
                                   const int32_t* __restrict__ seqlens, const int32_t* __restrict__ block_table,
                                   int max_pages, int num_pages, T* k, int64_t k_stride, T* v, int64_t v_stride) {
  grid_dependency_wait();
  allow_dependents();
  const int tok = blockIdx.x;
  const int b = tok / s_q, t = tok % s_q;
  const int pos = seqlens[b] - s_q + t;
  if (pos < 0 || (pos >> 6) >= max_pages) {
    if (threadIdx.x == 0) report(MLA_ERR_DEVICE_CHECK);
    return;
  }
  const int64_t row = cache_row(block_table + (int64_t)b * max_pages, pos, num_pages);
  if (row < 0) return;
  const uint4* ks = reinterpret_cast<const uint4*>(kbuf + (int64_t)tok * kw);
  const uint4* vs = reinterpret_cast<const uint4*>(vbuf + (int64_t)tok * vw);
  uint4* kd = reinterpret_cast<uint4*>(k + row * k_stride);
  uint4* vd = reinterpret_cast<uint4*>(v + row * v_stride);
  const int nk = kw * (int)sizeof(T) / 16, nv = vw * (int)sizeof(T) / 16;
  for (int i = threadIdx.x; i < nk; i += blockDim.x) kd[i] = ks[i];
  for (int i = threadIdx.x; i < nv; i += blockDim.x) vd[i] = vs[i];
}

// =============================================================================================
// Sum of K slices: out[tok, m] = sum_s part[s, tok, m], stored in T (split-K GEMM epilogue).
// Four columns per thread (M a multiple of 4), one block row of tokens per blockIdx.y.
// =============================================================================================
template <typename T>
__global__ void reduce_slices_kernel(const float* __restrict__ part, int ksplit, int n_tok, int M, T* out,
                                     int64_t out_stride) {
  grid_dependency_wait();
  allow_dependents();
  const int tok = blockIdx.y;
  const int i4 = blockIdx.x * blockDim.x + threadIdx.x;
  if (i4 >= M / 4) return;
  const float4* src = reinterpret_cast<const float4*>(part + (int64_t)tok * M) + i4;
  const int64_t step4 = (int64_t)n_tok * M / 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < ksplit; ++s) {
    const float4 v = src[s * step4];
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  T* o = out + (int64_t)tok * out_stride + 4 * i4;
  st(o, acc.x); st(o + 1, acc.y); st(o + 2, acc.z); st(o + 3, acc.w);
}

// =============================================================================================
// Query chain, middle step: c_q = RMSNorm(sum of the K slices of x·W_DQ) · gamma_q, one row of N
// values per token, stored in T. One block per token. With groups > 0 (N % 4 == 0, 16-byte aligned
// slices, blockDim.x >= groups * N/4, dynamic shared memory (1 + groups) * N floats) thread (g, q)
// sums columns 4q..4q+3 over slices g, g + groups, ... with all of its loads in flight, and the
// groups' sums are added in a fixed order; with groups == 0 a thread per column sums its slices.
// Rows of N % 8 == 0 bf16 values (or N % 4 fp32) are stored 16 bytes at a time.
// =============================================================================================
constexpr int RMS_THREADS = 1024;

template <typename T>
__global__ void __launch_bounds__(RMS_THREADS) rms_rows_kernel(const float* __restrict__ part, int ksplit, int n_tok, int N,
                                const T* __restrict__ gamma, float eps, T* __restrict__ out, int groups) {
  extern __shared__ float z[];
  __shared__ float red[32];
  grid_dependency_wait();   // launched with programmatic dependent launch after the projection
  allow_dependents();
  const int tok = blockIdx.x;
  if (groups > 0) {
    const int Q = N / 4;
    float* acc = z + N;   // [groups][N]
    if ((int)threadIdx.x < groups * Q) {
      const int q = threadIdx.x % Q, g = threadIdx.x / Q;
      const float4* src = reinterpret_cast<const float4*>(part + (int64_t)tok * N) + q;
      const int64_t step = (int64_t)n_tok * Q;   // one slice, in float4
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = g; s0 < ksplit; s0 += 8 * groups) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int sl = s0 + u * groups;
          v[u] = sl < ksplit ? __ldcg(src + sl * step) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) { a.x += v[u].x; a.y += v[u].y; a.z += v[u].z; a.w += v[u].w; }
      }
      reinterpret_cast<float4*>(acc + g * N)[q] = a;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      float v = 0.f;
      for (int g = 0; g < groups; ++g) v += acc[g * N + i];
      z[i] = v;
    }
  } else {
    for (int i = threadIdx.x; i < N; i += blockDim.x)
      z[i] = sum_slices(part + (int64_t)tok * N + i, ksplit, (int64_t)n_tok * N);
  }
  __syncthreads();
  float ss = 0.f;
  for (int i = threadIdx.x; i < N; i += blockDim.x) ss = fmaf(z[i], z[i], ss);
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)N + eps);
  T* row = out + (int64_t)tok * N;
  constexpr int V = Vec16<T>::n;
  if (N % V == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0) {
    for (int i = threadIdx.x * V; i < N; i += blockDim.x * V) {
      float v[V];
#pragma unroll
      for (int u = 0; u < V; ++u) v[u] = z[i + u] * inv * (gamma ? ld(gamma + i + u) : 1.f);
      Vec16<T>::store(row + i, v);
    }
  } else {
    for (int i = threadIdx.x; i < N; i += blockDim.x) st(row + i, z[i] * inv * (gamma ? ld(gamma + i) : 1.f));
  }
}

// =============================================================================================
// Per-head small GEMM: y[tok, h, :] = a[tok, h, :] · Wh[h]   (a row K wide, Wh[h] is [K, N]).
// Used for a2 (a = q_nope, W = W_UK, N = d_c) and a5 (a = o_lat, W = W_UV, N = d_v).
// Optional RoPE tail for a2: y[tok, h, N + 2i..] = RoPE(r[tok, h, :], pos).
// =============================================================================================
constexpr int HG_TOK = 8;

template <typename T>
__global__ void __launch_bounds__(128)
head_gemm_kernel(const T* __restrict__ a, int64_t a_head_stride, int K, const T* __restrict__ Wh,
                 int N, int n_tok, int H, T* __restrict__ y, int64_t y_head_stride,
                 const T* __restrict__ rope_raw, int d_r, const int32_t* __restrict__ seqlens,
                 int s_q, float rope_base) {
  extern __shared__ float as[];  // [HG_TOK][K]
  const int h = blockIdx.x;
  const int tok0 = blockIdx.y * HG_TOK;
  for (int i = threadIdx.x; i < HG_TOK * K; i += blockDim.x) {
    const int tt = i / K, k = i % K;
    const int tok = tok0 + tt;
    as[i] = (tok < n_tok) ? ld(a + ((int64_t)tok * H + h) * a_head_stride + k) : 0.f;
  }
  __syncthreads();
  const T* W = Wh + (int64_t)h * K * N;
  for (int c = threadIdx.x; c < N; c += blockDim.x) {
    float acc[HG_TOK];
#pragma unroll
    for (int t = 0; t < HG_TOK; ++t) acc[t] = 0.f;
    for (int k = 0; k < K; ++k) {
      const float w = ld(W + (int64_t)k * N + c);
#pragma unroll
      for (int t = 0; t < HG_TOK; ++t) acc[t] = fmaf(as[t * K + k], w, acc[t]);
    }
#pragma unroll
    for (int t = 0; t < HG_TOK; ++t) {
      const int tok = tok0 + t;
      if (tok < n_tok) st(y + ((int64_t)tok * H + h) * y_head_stride + c, acc[t]);
    }
  }
  if (rope_raw == nullptr) return;
  const int half = d_r / 2;
  for (int i = threadIdx.x; i < HG_TOK * half; i += blockDim.x) {
    const int tt = i / half, p = i % half;
    const int tok = tok0 + tt;
    if (tok >= n_tok) continue;
    const int pos = seqlens[tok / s_q] - s_q + tok % s_q;
    float cs, sn;
    rope_cos_sin(pos, p, d_r, rope_base, &cs, &sn);
    const T* r = rope_raw + ((int64_t)tok * H + h) * d_r;
    const float x0 = ld(r + 2 * p), x1 = ld(r + 2 * p + 1);
    T* o = y + ((int64_t)tok * H + h) * y_head_stride + N;
    st(o + 2 * p, x0 * cs - x1 * sn);
    st(o + 2 * p + 1, x0 * sn + x1 * cs);
  }
}

// =============================================================================================
// a3 / a6: split-KV flash-decoding on CUDA cores, generic over the absorbed and grouped paths.
// Key of row j = [kpart_j (Dk) ; rope_j (d_r)], value = vpart_j (Dv). For the absorbed path
// kpart and vpart are the same latent row (Dk = Dv = d_c) and the query is q_abs; for the grouped
// path they are the group's K and V rows and the query's RoPE part is rotated here.
// Block = 8 heads (one warp each) x 32 positions per tile; online softmax per head.
// =============================================================================================
constexpr int DEC_HEADS = 8;
constexpr int DEC_TILE = 32;
constexpr int DEC_MAX_OV = 16;  // Dv <= 512

struct DecodeArgs {
  const void* q;           // [n_tok, H, q_head_stride]: Dk query part, then d_r RoPE part (absorbed)
  int64_t q_head_stride;
  const void* q_rope_raw;  // grouped path: [n_tok, H, d_r] un-rotated; nullptr for absorbed
  const void* kpart; int64_t k_stride; int64_t k_group_off;
  const float* kscale;     // 8-bit latent cache: kpart holds E4M3 codes (k_stride in bytes), one fp32
                           // scale per row here; nullptr for a dtype cache
  const void* vpart; int64_t v_stride; int64_t v_group_off;
  const void* rope; int64_t rope_stride;
  int Dk, Dv, d_r, H, heads_per_group;
  int kv_shared;           // vpart rows are the kpart rows (absorbed)
  const int32_t* block_table; int max_pages; int num_pages;
  const int32_t* seqlens; int s_q;
  float sm_scale, rope_base;
  void* out; int64_t out_head_stride; float* lse;
  float* part_o; float* part_lse; int nsplit; int chunk;
};

// Value of an E4M3 code from the format's definition: sign, exponent field e (bias 7), mantissa m;
// (1 + m/8) * 2^(e-7) for e >= 1 (written straight into fp32's fields), m * 2^-9 for e = 0, NaN for
// e = 15, m = 7.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
  if (e == 15u && m == 7u) v = __uint_as_float(0x7fc00000u);
  return (c & 0x80u) ? -v : v;
}

// =============================================================================================
// f4 on the tensor cores, first pass: the pages a decode reads, dequantised into a dense bf16
// scratch. Block (p, b) takes page p of sequence b (p below the sequence's tile count): latent row r
// becomes s_r · value(code) rounded once to bf16 (value from the E4M3 table above), the RoPE key is
// copied; dense_table[b][p] = b * max_pages + p names the scratch page, for the decode that follows.
// A page id outside the pool is reported and its rows are zeros. d_c % 16 == 0, d_r % 8 == 0.
// =============================================================================================
__global__ void __launch_bounds__(256)
dequant_pages_kernel(const uint8_t* __restrict__ codes, int64_t code_stride, const float* __restrict__ scales,
                     const __nv_bfloat16* __restrict__ rope, int64_t rope_stride, int num_pages,
                     const int32_t* __restrict__ seqlens, const int32_t* __restrict__ block_table, int max_pages,
                     int d_c, int d_r, __nv_bfloat16* __restrict__ lat_out, __nv_bfloat16* __restrict__ rope_out,
                     int32_t* __restrict__ dense_table) {
  __shared__ float lut[256];
  grid_dependency_wait();   // the inputs may come from the previous kernel of the stream
  allow_dependents();
  lut[threadIdx.x] = e4m3_value(threadIdx.x);   // 256 threads, one code each
  const int p = blockIdx.x, b = blockIdx.y;
  if (threadIdx.x == 0) dense_table[(int64_t)b * max_pages + p] = b * max_pages + p;
  const int L = seqlens[b];
  const int tiles = L > 0 ? min((L + 63) / 64, max_pages) : 0;
  __syncthreads();
  if (p >= tiles) return;
  const int page = block_table[(int64_t)b * max_pages + p];
  const bool ok = page >= 0 && page < num_pages;
  if (!ok && threadIdx.x == 0) report(MLA_ERR_DEVICE_CHECK);
  const int64_t dst0 = ((int64_t)b * max_pages + p) * 64;
  const int per_row = d_c / 16;
  for (int i = threadIdx.x; i < 64 * per_row; i += blockDim.x) {
    const int r = i / per_row, c = i % per_row;
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (ok) {
      const int64_t src = (int64_t)page * 64 + r;
      const uint4 v = *reinterpret_cast<const uint4*>(codes + src * code_stride + 16 * c);
      const float sc = scales[src];
      const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t word = q[k >> 1] >> (16 * (k & 1));
        const __nv_bfloat162 h = __floats2bfloat162_rn(lut[word & 0xffu] * sc, lut[(word >> 8) & 0xffu] * sc);
        w[k] = *reinterpret_cast<const uint32_t*>(&h);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(lat_out + (dst0 + r) * d_c + 16 * c);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  const int per_rope = d_r / 8;
  for (int i = threadIdx.x; i < 64 * per_rope; i += blockDim.x) {
    const int r = i / per_rope, c = i % per_rope;
    const uint4 v = ok ? *reinterpret_cast<const uint4*>(rope + ((int64_t)page * 64 + r) * rope_stride + 8 * c)
                       : make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(rope_out + (dst0 + r) * d_r + 8 * c) = v;
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
decode_simt_kernel(DecodeArgs A) {
  extern __shared__ float sm[];
  __shared__ float lut[256];   // E4M3 code -> value, for an 8-bit latent cache
  const int W = A.Dk + A.d_r;
  const int WP = W + 1;  // padded key row: conflict-free column reads
  float* qs = sm;                              // [8][W]
  float* ks = qs + DEC_HEADS * W;              // [32][WP]
  float* vs = A.kv_shared ? ks : ks + DEC_TILE * WP;   // [32][Dv] (or aliases ks)
  float* ps = ks + DEC_TILE * WP + (A.kv_shared ? 0 : DEC_TILE * A.Dv);  // [8][32]
  int64_t* rows = reinterpret_cast<int64_t*>(ps + DEC_HEADS * DEC_TILE);  // [32]
  float* rscale = reinterpret_cast<float*>(rows + DEC_TILE);             // [32] (8-bit cache)
  const bool fp8 = A.kscale != nullptr;
  if (fp8) lut[threadIdx.x] = e4m3_value(threadIdx.x);   // 256 threads, one code each

  const int tok = blockIdx.x;
  const int h0 = blockIdx.y * DEC_HEADS;
  const int split = blockIdx.z;
  const int b = tok / A.s_q, t = tok % A.s_q;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = h0 + warp;
  const int grp = h0 / A.heads_per_group;      // all 8 heads of a block share one group
  const int L = A.seqlens[b];
  const int n_vis = L - A.s_q + t + 1;
  const int lo = split * A.chunk;
  const int hi = min(n_vis, lo + A.chunk);
  const int32_t* table = A.block_table + (int64_t)b * A.max_pages;
  if (n_vis < 1 || (L > 0 && ((L - 1) >> 6) >= A.max_pages)) {
    if (threadIdx.x == 0 && split == 0 && blockIdx.y == 0) report(MLA_ERR_DEVICE_CHECK);
    return;
  }

  // query rows of the 8 heads (fp32), RoPE part rotated here for the grouped path
  const T* q = reinterpret_cast<const T*>(A.q);
  for (int i = threadIdx.x; i < DEC_HEADS * W; i += blockDim.x) {
    const int hh = i / W, d = i % W;
    const int64_t base = ((int64_t)tok * A.H + h0 + hh) * A.q_head_stride;
    if (A.q_rope_raw == nullptr || d < A.Dk) {
      qs[i] = ld(q + base + d);
    } else {
      const int p = (d - A.Dk) >> 1;
      const T* r = reinterpret_cast<const T*>(A.q_rope_raw) + ((int64_t)tok * A.H + h0 + hh) * A.d_r;
      float cs, sn;
      rope_cos_sin(L - A.s_q + t, p, A.d_r, A.rope_base, &cs, &sn);
      const float x0 = ld(r + 2 * p), x1 = ld(r + 2 * p + 1);
      qs[i] = ((d - A.Dk) & 1) ? (x0 * sn + x1 * cs) : (x0 * cs - x1 * sn);
    }
  }

  const int nov = A.Dv / 32;
  float o[DEC_MAX_OV];
#pragma unroll
  for (int k = 0; k < DEC_MAX_OV; ++k) o[k] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const T* kp = reinterpret_cast<const T*>(A.kpart);
  const T* vp = reinterpret_cast<const T*>(A.vpart);
  const T* rp = reinterpret_cast<const T*>(A.rope);

  for (int p0 = lo; p0 < hi; p0 += DEC_TILE) {
    __syncthreads();
    if (threadIdx.x < DEC_TILE) {
      const int p = p0 + threadIdx.x;
      const int64_t row = (p < hi) ? cache_row(table, p, A.num_pages) : -1;
      rows[threadIdx.x] = row;
      if (fp8) rscale[threadIdx.x] = row >= 0 ? A.kscale[row] : 0.f;
    }
    __syncthreads();
    const uint8_t* k8 = reinterpret_cast<const uint8_t*>(A.kpart);
    for (int i = threadIdx.x; i < DEC_TILE * W; i += blockDim.x) {
      const int r = i / W, d = i % W;
      const int64_t row = rows[r];
      float v = 0.f;
      if (row >= 0) {
        if (d >= A.Dk) v = ld(rp + row * A.rope_stride + (d - A.Dk));
        else if (fp8) v = lut[k8[row * A.k_stride + d]] * rscale[r];   // the dequantised latent
        else v = ld(kp + row * A.k_stride + grp * A.k_group_off + d);
      }
      ks[r * WP + d] = v;
    }
    if (!A.kv_shared) {
      for (int i = threadIdx.x; i < DEC_TILE * A.Dv; i += blockDim.x) {
        const int r = i / A.Dv, d = i % A.Dv;
        const int64_t row = rows[r];
        vs[i] = (row >= 0) ? ld(vp + row * A.v_stride + grp * A.v_group_off + d) : 0.f;
      }
    }
    __syncthreads();
    // score of (head = warp, position = lane)
    float s = -INFINITY;
    if (rows[lane] >= 0) {
      const float* qh = qs + warp * W;
      const float* kr = ks + lane * WP;
      float acc = 0.f;
      for (int d = 0; d < W; ++d) acc = fmaf(qh[d], kr[d], acc);
      s = acc * A.sm_scale;
    }
    const float m_tile = warp_max(s);
    const float m_new = fmaxf(m_run, m_tile);
    const float alpha = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
    const float pj = (s == -INFINITY) ? 0.f : expf(s - m_new);
    l_run = l_run * alpha + warp_sum(pj);
    m_run = m_new;
    ps[warp * DEC_TILE + lane] = pj;
    __syncwarp();
    const int vstride = A.kv_shared ? WP : A.Dv;
#pragma unroll
    for (int k = 0; k < DEC_MAX_OV; ++k) {
      if (k < nov) {
        float acc = o[k] * alpha;
        const int d = lane + 32 * k;
        for (int j = 0; j < DEC_TILE; ++j) acc = fmaf(ps[warp * DEC_TILE + j], vs[j * vstride + d], acc);
        o[k] = acc;
      }
    }
  }

  const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
  const float lse = (l_run > 0.f) ? m_run + logf(l_run) : -INFINITY;
  if (A.nsplit == 1) {
    T* out = reinterpret_cast<T*>(A.out) + ((int64_t)tok * A.H + h) * A.out_head_stride;
#pragma unroll
    for (int k = 0; k < DEC_MAX_OV; ++k)
      if (k < nov) st(out + lane + 32 * k, o[k] * inv_l);
    if (lane == 0) A.lse[(int64_t)tok * A.H + h] = lse;
  } else {
    const int64_t slot = ((int64_t)tok * A.H + h) * A.nsplit + split;
    float* po = A.part_o + slot * A.Dv;
#pragma unroll
    for (int k = 0; k < DEC_MAX_OV; ++k)
      if (k < nov) po[lane + 32 * k] = o[k] * inv_l;
    if (lane == 0) A.part_lse[slot] = lse;
  }
}

// 8-bit latent cache: row j of `lat` becomes the E4M3 codes of c_j / s_j, s_j = max|c_j| / 448 (both
// in fp32, each operation rounded once; round to nearest, ties to even, saturated at 448 by the
// conversion instruction; a zero magnitude is stored as +0). One warp per row, 8 rows per block.
template <typename T>
__global__ void __launch_bounds__(256)
quantize_e4m3_kernel(const T* __restrict__ lat, int64_t lat_stride, int64_t rows, int d_c, uint8_t* __restrict__ codes,
                     int64_t code_stride, float* __restrict__ scales) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T* src = lat + row * lat_stride;
  float amax = 0.f;
  for (int i = lane; i < d_c; i += 32) amax = fmaxf(amax, fabsf(ld(src + i)));
  amax = warp_max(amax);
  const float s = __fdiv_rn(amax, 448.f);
  const float safe = s > 0.f ? s : 1.f;
  uint8_t* dst = codes + row * code_stride;
  for (int i = 2 * lane; i < d_c; i += 64) {
    const float a = __fdiv_rn(ld(src + i), safe), b = __fdiv_rn(ld(src + i + 1), safe);
    uint16_t pr;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(b), "f"(a));   // a -> low byte
    uint32_t lo = pr & 0xffu, hi = pr >> 8;
    if ((lo & 0x7fu) == 0u) lo = 0u;   // -0 -> +0
    if ((hi & 0x7fu) == 0u) hi = 0u;
    *reinterpret_cast<uint16_t*>(dst + i) = (uint16_t)(lo | (hi << 8));
  }
  if (lane == 0) scales[row] = s;
}

// a4: combine the split partials of every (token, head): weights exp(lse_s - LSE).
template <typename T>
__global__ void merge_splits_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                    int nsplit, int Dv, T* __restrict__ out, int64_t out_head_stride,
                                    float* __restrict__ lse_out) {
  const int64_t th = blockIdx.x;  // token * H + head
  const float* pl = part_lse + th * nsplit;
  float m = -INFINITY;
  for (int s = 0; s < nsplit; ++s) m = fmaxf(m, pl[s]);
  float tot = 0.f;
  for (int s = 0; s < nsplit; ++s) tot += (pl[s] == -INFINITY) ? 0.f : expf(pl[s] - m);
  const float inv = 1.f / tot;
  for (int d = threadIdx.x; d < Dv; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      if (pl[s] == -INFINITY) continue;
      acc = fmaf(expf(pl[s] - m), part_o[(th * nsplit + s) * Dv + d], acc);
    }
    st(out + th * out_head_stride + d, acc * inv);
  }
  if (threadIdx.x == 0) lse_out[th] = m + logf(tot);
}

}  // namespace simt
}  // namespace mla

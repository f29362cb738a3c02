// Host entry points of libmla: argument validation, kernel selection by dtype and shape, launch.
// Nothing here allocates, frees or synchronises (except mla_check_status, which reads the
// device status word after synchronising the stream it is given).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <algorithm>
#include <mutex>

#include "mla.h"
#include "common.cuh"
#include "simt.cuh"
#include "decode_sm100.cuh"
#include "gemm_sm100.cuh"
#include "gqla_sm100.cuh"

namespace {

using mla::simt::DecodeArgs;

constexpr int kMaxDevices = 64;

using mla::launch;

int num_sms() {
  static int cached[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t esize(int32_t dtype) { return dtype == MLA_F32 ? 4 : 2; }
inline bool stride_ok(int64_t stride, int32_t dtype, int64_t min_elems) {
  return stride >= min_elems && ((stride * (int64_t)esize(dtype)) % 16) == 0;
}

int check_dims(const mla_dims_t* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->H <= 0 || d->D <= 0 || d->d_r <= 0 || (d->d_r & 1) || d->d_c <= 0 || d->d_v <= 0)
    return MLA_ERR_INVALID_ARG;
  if (d->page_size != 64) return MLA_ERR_INVALID_ARG;
  if (!(d->sm_scale >= 0.f) || !(d->rms_eps >= 0.f) || !(d->rope_base > 0.f)) return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

// The score scale a call uses: dims->sm_scale, or 1/sqrt(D + d_r) when it is 0.
float score_scale(const mla_dims_t* d) {
  return d->sm_scale > 0.f ? d->sm_scale : (float)(1.0 / sqrt((double)d->D + (double)d->d_r));
}
mla_dims_t with_scale(const mla_dims_t* d) {
  mla_dims_t r = *d;
  r.sm_scale = score_scale(d);
  return r;
}

// Token counts are formed as B * s_q in 32 bits; a product past INT32_MAX is an invalid argument.
bool tokens_ok(int32_t B, int32_t s_q) { return B > 0 && s_q > 0 && (int64_t)B * s_q <= INT32_MAX; }

int check_dtype(int32_t dtype) { return (dtype == MLA_F32 || dtype == MLA_BF16) ? MLA_OK : MLA_ERR_INVALID_ARG; }

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

template <typename K>
int set_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return MLA_OK;
  if (bytes > 227 * 1024) return MLA_ERR_UNSUPPORTED;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess
             ? MLA_OK : MLA_ERR_CUDA;
}

// ---- a1 split-K choice: enough blocks to cover the SMs about twice ----------------------------
int append_ksplit(int n_tok, int K, int N) {
  const int col_blocks = (N + mla::simt::PROJ_COLS - 1) / mla::simt::PROJ_COLS;
  const int tok_blocks = (n_tok + mla::simt::PROJ_TOK - 1) / mla::simt::PROJ_TOK;
  const int base = col_blocks * tok_blocks;
  int ks = (2 * num_sms() + base - 1) / base;
  ks = std::max(1, std::min(ks, std::min(32, (K + 63) / 64)));
  return ks;
}

// A tensor-core projection problem with the device's SM count filled in (it sizes the ring).
mla::gemm::Problem with_sms(mla::gemm::Problem pr) {
  pr.num_sms = num_sms();
  return pr;
}

// The tensor-core projection takes bf16 with whole 64-wide K chunks and 16-byte weight rows.
bool append_on_tc(int32_t dtype, int C, int N) { return dtype == MLA_BF16 && mla::gemm::supported(C, N); }
int append_tc_splits(int n_tok, int C, int N) { return mla::gemm::plan_splits(N, C, n_tok, num_sms(), 64); }

// Launch shape of the query chain's RMS step (one block per token): float4 slice reads in `groups`
// interleaved sets when N is a multiple of 4 and the slices are 16-byte aligned.
struct RmsShape {
  int threads, groups;
  size_t smem;
};
RmsShape rms_shape(int N, const void* part) {
  if (N % 4 == 0 && aligned16(part) && N / 4 <= mla::simt::RMS_THREADS) {
    const int groups = std::min(8, mla::simt::RMS_THREADS / (N / 4));
    return {std::min(mla::simt::RMS_THREADS, (groups * (N / 4) + 31) / 32 * 32), groups,
            (size_t)(1 + groups) * N * sizeof(float)};
  }
  return {std::min(mla::simt::RMS_THREADS, (N + 31) / 32 * 32), 0, (size_t)N * sizeof(float)};
}

// Launch shape of the a1 finish (one block per new token): with N a multiple of 4 and 16-byte aligned
// slices, readers of float4 pieces (`groups` slices at a time) plus one warp that finds the row's place
// meanwhile; otherwise one thread per column.
struct FinishShape {
  int threads, groups;
  size_t smem;
};
FinishShape finish_shape(int N, int d_r, const void* part) {
  if (N % 4 == 0 && aligned16(part) && N / 4 <= 496) {
    const int groups = std::min(8, 992 / (N / 4));
    return {mla::simt::finish_readers(N, groups) + 32, groups, ((size_t)(1 + groups) * N + d_r) * sizeof(float)};
  }
  return {std::min(1024, (N + 31) / 32 * 32), 0, (size_t)N * sizeof(float)};
}

// ---- a3 split choice for the CUDA-core decode ---------------------------------------------------
struct SimtSplit { int nsplit, chunk; };
SimtSplit simt_split(int n_tok, int H, int max_pages) {
  const int max_len = max_pages * 64;
  const int base = n_tok * (H / mla::simt::DEC_HEADS);
  int ns = (4 * num_sms() + base - 1) / base;
  ns = std::max(1, std::min(ns, std::max(1, max_len / 256)));
  ns = std::min(ns, 64);
  int chunk = (max_len + ns - 1) / ns;
  chunk = (chunk + 31) / 32 * 32;
  ns = (max_len + chunk - 1) / chunk;
  return {ns, chunk};
}

size_t simt_decode_ws(int n_tok, int H, int Dv, int max_pages) {
  SimtSplit s = simt_split(n_tok, H, max_pages);
  if (s.nsplit <= 1) return 0;
  const size_t slots = (size_t)n_tok * H * s.nsplit;
  return slots * Dv * sizeof(float) + slots * sizeof(float) + 256;
}

template <typename T>
int launch_decode_simt(DecodeArgs A, int n_tok, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int W = A.Dk + A.d_r;
  const size_t smem = ((size_t)8 * W + (size_t)32 * (W + 1) + (A.kv_shared ? 0 : (size_t)32 * A.Dv) + 256) * 4 + 32 * 8 + 32 * 4;
  if (A.nsplit > 1) {   // argument errors before any CUDA call
    const size_t slots = (size_t)n_tok * A.H * A.nsplit;
    if (!ws || ws_bytes < slots * A.Dv * sizeof(float) + slots * sizeof(float)) return MLA_ERR_WORKSPACE;
    A.part_o = reinterpret_cast<float*>(ws);
    A.part_lse = A.part_o + slots * A.Dv;
  }
  int rc = set_smem(mla::simt::decode_simt_kernel<T>, smem);
  if (rc) return rc;
  dim3 grid(n_tok, A.H / mla::simt::DEC_HEADS, A.nsplit);
  launch(mla::simt::decode_simt_kernel<T>, grid, 256, smem, st, A);
  if (A.nsplit > 1) {
    launch(mla::simt::merge_splits_kernel<T>, n_tok * A.H, 128, 0, st, 
        A.part_o, A.part_lse, A.nsplit, A.Dv, reinterpret_cast<T*>(A.out), A.out_head_stride, A.lse);
  }
  return launch_status();
}

}  // namespace

extern "C" {

const char* mla_status_string(int s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: null pointer, bad size, misaligned pointer or stride";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: no kernel for this dtype/shape";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace missing or too small";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA runtime call failed";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
    case MLA_ERR_DEVICE_CHECK: return "MLA_ERR_DEVICE_CHECK: an index read on the device was out of range";
    default: return "unknown mla status";
  }
}

uint64_t mla_launch_count(void) { return mla::g_launches.load(std::memory_order_relaxed); }

#ifdef MLA_TEST_HOOKS
// Test builds only (not declared in mla.h): makes every per-head GEMM's MMA issuer wait for a phase
// that nothing completes, so that a test can watch a bounded wait run out on the GPU.
MLA_API int mla_test_set_stall(int on) {
  return cudaMemcpyToSymbol(mla::gemm::g_test_stall, &on, sizeof(int)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
// Test builds only: the decode goes as two launches (decode, then the merge kernel) while on is set.
MLA_API int mla_test_set_two_launches(int on) {
  mla::sm100::g_test_two_launches = on != 0;
  return MLA_OK;
}
#endif

const char* mla_build_info(void) {
  return "libmla: sm_100a; kernels: simt (fp32/bf16 all steps), sm100 absorbed decode, GQLA grouped decode and per-head projections (tcgen05/TMA)";
}

int mla_check_status(void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, mla::g_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(mla::g_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  }
  return v;
}

// ------------------------------------------------------------------------------------------------
// a1
// ------------------------------------------------------------------------------------------------
size_t mla_append_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t C) {
  if (check_dims(dims) || !tokens_ok(B, s_q) || C <= 0) return 0;
  const int n_tok = B * s_q, N = dims->d_c + dims->d_r;
  int ks = append_ksplit(n_tok, C, N);
  if (mla::gemm::supported(C, N)) ks = std::max(ks, append_tc_splits(n_tok, C, N));
  return (size_t)ks * n_tok * N * sizeof(float);
}

namespace {
// The arguments of a1 (everything but the workspace); MLA_OK or the error status.
int append_args(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* x, int32_t C,
                const void* w_dkv_kr, const void* gamma, const int32_t* seqlens, const int32_t* block_table,
                int32_t max_pages, const mla_latent_cache_t* cache) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!tokens_ok(B, s_q) || C <= 0 || max_pages <= 0 || !x || !w_dkv_kr || !seqlens || !block_table || !cache)
    return MLA_ERR_INVALID_ARG;
  if (!cache->latent || !cache->rope || cache->num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_dkv_kr) || (gamma && !aligned16(gamma)) || !aligned16(cache->latent) ||
      !aligned16(cache->rope) || !aligned16(seqlens) || !aligned16(block_table))
    return MLA_ERR_INVALID_ARG;
  if (!stride_ok(cache->latent_stride, dtype, dims->d_c) || !stride_ok(cache->rope_stride, dtype, dims->d_r))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}
}  // namespace

int mla_append_cache(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* x,
                     int32_t C, const void* w_dkv_kr, const void* gamma, const int32_t* seqlens,
                     const int32_t* block_table, int32_t max_pages, const mla_latent_cache_t* cache,
                     void* workspace, size_t ws_bytes, void* stream) {
  int rc = append_args(dims, dtype, B, s_q, x, C, w_dkv_kr, gamma, seqlens, block_table, max_pages, cache);
  if (rc) return rc;
  const int n_tok = B * s_q, N = dims->d_c + dims->d_r;
  const bool tc = append_on_tc(dtype, C, N);
  const int ks = tc ? append_tc_splits(n_tok, C, N) : append_ksplit(n_tok, C, N);
  const size_t need = (size_t)ks * n_tok * N * sizeof(float);
  if (!workspace || ws_bytes < need) return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const FinishShape fs = finish_shape(N, dims->d_r, workspace);
  // attributes first: a failure here leaves nothing enqueued
  if ((rc = dtype == MLA_F32 ? set_smem(mla::simt::append_finish_kernel<float>, fs.smem)
                             : set_smem(mla::simt::append_finish_kernel<__nv_bfloat16>, fs.smem)))
    return rc;
  if (tc) {
    using T = __nv_bfloat16;
    mla::gemm::Params p{};
    p.mode = 1;
    p.part = reinterpret_cast<float*>(workspace);
    p.w_early = 1;
    if ((rc = mla::gemm::run(with_sms({w_dkv_kr, x, 1, C, N, n_tok, ks}), p, st))) return rc;
    mla::launch_pdl(mla::simt::append_finish_kernel<T>, dim3(n_tok), dim3(fs.threads), fs.smem, st, (const float*)p.part, ks, n_tok, s_q,
           dims->d_c, dims->d_r, (const T*)gamma, dims->rms_eps, dims->rope_base, seqlens, block_table, max_pages,
           (T*)cache->latent, cache->latent_stride, (T*)cache->rope, cache->rope_stride, cache->num_pages, 0, fs.groups);
    return launch_status();
  }
  const int k_chunk = ((C + ks - 1) / ks + 63) / 64 * 64;
  dim3 grid((N + mla::simt::PROJ_COLS - 1) / mla::simt::PROJ_COLS,
            (n_tok + mla::simt::PROJ_TOK - 1) / mla::simt::PROJ_TOK, ks);
  float* part = reinterpret_cast<float*>(workspace);
  if (dtype == MLA_F32) {
    using T = float;
    launch(mla::simt::proj_partial_kernel<T>, grid, mla::simt::PROJ_COLS, 0, st, 
        (const T*)x, n_tok, C, (const T*)w_dkv_kr, N, k_chunk, part, nullptr);
    launch(mla::simt::append_finish_kernel<T>, n_tok, fs.threads, fs.smem, st, 
        part, ks, n_tok, s_q, dims->d_c, dims->d_r, (const T*)gamma, dims->rms_eps, dims->rope_base, seqlens,
        block_table, max_pages, (T*)cache->latent, cache->latent_stride, (T*)cache->rope, cache->rope_stride,
        cache->num_pages, 0, fs.groups);
  } else {
    using T = __nv_bfloat16;
    launch(mla::simt::proj_partial_kernel<T>, grid, mla::simt::PROJ_COLS, 0, st, 
        (const T*)x, n_tok, C, (const T*)w_dkv_kr, N, k_chunk, part, nullptr);
    launch(mla::simt::append_finish_kernel<T>, n_tok, fs.threads, fs.smem, st, 
        part, ks, n_tok, s_q, dims->d_c, dims->d_r, (const T*)gamma, dims->rms_eps, dims->rope_base, seqlens,
        block_table, max_pages, (T*)cache->latent, cache->latent_stride, (T*)cache->rope, cache->rope_stride,
        cache->num_pages, 0, fs.groups);
  }
  return launch_status();
}

// ------------------------------------------------------------------------------------------------
// f2: query projection chain
// ------------------------------------------------------------------------------------------------
namespace {
// The tensor-core route takes bf16 with every K a whole number of 64-wide chunks.
bool query_on_tc(int32_t dtype, int C, int d_q, int H, int D, int d_r) {
  return dtype == MLA_BF16 && mla::gemm::supported(C, d_q) && mla::gemm::supported(d_q, H * D) &&
         mla::gemm::supported(d_q, H * d_r);
}
// fp32 partial sums of x·W_DQ first (256-byte aligned size), then c_q
size_t query_part_bytes(int ks, int n_tok, int d_q) { return ((size_t)ks * n_tok * d_q * sizeof(float) + 255) / 256 * 256; }
}  // namespace

size_t mla_query_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t C, int32_t d_q) {
  if (check_dims(dims) || !tokens_ok(B, s_q) || C <= 0 || d_q <= 0) return 0;
  const int n_tok = B * s_q;
  int ks = append_ksplit(n_tok, C, d_q);
  if (mla::gemm::supported(C, d_q)) ks = std::max(ks, append_tc_splits(n_tok, C, d_q));
  return query_part_bytes(ks, n_tok, d_q) + (size_t)n_tok * d_q * sizeof(float);
}

int mla_project_query(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* x, int32_t C,
                      int32_t d_q, const void* w_dq, const void* gamma_q, const void* w_uq, const void* w_qr,
                      void* q_nope, void* q_rope_raw, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!tokens_ok(B, s_q) || C <= 0 || d_q <= 0 || !x || !w_dq || !w_uq || !w_qr || !q_nope || !q_rope_raw)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_dq) || (gamma_q && !aligned16(gamma_q)) || !aligned16(w_uq) ||
      !aligned16(w_qr) || !aligned16(q_nope) || !aligned16(q_rope_raw))
    return MLA_ERR_INVALID_ARG;
  const int n_tok = B * s_q, H = dims->H, D = dims->D, d_r = dims->d_r;
  const bool tc = query_on_tc(dtype, C, d_q, H, D, d_r);
  const int ks = tc ? append_tc_splits(n_tok, C, d_q) : append_ksplit(n_tok, C, d_q);
  const size_t pb = query_part_bytes(ks, n_tok, d_q);
  const size_t need = pb + (size_t)n_tok * d_q * esize(dtype);
  if (!workspace || ws_bytes < need) return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* part = reinterpret_cast<float*>(workspace);
  void* c_q = reinterpret_cast<char*>(workspace) + pb;
  const RmsShape rs = rms_shape(d_q, part);
  // attributes first: a failure here leaves nothing enqueued
  if ((rc = dtype == MLA_F32 ? set_smem(mla::simt::rms_rows_kernel<float>, rs.smem)
                             : set_smem(mla::simt::rms_rows_kernel<__nv_bfloat16>, rs.smem)))
    return rc;
  if (tc) {
    using T = __nv_bfloat16;
    mla::gemm::Params p{};
    p.mode = 1;
    p.part = part;
    p.w_early = 1;
    if ((rc = mla::gemm::run(with_sms({w_dq, x, 1, C, d_q, n_tok, ks}), p, st))) return rc;
    mla::launch_pdl(mla::simt::rms_rows_kernel<T>, dim3(n_tok), dim3(rs.threads), rs.smem, st, (const float*)part, ks,
                    n_tok, d_q, (const T*)gamma_q, dims->rms_eps, (T*)c_q, rs.groups);
    // both up-projections in one launch, each a single-"head" GEMM over its whole output width
    mla::gemm::Params pu{};
    pu.mode = 0;
    pu.y = reinterpret_cast<T*>(q_nope);
    pu.y_tok_stride = (int64_t)H * D;
    pu.y2 = reinterpret_cast<T*>(q_rope_raw);
    pu.y2_tok_stride = (int64_t)H * d_r;
    pu.w_early = 1;
    mla::gemm::Problem up{w_uq, c_q, 1, d_q, H * D, n_tok, 1};
    up.w2 = w_qr;
    up.M2 = H * d_r;
    up.num_sms = num_sms();
    if ((rc = mla::gemm::run(up, pu, st))) return rc;
    return launch_status();
  }
  const int k_chunk = ((C + ks - 1) / ks + 63) / 64 * 64;
  const int tok_blocks = (n_tok + mla::simt::PROJ_TOK - 1) / mla::simt::PROJ_TOK;
  auto cols = [](int n) { return (n + mla::simt::PROJ_COLS - 1) / mla::simt::PROJ_COLS; };
  auto chain = [&](auto zero) -> int {
    using T = decltype(zero);
    launch(mla::simt::proj_partial_kernel<T>, dim3(cols(d_q), tok_blocks, ks), mla::simt::PROJ_COLS, 0, st,
           (const T*)x, n_tok, C, (const T*)w_dq, d_q, k_chunk, part, (T*)nullptr);
    launch(mla::simt::rms_rows_kernel<T>, n_tok, rs.threads, rs.smem, st, (const float*)part, ks, n_tok, d_q,
           (const T*)gamma_q, dims->rms_eps, (T*)c_q, rs.groups);
    // one K slice: the kernel writes the finished dot products straight to its output
    launch(mla::simt::proj_partial_kernel<T>, dim3(cols(H * D), tok_blocks, 1), mla::simt::PROJ_COLS, 0, st,
           (const T*)c_q, n_tok, d_q, (const T*)w_uq, H * D, d_q, (float*)nullptr, (T*)q_nope);
    launch(mla::simt::proj_partial_kernel<T>, dim3(cols(H * d_r), tok_blocks, 1), mla::simt::PROJ_COLS, 0, st,
           (const T*)c_q, n_tok, d_q, (const T*)w_qr, H * d_r, d_q, (float*)nullptr, (T*)q_rope_raw);
    return launch_status();
  };
  return dtype == MLA_F32 ? chain(0.f) : chain(__nv_bfloat16());
}

// ------------------------------------------------------------------------------------------------
// a2
// ------------------------------------------------------------------------------------------------
namespace {
// The arguments of a2; MLA_OK or the error status.
int absorb_args(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* q_nope,
                const void* q_rope_raw, const void* w_uk, const int32_t* seqlens, const void* q_abs) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!tokens_ok(B, s_q) || !q_nope || !q_rope_raw || !w_uk || !seqlens || !q_abs) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || !aligned16(q_rope_raw) || !aligned16(w_uk) || !aligned16(q_abs) || !aligned16(seqlens))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

// a2 on the tensor cores: bf16, whole 64-wide K chunks, 16-byte weight rows, a RoPE tail that fits.
bool absorb_on_tc(const mla_dims_t* dims, int32_t dtype) {
  return dtype == MLA_BF16 && mla::gemm::supported(dims->D, dims->d_c) && mla::gemm::supported_rope(dims->d_r);
}

// The tensor-core problem of a2: per head, q_nope[:, h, :] · W_UK[h] into q_abs[:, h, 0:d_c], with the
// rotated tail q_abs[:, h, d_c:] written by the m-tile-0 CTAs.
void absorb_problem(const mla_dims_t* dims, int32_t B, int32_t s_q, const void* q_nope, const void* q_rope_raw,
                    const void* w_uk, const int32_t* seqlens, void* q_abs, mla::gemm::Problem* pr,
                    mla::gemm::Params* p) {
  const int H = dims->H, d_c = dims->d_c, d_r = dims->d_r;
  *p = mla::gemm::Params{};
  p->mode = 0;
  p->y = reinterpret_cast<__nv_bfloat16*>(q_abs);
  p->y_tok_stride = (int64_t)H * (d_c + d_r);
  p->y_head_stride = d_c + d_r;
  p->rope_in = reinterpret_cast<const __nv_bfloat16*>(q_rope_raw);
  p->d_r = d_r;
  p->s_q = s_q;
  p->seqlens = seqlens;
  p->rope_base = dims->rope_base;
  p->w_early = 1;
  *pr = with_sms({w_uk, q_nope, H, dims->D, d_c, B * s_q, 1});
  pr->m_per_cta = 2;   // two CTAs per head and token block, each streaming half of W_UK[h]
}
}  // namespace

int mla_absorb_q(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* q_nope,
                 const void* q_rope_raw, const void* w_uk, const int32_t* seqlens, void* q_abs, void* stream) {
  int rc = absorb_args(dims, dtype, B, s_q, q_nope, q_rope_raw, w_uk, seqlens, q_abs);
  if (rc) return rc;
  const int n_tok = B * s_q;
  const int D = dims->D, H = dims->H, d_c = dims->d_c, d_r = dims->d_r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (absorb_on_tc(dims, dtype)) {
    mla::gemm::Problem pr;
    mla::gemm::Params p;
    absorb_problem(dims, B, s_q, q_nope, q_rope_raw, w_uk, seqlens, q_abs, &pr, &p);
    return mla::gemm::run(pr, p, st);
  }
  dim3 grid(H, (n_tok + mla::simt::HG_TOK - 1) / mla::simt::HG_TOK);
  const size_t smem = (size_t)mla::simt::HG_TOK * D * sizeof(float);
  if (dtype == MLA_F32) {
    using T = float;
    if ((rc = set_smem(mla::simt::head_gemm_kernel<T>, smem))) return rc;
    launch(mla::simt::head_gemm_kernel<T>, grid, 128, smem, st, 
        (const T*)q_nope, D, D, (const T*)w_uk, d_c, n_tok, H, (T*)q_abs, d_c + d_r, (const T*)q_rope_raw, d_r,
        seqlens, s_q, dims->rope_base);
  } else {
    using T = __nv_bfloat16;
    if ((rc = set_smem(mla::simt::head_gemm_kernel<T>, smem))) return rc;
    launch(mla::simt::head_gemm_kernel<T>, grid, 128, smem, st, 
        (const T*)q_nope, D, D, (const T*)w_uk, d_c, n_tok, H, (T*)q_abs, d_c + d_r, (const T*)q_rope_raw, d_r,
        seqlens, s_q, dims->rope_base);
  }
  return launch_status();
}

// ------------------------------------------------------------------------------------------------
// a1 + a2 in one call
// ------------------------------------------------------------------------------------------------
int mla_append_cache_absorb_q(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* x,
                              int32_t C, const void* w_dkv_kr, const void* gamma, const void* q_nope,
                              const void* q_rope_raw, const void* w_uk, const int32_t* seqlens,
                              const int32_t* block_table, int32_t max_pages, const mla_latent_cache_t* cache,
                              void* q_abs, void* workspace, size_t ws_bytes, void* stream) {
  // every argument of both halves is checked before anything is launched
  int rc = append_args(dims, dtype, B, s_q, x, C, w_dkv_kr, gamma, seqlens, block_table, max_pages, cache);
  if (rc) return rc;
  if ((rc = absorb_args(dims, dtype, B, s_q, q_nope, q_rope_raw, w_uk, seqlens, q_abs))) return rc;
  if (mla_append_workspace_size(dims, B, s_q, C) > ws_bytes || !workspace) return MLA_ERR_WORKSPACE;
  // the append first: the absorption's CTAs then stream W_UK while the append's finish runs
  if ((rc = mla_append_cache(dims, dtype, B, s_q, x, C, w_dkv_kr, gamma, seqlens, block_table, max_pages, cache,
                             workspace, ws_bytes, stream)))
    return rc;
  return mla_absorb_q(dims, dtype, B, s_q, q_nope, q_rope_raw, w_uk, seqlens, q_abs, stream);
}

// ------------------------------------------------------------------------------------------------
// a3 + a4
// ------------------------------------------------------------------------------------------------
size_t mla_decode_workspace_size(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, int32_t max_pages) {
  if (check_dims(dims) || check_dtype(dtype) || !tokens_ok(B, s_q) || max_pages <= 0) return 0;
  size_t ws = simt_decode_ws(B * s_q, dims->H, dims->d_c, max_pages);
  ws = std::max(ws, mla::sm100::decode_workspace_bytes(dims, dtype, B, s_q, num_sms()));
  return ws;
}

int mla_decode_absorbed_hinted(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* q_abs,
                               const mla_latent_cache_t* cache, const int32_t* block_table, int32_t max_pages,
                               const int32_t* seqlens, const int32_t* seqlens_host, void* o_lat, float* lse,
                               void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!tokens_ok(B, s_q) || max_pages <= 0 || !q_abs || !cache || !block_table || !seqlens || !o_lat || !lse)
    return MLA_ERR_INVALID_ARG;
  if (!cache->latent || !cache->rope || cache->num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_abs) || !aligned16(cache->latent) || !aligned16(cache->rope) || !aligned16(block_table) ||
      !aligned16(seqlens) || !aligned16(o_lat) || !aligned16(lse) || (workspace && !aligned16(workspace)))
    return MLA_ERR_INVALID_ARG;
  if (!stride_ok(cache->latent_stride, dtype, dims->d_c) || !stride_ok(cache->rope_stride, dtype, dims->d_r))
    return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int n_tok = B * s_q;

  if (mla::sm100::decode_supported(dims, dtype, B, s_q)) {
    const mla_dims_t dd = with_scale(dims);
    return mla::sm100::launch_decode(&dd, B, s_q, q_abs, cache, block_table, max_pages, seqlens, o_lat, lse,
                                     workspace, ws_bytes, num_sms(), seqlens_host, st);
  }

  if (dims->H % mla::simt::DEC_HEADS || dims->d_c % 32 || dims->d_c > 32 * mla::simt::DEC_MAX_OV)
    return MLA_ERR_UNSUPPORTED;
  DecodeArgs A{};
  A.q = q_abs;
  A.q_head_stride = dims->d_c + dims->d_r;
  A.q_rope_raw = nullptr;
  A.kpart = cache->latent; A.k_stride = cache->latent_stride; A.k_group_off = 0;
  A.vpart = cache->latent; A.v_stride = cache->latent_stride; A.v_group_off = 0;
  A.rope = cache->rope; A.rope_stride = cache->rope_stride;
  A.Dk = dims->d_c; A.Dv = dims->d_c; A.d_r = dims->d_r; A.H = dims->H; A.heads_per_group = dims->H;
  A.kv_shared = 1;
  A.block_table = block_table; A.max_pages = max_pages; A.num_pages = cache->num_pages;
  A.seqlens = seqlens; A.s_q = s_q; A.sm_scale = score_scale(dims); A.rope_base = dims->rope_base;
  A.out = o_lat; A.out_head_stride = dims->d_c; A.lse = lse;
  SimtSplit sp = simt_split(n_tok, dims->H, max_pages);
  A.nsplit = sp.nsplit; A.chunk = sp.chunk;
  return dtype == MLA_F32 ? launch_decode_simt<float>(A, n_tok, workspace, ws_bytes, st)
                          : launch_decode_simt<__nv_bfloat16>(A, n_tok, workspace, ws_bytes, st);
}

int mla_decode_absorbed(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* q_abs,
                        const mla_latent_cache_t* cache, const int32_t* block_table, int32_t max_pages,
                        const int32_t* seqlens, void* o_lat, float* lse, void* workspace, size_t ws_bytes,
                        void* stream) {
  return mla_decode_absorbed_hinted(dims, dtype, B, s_q, q_abs, cache, block_table, max_pages, seqlens, nullptr, o_lat,
                                    lse, workspace, ws_bytes, stream);
}

// ------------------------------------------------------------------------------------------------
// 8-bit latent cache
// ------------------------------------------------------------------------------------------------
int mla_quantize_latent_fp8(const mla_dims_t* dims, int32_t dtype, const void* latent, int64_t latent_stride,
                            int64_t rows, uint8_t* codes, int64_t code_stride, float* scales, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!latent || !codes || !scales || rows <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(latent) || !aligned16(codes) || !aligned16(scales)) return MLA_ERR_INVALID_ARG;
  if (!stride_ok(latent_stride, dtype, dims->d_c) || code_stride < dims->d_c || code_stride % 16) return MLA_ERR_INVALID_ARG;
  if (dims->d_c % 16) return MLA_ERR_UNSUPPORTED;
  if ((rows + 7) / 8 > INT32_MAX) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid((unsigned)((rows + 7) / 8));
  if (dtype == MLA_F32)
    launch(mla::simt::quantize_e4m3_kernel<float>, grid, 256, 0, st, (const float*)latent, latent_stride, rows,
           dims->d_c, codes, code_stride, scales);
  else
    launch(mla::simt::quantize_e4m3_kernel<__nv_bfloat16>, grid, 256, 0, st, (const __nv_bfloat16*)latent,
           latent_stride, rows, dims->d_c, codes, code_stride, scales);
  return launch_status();
}

namespace {
// The tensor-core route of the 8-bit decode: the batch's pages dequantised into a dense bf16 scratch
// (latent rows, RoPE rows, a dense page table), then the bf16 tensor-core decode over it.
struct Fp8Scratch {
  size_t lat, rope, table, dec, total;
};
bool fp8_on_tc(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q) {
  // (the dequantising pass takes one block row per sequence: B within a grid's y extent)
  return mla::sm100::decode_supported(dims, dtype, B, s_q) && dims->d_c % 16 == 0 && dims->d_r % 8 == 0 &&
         B <= 65535;
}
Fp8Scratch fp8_scratch(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t max_pages) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t rows = (size_t)B * max_pages * 64;
  Fp8Scratch f;
  f.lat = 0;
  f.rope = up(rows * dims->d_c * 2);
  f.table = f.rope + up(rows * dims->d_r * 2);
  f.dec = f.table + up((size_t)B * max_pages * 4);
  f.total = f.dec + mla::sm100::decode_workspace_bytes(dims, MLA_BF16, B, s_q, num_sms());
  return f;
}
}  // namespace

size_t mla_decode_fp8_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t max_pages) {
  if (check_dims(dims) || !tokens_ok(B, s_q) || max_pages <= 0) return 0;
  const size_t simt = simt_decode_ws(B * s_q, dims->H, dims->d_c, max_pages);
  const bool tc = fp8_on_tc(dims, MLA_BF16, B, s_q) && (int64_t)B * max_pages * 64 <= INT32_MAX;
  return tc ? std::max(simt, fp8_scratch(dims, B, s_q, max_pages).total) : simt;
}

int mla_decode_absorbed_fp8(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* q_abs,
                            const mla_latent_cache_fp8_t* cache, const int32_t* block_table, int32_t max_pages,
                            const int32_t* seqlens, void* o_lat, float* lse, void* workspace, size_t ws_bytes,
                            void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!tokens_ok(B, s_q) || max_pages <= 0 || !q_abs || !cache || !block_table || !seqlens || !o_lat || !lse)
    return MLA_ERR_INVALID_ARG;
  if (!cache->codes || !cache->scales || !cache->rope || cache->num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_abs) || !aligned16(cache->codes) || !aligned16(cache->scales) || !aligned16(cache->rope) ||
      !aligned16(block_table) || !aligned16(seqlens) || !aligned16(o_lat) || !aligned16(lse) ||
      (workspace && !aligned16(workspace)))
    return MLA_ERR_INVALID_ARG;
  if (cache->code_stride < dims->d_c || cache->code_stride % 16 || !stride_ok(cache->rope_stride, dtype, dims->d_r))
    return MLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (fp8_on_tc(dims, dtype, B, s_q) && (int64_t)B * max_pages * 64 <= INT32_MAX) {
    // dequantise the pages the decode reads into bf16 (one rounding of s * value), then decode them
    // on the tensor cores through a dense page table
    const Fp8Scratch f = fp8_scratch(dims, B, s_q, max_pages);
    if (!workspace || ws_bytes < f.total) return MLA_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    using T = __nv_bfloat16;
    mla::launch_pdl(mla::simt::dequant_pages_kernel, dim3(max_pages, B), dim3(256), 0, st,
                    (const uint8_t*)cache->codes, cache->code_stride, (const float*)cache->scales, (const T*)cache->rope,
                    cache->rope_stride, cache->num_pages, seqlens, block_table, max_pages, dims->d_c, dims->d_r,
                    (T*)(ws + f.lat), (T*)(ws + f.rope), (int32_t*)(ws + f.table));
    if ((rc = launch_status())) return rc;
    mla_latent_cache_t dense{ws + f.lat, dims->d_c, ws + f.rope, dims->d_r, B * max_pages};
    const mla_dims_t dd = with_scale(dims);
    return mla::sm100::launch_decode(&dd, B, s_q, q_abs, &dense, (const int32_t*)(ws + f.table), max_pages, seqlens,
                                     o_lat, lse, ws + f.dec, ws_bytes - f.dec, num_sms(), nullptr, st);
  }
  if (dims->H % mla::simt::DEC_HEADS || dims->d_c % 32 || dims->d_c > 32 * mla::simt::DEC_MAX_OV)
    return MLA_ERR_UNSUPPORTED;
  const int n_tok = B * s_q;
  DecodeArgs A{};
  A.q = q_abs;
  A.q_head_stride = dims->d_c + dims->d_r;
  A.q_rope_raw = nullptr;
  A.kpart = cache->codes; A.k_stride = cache->code_stride; A.k_group_off = 0; A.kscale = cache->scales;
  A.vpart = cache->codes; A.v_stride = cache->code_stride; A.v_group_off = 0;
  A.rope = cache->rope; A.rope_stride = cache->rope_stride;
  A.Dk = dims->d_c; A.Dv = dims->d_c; A.d_r = dims->d_r; A.H = dims->H; A.heads_per_group = dims->H;
  A.kv_shared = 1;
  A.block_table = block_table; A.max_pages = max_pages; A.num_pages = cache->num_pages;
  A.seqlens = seqlens; A.s_q = s_q; A.sm_scale = score_scale(dims); A.rope_base = dims->rope_base;
  A.out = o_lat; A.out_head_stride = dims->d_c; A.lse = lse;
  SimtSplit sp = simt_split(n_tok, dims->H, max_pages);
  A.nsplit = sp.nsplit; A.chunk = sp.chunk;
  return dtype == MLA_F32 ? launch_decode_simt<float>(A, n_tok, workspace, ws_bytes, st)
                          : launch_decode_simt<__nv_bfloat16>(A, n_tok, workspace, ws_bytes, st);
}

// ------------------------------------------------------------------------------------------------
// a5
// ------------------------------------------------------------------------------------------------
int mla_out_proj(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* o_lat,
                 const void* w_uv, void* out, const void* w_o, int32_t C, void* out_model, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!tokens_ok(B, s_q) || !o_lat || !w_uv || !out) return MLA_ERR_INVALID_ARG;
  if (w_o && (C <= 0 || !out_model)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_lat) || !aligned16(w_uv) || !aligned16(out) || (w_o && (!aligned16(w_o) || !aligned16(out_model))))
    return MLA_ERR_INVALID_ARG;
  const int n_tok = B * s_q;
  const int H = dims->H, d_c = dims->d_c, d_v = dims->d_v;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  dim3 grid(H, (n_tok + mla::simt::HG_TOK - 1) / mla::simt::HG_TOK);
  const size_t smem = (size_t)mla::simt::HG_TOK * d_c * sizeof(float);
  dim3 ogrid((C + mla::simt::PROJ_COLS - 1) / mla::simt::PROJ_COLS, (n_tok + mla::simt::PROJ_TOK - 1) / mla::simt::PROJ_TOK, 1);
  const int K = H * d_v;
  if (dtype == MLA_BF16 && mla::gemm::supported(d_c, d_v)) {
    mla::gemm::Params p{};
    p.mode = 0;
    p.y = reinterpret_cast<__nv_bfloat16*>(out);
    p.y_tok_stride = (int64_t)H * d_v;
    p.y_head_stride = d_v;
    p.w_early = 1;
    if ((rc = mla::gemm::run(with_sms({w_uv, o_lat, H, d_c, d_v, n_tok, 1}), p, st))) return rc;
    if (w_o) {
      if (mla::gemm::supported(K, C)) {   // the heads concatenated, times W_O, on the tensor cores
        mla::gemm::Params po{};
        po.mode = 0;
        po.y = reinterpret_cast<__nv_bfloat16*>(out_model);
        po.y_tok_stride = C;
        po.y_head_stride = 0;
        po.w_early = 1;
        if ((rc = mla::gemm::run(with_sms({w_o, out, 1, K, C, n_tok, 1}), po, st))) return rc;
      } else {
        using T = __nv_bfloat16;
        launch(mla::simt::proj_partial_kernel<T>, ogrid, mla::simt::PROJ_COLS, 0, st, (const T*)out, n_tok, K,
               (const T*)w_o, C, K, nullptr, (T*)out_model);
      }
    }
    return launch_status();
  }
  if (dtype == MLA_F32) {
    using T = float;
    if ((rc = set_smem(mla::simt::head_gemm_kernel<T>, smem))) return rc;
    launch(mla::simt::head_gemm_kernel<T>, grid, 128, smem, st, (const T*)o_lat, d_c, d_c, (const T*)w_uv, d_v, n_tok, H,
                                                            (T*)out, d_v, nullptr, 0, nullptr, 1, 0.f);
    if (w_o)
      launch(mla::simt::proj_partial_kernel<T>, ogrid, mla::simt::PROJ_COLS, 0, st, (const T*)out, n_tok, K, (const T*)w_o,
                                                                               C, K, nullptr, (T*)out_model);
  } else {
    using T = __nv_bfloat16;
    if ((rc = set_smem(mla::simt::head_gemm_kernel<T>, smem))) return rc;
    launch(mla::simt::head_gemm_kernel<T>, grid, 128, smem, st, (const T*)o_lat, d_c, d_c, (const T*)w_uv, d_v, n_tok, H,
                                                            (T*)out, d_v, nullptr, 0, nullptr, 1, 0.f);
    if (w_o)
      launch(mla::simt::proj_partial_kernel<T>, ogrid, mla::simt::PROJ_COLS, 0, st, (const T*)out, n_tok, K, (const T*)w_o,
                                                                               C, K, nullptr, (T*)out_model);
  }
  return launch_status();
}

// ------------------------------------------------------------------------------------------------
// f3: W_UV·W_O absorbed into one output weight, and the output projection through it
// ------------------------------------------------------------------------------------------------
int mla_preabsorb_out_weights(const mla_dims_t* dims, int32_t dtype, const void* w_uv, const void* w_o, int32_t C,
                              void* w_uvo, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (C <= 0 || !w_uv || !w_o || !w_uvo) return MLA_ERR_INVALID_ARG;
  if (!aligned16(w_uv) || !aligned16(w_o) || !aligned16(w_uvo)) return MLA_ERR_INVALID_ARG;
  const int H = dims->H, d_c = dims->d_c, d_v = dims->d_v;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t es = esize(dtype);
  // head h: W_UVO[h] [d_c, C] = W_UV[h] [d_c, d_v] · W_O[h*d_v : (h+1)*d_v, :]
  for (int h = 0; h < H; ++h) {
    const char* wuv_h = static_cast<const char*>(w_uv) + (size_t)h * d_c * d_v * es;
    const char* wo_h = static_cast<const char*>(w_o) + (size_t)h * d_v * C * es;
    char* y_h = static_cast<char*>(w_uvo) + (size_t)h * d_c * C * es;
    if (dtype == MLA_BF16 && mla::gemm::supported(d_v, C) && aligned16(wuv_h) && aligned16(wo_h) && aligned16(y_h) &&
        ((size_t)d_v * es) % 16 == 0) {
      mla::gemm::Params p{};
      p.mode = 0;
      p.y = reinterpret_cast<__nv_bfloat16*>(y_h);
      p.y_tok_stride = C;
      p.y_head_stride = 0;
      if ((rc = mla::gemm::run(with_sms({wo_h, wuv_h, 1, d_v, C, d_c, 1}), p, st))) return rc;
    } else {
      dim3 grid((C + mla::simt::PROJ_COLS - 1) / mla::simt::PROJ_COLS, (d_c + mla::simt::PROJ_TOK - 1) / mla::simt::PROJ_TOK, 1);
      if (dtype == MLA_F32)
        launch(mla::simt::proj_partial_kernel<float>, grid, mla::simt::PROJ_COLS, 0, st, (const float*)wuv_h, d_c, d_v,
               (const float*)wo_h, C, d_v, nullptr, (float*)y_h);
      else
        launch(mla::simt::proj_partial_kernel<__nv_bfloat16>, grid, mla::simt::PROJ_COLS, 0, st,
               (const __nv_bfloat16*)wuv_h, d_c, d_v, (const __nv_bfloat16*)wo_h, C, d_v, nullptr, (__nv_bfloat16*)y_h);
    }
  }
  return launch_status();
}

int mla_out_proj_preabsorbed(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* o_lat,
                             const void* w_uvo, int32_t C, void* out_model, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!tokens_ok(B, s_q) || C <= 0 || !o_lat || !w_uvo || !out_model) return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_lat) || !aligned16(w_uvo) || !aligned16(out_model)) return MLA_ERR_INVALID_ARG;
  const int n_tok = B * s_q, K = dims->H * dims->d_c;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // out_model[tok, :] = concat_h(o_lat[tok, h, :]) · W_UVO, W_UVO = [H*d_c, C]
  if (dtype == MLA_BF16 && mla::gemm::supported(K, C)) {
    mla::gemm::Params p{};
    p.mode = 0;
    p.y = reinterpret_cast<__nv_bfloat16*>(out_model);
    p.y_tok_stride = C;
    p.y_head_stride = 0;
    if ((rc = mla::gemm::run(with_sms({w_uvo, o_lat, 1, K, C, n_tok, 1}), p, st))) return rc;
    return launch_status();
  }
  dim3 grid((C + mla::simt::PROJ_COLS - 1) / mla::simt::PROJ_COLS, (n_tok + mla::simt::PROJ_TOK - 1) / mla::simt::PROJ_TOK, 1);
  if (dtype == MLA_F32)
    launch(mla::simt::proj_partial_kernel<float>, grid, mla::simt::PROJ_COLS, 0, st, (const float*)o_lat, n_tok, K,
           (const float*)w_uvo, C, K, nullptr, (float*)out_model);
  else
    launch(mla::simt::proj_partial_kernel<__nv_bfloat16>, grid, mla::simt::PROJ_COLS, 0, st, (const __nv_bfloat16*)o_lat,
           n_tok, K, (const __nv_bfloat16*)w_uvo, C, K, nullptr, (__nv_bfloat16*)out_model);
  return launch_status();
}

// ------------------------------------------------------------------------------------------------
// f3: append to the expanded (GQA) cache
// ------------------------------------------------------------------------------------------------
namespace {
struct GqaAppendLayout { int ks; size_t part, cbuf, kbuf, vbuf, total; };
size_t up256(size_t x) { return (x + 255) / 256 * 256; }
GqaAppendLayout gqa_append_layout(const mla_dims_t* d, int n_tok, int C) {
  GqaAppendLayout L{};
  const int N = d->d_c + d->d_r;
  L.ks = append_tc_splits(n_tok, C, N);
  L.part = 0;
  L.cbuf = up256((size_t)L.ks * n_tok * N * sizeof(float));
  L.kbuf = L.cbuf + up256((size_t)n_tok * d->d_c * 2);
  L.vbuf = L.kbuf + up256((size_t)n_tok * d->g * d->D * 2);
  L.total = L.vbuf + up256((size_t)n_tok * d->g * d->d_v * 2);
  return L;
}
bool gqa_append_supported(const mla_dims_t* d, int32_t dtype, int C) {
  return dtype == MLA_BF16 && d->g > 0 && d->H % d->g == 0 && mla::gemm::supported(C, d->d_c + d->d_r) &&
         mla::gemm::supported(d->d_c, d->D) && mla::gemm::supported(d->d_c, d->d_v);
}
}  // namespace

size_t mla_gqa_append_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t C) {
  if (check_dims(dims) || !tokens_ok(B, s_q) || C <= 0 || !gqa_append_supported(dims, MLA_BF16, C)) return 0;
  return gqa_append_layout(dims, B * s_q, C).total;
}

int mla_append_gqa_cache(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* x, int32_t C,
                         const void* w_dkv_kr, const void* gamma, const void* w_uk_g, const void* w_uv_g,
                         const int32_t* seqlens, const int32_t* block_table, int32_t max_pages,
                         const mla_gqa_cache_t* cache, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (dims->g <= 0 || dims->H % dims->g) return MLA_ERR_INVALID_ARG;
  if (!tokens_ok(B, s_q) || C <= 0 || max_pages <= 0 || !x || !w_dkv_kr || !w_uk_g || !w_uv_g || !seqlens ||
      !block_table || !cache)
    return MLA_ERR_INVALID_ARG;
  if (!cache->k || !cache->v || !cache->rope || cache->num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_dkv_kr) || (gamma && !aligned16(gamma)) || !aligned16(w_uk_g) ||
      !aligned16(w_uv_g) || !aligned16(seqlens) || !aligned16(block_table) || !aligned16(cache->k) ||
      !aligned16(cache->v) || !aligned16(cache->rope))
    return MLA_ERR_INVALID_ARG;
  if (!stride_ok(cache->k_stride, dtype, (int64_t)dims->g * dims->D) ||
      !stride_ok(cache->v_stride, dtype, (int64_t)dims->g * dims->d_v) || !stride_ok(cache->rope_stride, dtype, dims->d_r))
    return MLA_ERR_INVALID_ARG;
  if (!gqa_append_supported(dims, dtype, C)) return MLA_ERR_UNSUPPORTED;
  const int n_tok = B * s_q, N = dims->d_c + dims->d_r, g = dims->g;
  const GqaAppendLayout lay = gqa_append_layout(dims, n_tok, C);
  if (!workspace || ws_bytes < lay.total) return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_INVALID_ARG;
  using T = __nv_bfloat16;
  char* ws = static_cast<char*>(workspace);
  float* part = reinterpret_cast<float*>(ws + lay.part);
  T* cbuf = reinterpret_cast<T*>(ws + lay.cbuf);
  T* kbuf = reinterpret_cast<T*>(ws + lay.kbuf);
  T* vbuf = reinterpret_cast<T*>(ws + lay.vbuf);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const FinishShape fs = finish_shape(N, dims->d_r, part);
  if ((rc = set_smem(mla::simt::append_finish_kernel<T>, fs.smem))) return rc;
  // 1. z = x · [W_DKV | W_KR] (split-K partial sums)
  mla::gemm::Params p{};
  p.mode = 1;
  p.part = part;
  if ((rc = mla::gemm::run(with_sms({w_dkv_kr, x, 1, C, N, n_tok, lay.ks}), p, st))) return rc;
  // 2. c = RMSNorm(z_c)·gamma into a plain buffer (rounded to the storage type, as a latent cache row
  //    would be); k_r = RoPE(z_r) into the cache's RoPE rows
  mla::launch_pdl(mla::simt::append_finish_kernel<T>, dim3(n_tok), dim3(fs.threads), fs.smem, st, (const float*)part,
                  lay.ks, n_tok, s_q, dims->d_c, dims->d_r, (const T*)gamma, dims->rms_eps, dims->rope_base, seqlens,
                  block_table, max_pages, cbuf, (int64_t)dims->d_c, (T*)cache->rope, cache->rope_stride,
                  cache->num_pages, 1, fs.groups);
  // 3. K_g = W_UK[g] · c (W_UK stored [g, D, d_c]: read K-major), V_g = c · W_UV[g], every group
  mla::gemm::Problem pk{w_uk_g, cbuf, g, dims->d_c, dims->D, n_tok, 1};
  pk.a_kmajor = true;
  pk.x_shared = true;
  mla::gemm::Params pkp{};
  pkp.mode = 0;
  pkp.y = kbuf;
  pkp.y_tok_stride = (int64_t)g * dims->D;
  pkp.y_head_stride = dims->D;
  if ((rc = mla::gemm::run(with_sms(pk), pkp, st))) return rc;
  mla::gemm::Problem pv{w_uv_g, cbuf, g, dims->d_c, dims->d_v, n_tok, 1};
  pv.x_shared = true;
  mla::gemm::Params pvp{};
  pvp.mode = 0;
  pvp.y = vbuf;
  pvp.y_tok_stride = (int64_t)g * dims->d_v;
  pvp.y_head_stride = dims->d_v;
  if ((rc = mla::gemm::run(with_sms(pv), pvp, st))) return rc;
  // 4. the rows into the cache slots of their positions
  mla::launch_pdl(mla::simt::gqa_scatter_kernel<T>, dim3(n_tok), dim3(128), 0, st, (const T*)kbuf, (const T*)vbuf, s_q,
                  g * dims->D, g * dims->d_v, seqlens, block_table, max_pages, cache->num_pages, (T*)cache->k,
                  cache->k_stride, (T*)cache->v, cache->v_stride);
  return launch_status();
}

// ------------------------------------------------------------------------------------------------
// a6
// ------------------------------------------------------------------------------------------------
size_t mla_gqla_workspace_size(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, int32_t max_pages) {
  if (check_dims(dims) || check_dtype(dtype) || !tokens_ok(B, s_q) || max_pages <= 0) return 0;
  size_t ws = simt_decode_ws(B * s_q, dims->H, dims->d_v, max_pages);
  if (dims->g > 0 && mla::gqla::supported(dims, dtype, s_q))
    ws = std::max(ws, mla::gqla::workspace_bytes(dims, B, max_pages, num_sms()));
  return ws;
}

int mla_decode_gqla_grouped(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* q_nope,
                            const void* q_rope_raw, const mla_gqa_cache_t* cache, const int32_t* block_table,
                            int32_t max_pages, const int32_t* seqlens, void* out, float* lse, void* workspace,
                            size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (dims->g <= 0 || dims->H % dims->g) return MLA_ERR_INVALID_ARG;
  if (!tokens_ok(B, s_q) || max_pages <= 0 || !q_nope || !q_rope_raw || !cache || !block_table || !seqlens ||
      !out || !lse)
    return MLA_ERR_INVALID_ARG;
  if (!cache->k || !cache->v || !cache->rope || cache->num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || !aligned16(q_rope_raw) || !aligned16(cache->k) || !aligned16(cache->v) ||
      !aligned16(cache->rope) || !aligned16(block_table) || !aligned16(seqlens) || !aligned16(out) ||
      !aligned16(lse) || (workspace && !aligned16(workspace)))
    return MLA_ERR_INVALID_ARG;
  const int hpg = dims->H / dims->g;
  if (!stride_ok(cache->k_stride, dtype, (int64_t)dims->g * dims->D) ||
      !stride_ok(cache->v_stride, dtype, (int64_t)dims->g * dims->d_v) || !stride_ok(cache->rope_stride, dtype, dims->d_r))
    return MLA_ERR_INVALID_ARG;
  if (mla::gqla::supported(dims, dtype, s_q)) {
    const mla_dims_t dd = with_scale(dims);
    return mla::gqla::launch_gqla(&dd, B, q_nope, q_rope_raw, cache, block_table, max_pages, seqlens, out, lse,
                                  workspace, ws_bytes, num_sms(), reinterpret_cast<cudaStream_t>(stream));
  }
  if (hpg % mla::simt::DEC_HEADS || dims->d_v % 32 || dims->d_v > 32 * mla::simt::DEC_MAX_OV) return MLA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int n_tok = B * s_q;
  DecodeArgs A{};
  A.q = q_nope;
  A.q_head_stride = dims->D;
  A.q_rope_raw = q_rope_raw;
  A.kpart = cache->k; A.k_stride = cache->k_stride; A.k_group_off = dims->D;
  A.vpart = cache->v; A.v_stride = cache->v_stride; A.v_group_off = dims->d_v;
  A.rope = cache->rope; A.rope_stride = cache->rope_stride;
  A.Dk = dims->D; A.Dv = dims->d_v; A.d_r = dims->d_r; A.H = dims->H; A.heads_per_group = hpg;
  A.kv_shared = 0;
  A.block_table = block_table; A.max_pages = max_pages; A.num_pages = cache->num_pages;
  A.seqlens = seqlens; A.s_q = s_q; A.sm_scale = score_scale(dims); A.rope_base = dims->rope_base;
  A.out = out; A.out_head_stride = dims->d_v; A.lse = lse;
  SimtSplit sp = simt_split(n_tok, dims->H, max_pages);
  A.nsplit = sp.nsplit; A.chunk = sp.chunk;
  return dtype == MLA_F32 ? launch_decode_simt<float>(A, n_tok, workspace, ws_bytes, st)
                          : launch_decode_simt<__nv_bfloat16>(A, n_tok, workspace, ws_bytes, st);
}

}  // extern "C"

// ================================================================================================
// Cache append for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs inside a framework
// whose memory pool owns every byte of the device and forbids side allocations, plugins that only
// receive the tensors of the call, or processes that must not call cudaMalloc once serving has
// started. mla_append_cache_noalloc serves them: its split-K partial sums live in a fixed buffer
// that is part of this library's device image (g_append_scratch, 4 MiB). The caller still passes
// every input and output; nothing is allocated or freed, by this call or by any library it calls.
//
// In host code g_append_scratch is only a host-side stand-in for the device array: its device
// address is looked up once per device with cudaGetSymbolAddress (with that device current) and
// cached; that set-up happens in the first call made on each device. Every call shares the one
// buffer, which keeps the previous call's contents; nothing in it needs to start at zero (each
// call writes every partial sum it later reads). Calls that overlap on the GPU (different streams
// without ordering between them) race on the buffer.
// ================================================================================================
namespace {

constexpr size_t kAppendScratchFloats = size_t(1) << 20;   // 4 MiB of fp32 partial sums
__device__ __align__(256) float g_append_scratch[kAppendScratchFloats];

std::mutex g_append_scratch_mu;
float* g_append_scratch_dev[kMaxDevices] = {nullptr};

// Device address of g_append_scratch on the current device (looked up once per device).
int append_scratch_address(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_append_scratch_mu);
  if (g_append_scratch_dev[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_append_scratch) != cudaSuccess || ptr == nullptr) return MLA_ERR_CUDA;
    g_append_scratch_dev[dev] = static_cast<float*>(ptr);
  }
  *out = g_append_scratch_dev[dev];
  return MLA_OK;
}

}  // namespace

extern "C" int mla_append_cache_noalloc(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* x,
                                        int32_t C, const void* w_dkv_kr, const void* gamma, const int32_t* seqlens,
                                        const int32_t* block_table, int32_t max_pages, const mla_latent_cache_t* cache,
                                        void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  if (!tokens_ok(B, s_q) || C <= 0 || max_pages <= 0 || !x || !w_dkv_kr || !seqlens || !block_table || !cache)
    return MLA_ERR_INVALID_ARG;
  if (!cache->latent || !cache->rope || cache->num_pages <= 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_dkv_kr) || (gamma && !aligned16(gamma)) || !aligned16(cache->latent) ||
      !aligned16(cache->rope) || !aligned16(seqlens) || !aligned16(block_table))
    return MLA_ERR_INVALID_ARG;
  if (!stride_ok(cache->latent_stride, dtype, dims->d_c) || !stride_ok(cache->rope_stride, dtype, dims->d_r))
    return MLA_ERR_INVALID_ARG;
  const int n_tok = B * s_q, N = dims->d_c + dims->d_r;
  // as many K slices as the built-in buffer holds, at most the number the workspace path uses
  const size_t per_slice = (size_t)n_tok * N;
  if (per_slice > kAppendScratchFloats) return MLA_ERR_WORKSPACE;   // B*s_q*(d_c+d_r) > 1,048,576
  const int cap = (int)(kAppendScratchFloats / per_slice);
  const bool tc = append_on_tc(dtype, C, N);
  const int ks = std::min(tc ? append_tc_splits(n_tok, C, N) : append_ksplit(n_tok, C, N), cap);
  float* part = nullptr;
  if ((rc = append_scratch_address(&part))) return rc;
  const FinishShape fs = finish_shape(N, dims->d_r, part);
  // attributes first: a failure here leaves nothing enqueued
  if ((rc = dtype == MLA_F32 ? set_smem(mla::simt::append_finish_kernel<float>, fs.smem)
                             : set_smem(mla::simt::append_finish_kernel<__nv_bfloat16>, fs.smem)))
    return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (tc) {
    // the tensor-core projection writes one fp32 slice per K split (an empty split writes zeros)
    using T = __nv_bfloat16;
    mla::gemm::Params p{};
    p.mode = 1;
    p.part = part;
    if ((rc = mla::gemm::run(with_sms({w_dkv_kr, x, 1, C, N, n_tok, ks}), p, st))) return rc;
    mla::launch_pdl(mla::simt::append_finish_kernel<T>, dim3(n_tok), dim3(fs.threads), fs.smem, st,
                    (const float*)part, ks, n_tok, s_q, dims->d_c, dims->d_r, (const T*)gamma, dims->rms_eps,
                    dims->rope_base, seqlens, block_table, max_pages, (T*)cache->latent, cache->latent_stride,
                    (T*)cache->rope, cache->rope_stride, cache->num_pages, 0, fs.groups);
    return launch_status();
  }
  const int k_chunk = ((C + ks - 1) / ks + 63) / 64 * 64;
  dim3 grid((N + mla::simt::PROJ_COLS - 1) / mla::simt::PROJ_COLS,
            (n_tok + mla::simt::PROJ_TOK - 1) / mla::simt::PROJ_TOK, ks);
  if (dtype == MLA_F32) {
    using T = float;
    launch(mla::simt::proj_partial_kernel<T>, grid, mla::simt::PROJ_COLS, 0, st, (const T*)x, n_tok, C,
           (const T*)w_dkv_kr, N, k_chunk, part, (T*)nullptr);
    launch(mla::simt::append_finish_kernel<T>, n_tok, fs.threads, fs.smem, st, (const float*)part, ks, n_tok, s_q,
           dims->d_c, dims->d_r, (const T*)gamma, dims->rms_eps, dims->rope_base, seqlens, block_table, max_pages,
           (T*)cache->latent, cache->latent_stride, (T*)cache->rope, cache->rope_stride, cache->num_pages, 0, fs.groups);
  } else {
    using T = __nv_bfloat16;
    launch(mla::simt::proj_partial_kernel<T>, grid, mla::simt::PROJ_COLS, 0, st, (const T*)x, n_tok, C,
           (const T*)w_dkv_kr, N, k_chunk, part, (T*)nullptr);
    launch(mla::simt::append_finish_kernel<T>, n_tok, fs.threads, fs.smem, st, (const float*)part, ks, n_tok, s_q,
           dims->d_c, dims->d_r, (const T*)gamma, dims->rms_eps, dims->rope_base, seqlens, block_table, max_pages,
           (T*)cache->latent, cache->latent_stride, (T*)cache->rope, cache->rope_stride, cache->num_pages, 0, fs.groups);
  }
  return launch_status();
}

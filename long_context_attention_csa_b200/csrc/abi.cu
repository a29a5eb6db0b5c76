// extern "C" entry points of libcsa.so: argument validation, workspace
// layout, kernel selection and the device status word.  See include/csa.h for
// the contract of each call.
#include <atomic>

#include "common.cuh"
#include "sm100.cuh"
#include "internal.h"
#include "tc.h"

using namespace csa;

namespace {

std::atomic<unsigned long long> g_launches{0};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

inline cudaStream_t S(void* stream) { return reinterpret_cast<cudaStream_t>(stream); }

inline csa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_E_CUDA; }

// Common checks of the entry format.
csa_status check_fmt(int32_t dtype, const csa_fmt* fmt, Fmt* out) {
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_E_ARG;
  if (fmt == nullptr) return CSA_E_ARG;
  if (fmt->c <= 0 || fmt->rope_dims < 0 || fmt->rope_dims > fmt->c || (fmt->rope_dims & 1))
    return CSA_E_ARG;
  if (!(fmt->norm_eps >= 0.f) || !(fmt->rope_base > 0.f)) return CSA_E_ARG;
  if (fmt->flags & ~(CSA_F_NO_NORM | CSA_F_NO_ROPE | CSA_F_PORTABLE | CSA_F_MIXED))
    return CSA_E_ARG;
  const int vec = dtype == CSA_BF16 ? 8 : 4;
  if (fmt->c % vec != 0 || !pow2(fmt->c / vec) || fmt->c / vec > 256) return CSA_E_UNSUPPORTED;
  out->c = fmt->c;
  out->r = fmt->rope_dims;
  out->base = fmt->rope_base;
  out->eps = fmt->norm_eps;
  out->flags = fmt->flags;
  return CSA_OK;
}

unsigned* status_word(void* ws) { return static_cast<unsigned*>(ws); }

csa_status compress_common(int32_t dtype, int64_t B, int64_t T, int32_t m, bool overlap,
                           const csa_fmt* fmt, const void* kv_a, const void* kv_b,
                           const void* z_a, const void* z_b, int32_t z_cols, int64_t pos0,
                           void* entries, void* win_out, void* ws, size_t ws_bytes,
                           void* stream) {
  Fmt f;
  csa_status st = check_fmt(dtype, fmt, &f);
  if (st != CSA_OK) return st;
  if (B < 0 || T < 0 || m < 1 || B > 65535) return CSA_E_ARG;
  if (z_cols != 1 && z_cols != f.c) return CSA_E_ARG;
  if (overlap ? (2 * m > 256) : (m > 4096)) return CSA_E_UNSUPPORTED;
  if (f.c != 64 && f.c != 128 && f.c != 256 && f.c != 512) return CSA_E_UNSUPPORTED;
  const int64_t n = T / m;
  if (B == 0 || T == 0) return CSA_OK;
  if (!kv_a || !z_a || (overlap && (!kv_b || !z_b))) return CSA_E_ARG;
  if (n > 0 && !entries) return CSA_E_ARG;
  if (!aligned16(kv_a) || (overlap && !aligned16(kv_b)) || (entries && !aligned16(entries)) ||
      (win_out && !aligned16(win_out)))
    return CSA_E_ARG;
  if (z_cols != 1 && (!aligned16(z_a) || (overlap && !aligned16(z_b)))) return CSA_E_ARG;
  if (n == 0 && !win_out) return CSA_OK;
  if (n + 1 > 0x7fffffffLL) return CSA_E_UNSUPPORTED;
  if (!ws || ws_bytes < kWsScratch) return CSA_E_WORKSPACE;
  CompressParams p{};
  p.kv_a = kv_a;
  p.kv_b = kv_b;
  p.z_a = z_a;
  p.z_b = z_b;
  p.z_cols = z_cols;
  p.T = T;
  p.n_entries = n;
  p.m = m;
  p.overlap = overlap ? 1 : 0;
  p.f = f;
  p.pos0 = pos0;
  p.entries = entries;
  p.win = win_out;
  p.status = status_word(ws);
  g_launches.fetch_add(1);
  return cuda_status(launch_compress(dtype, p, B, S(stream)));
}

}  // namespace

namespace csa {

void note_launches(unsigned long long n) { g_launches.fetch_add(n); }

csa_status indexer_prepare(int32_t dtype, int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                           const void* q_I, const float* w, const void* k_I, int64_t N,
                           const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                           float* score_out, IndexerParams* out, bool* tc) {
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_E_ARG;
  if (B < 0 || Tq < 0 || N < 0 || H_I <= 0 || d_I <= 0 || m < 1 || k < 1) return CSA_E_ARG;
  if (B > 65535 || Tq > 0x7fffffffLL || N > 0x7fffffffLL) return CSA_E_UNSUPPORTED;
  if (H_I > 64 || d_I > 1024) return CSA_E_UNSUPPORTED;
  if (B == 0 || Tq == 0) return CSA_OK;
  if (!q_I || !w || !idx_out || (N > 0 && !k_I)) return CSA_E_ARG;
  if (!aligned16(q_I) || (N > 0 && !aligned16(k_I))) return CSA_E_ARG;
  IndexerParams& p = *out;
  p.B = B;
  p.Tq = Tq;
  p.HI = H_I;
  p.dI = d_I;
  p.q_I = q_I;
  p.w = w;
  p.k_I = k_I;
  p.N = N;
  p.q_pos = q_pos;
  p.m = m;
  p.k = k;
  p.idx_out = idx_out;
  p.score_out = score_out;
  // bf16 runs on the tensor cores only; shapes outside that kernel's envelope
  // are rejected rather than sent to the CUDA-core kernels, which serve float32
  *tc = dtype == CSA_BF16;
  if (*tc && !indexer_tc_supported(p)) return CSA_E_UNSUPPORTED;
  return CSA_OK;
}

size_t indexer_scratch(bool tc, const IndexerParams& p) {
  return tc ? indexer_tc_scratch(p.B, p.Tq, p.N, p.k)
            : indexer_portable_scratch(p.B, p.Tq, p.N, p.k);
}

csa_status indexer_launch(int32_t dtype, bool tc, const IndexerParams& p, cudaStream_t stream) {
  if (tc) {
    unsigned long long n_launch = 0;
    cudaError_t e = launch_indexer_tc(p, stream, &n_launch);
    note_launches(n_launch);
    return cuda_status(e);
  }
  note_launches(2);
  return cuda_status(launch_indexer_portable(dtype, p, stream));
}

}  // namespace csa

extern "C" {

csa_status csa_compress(int32_t dtype, int64_t B, int64_t T, int32_t m, const csa_fmt* fmt,
                        const void* kv_a, const void* kv_b, const void* z_a, const void* z_b,
                        int32_t z_cols, int64_t pos0, void* entries, void* win_out, void* ws,
                        size_t ws_bytes, void* stream) {
  return compress_common(dtype, B, T, m, true, fmt, kv_a, kv_b, z_a, z_b, z_cols, pos0, entries,
                         win_out, ws, ws_bytes, stream);
}

csa_status hca_compress(int32_t dtype, int64_t B, int64_t T, int32_t m_prime, const csa_fmt* fmt,
                        const void* kv, const void* z, int32_t z_cols, int64_t pos0, void* entries,
                        void* win_out, void* ws, size_t ws_bytes, void* stream) {
  return compress_common(dtype, B, T, m_prime, false, fmt, kv, nullptr, z, nullptr, z_cols, pos0,
                         entries, win_out, ws, ws_bytes, stream);
}

size_t csa_stream_state_bytes(int32_t dtype, int32_t m, int32_t overlap, int32_t c,
                              int32_t z_cols) {
  if ((dtype != CSA_F32 && dtype != CSA_BF16) || m < 1 || c <= 0 || (z_cols != 1 && z_cols != c))
    return 0;
  return stream_state_bytes(dtype == CSA_BF16 ? 2 : 4, m, overlap ? 1 : 0, c, z_cols);
}

static csa_status append_common(int32_t dtype, int64_t B, int32_t m, bool overlap,
                                const csa_fmt* fmt, const void* kv_a, const void* kv_b,
                                const void* z_a, const void* z_b, int32_t z_cols, int64_t pos0,
                                void* state, size_t state_stride, void* entries, int64_t n_cap,
                                void* win_out, void* ws, size_t ws_bytes, void* stream) {
  Fmt f;
  csa_status st = check_fmt(dtype, fmt, &f);
  if (st != CSA_OK) return st;
  if (B < 0 || m < 1 || n_cap < 0 || B > 0x7fffffffLL) return CSA_E_ARG;
  if (z_cols != 1 && z_cols != f.c) return CSA_E_ARG;
  if (overlap ? (2 * m > 256) : (m > 4096)) return CSA_E_UNSUPPORTED;
  if (f.c < 64 || f.c > 1024 || f.r > 2 * kStreamMaxPairs) return CSA_E_UNSUPPORTED;
  if (B == 0) return CSA_OK;
  if (!kv_a || !z_a || !state || (overlap && (!kv_b || !z_b)) || (n_cap > 0 && !entries))
    return CSA_E_ARG;
  if (!aligned16(kv_a) || !aligned16(state) || (overlap && !aligned16(kv_b)) ||
      (entries && !aligned16(entries)) || (win_out && !aligned16(win_out)))
    return CSA_E_ARG;
  if (z_cols != 1 && (!aligned16(z_a) || (overlap && !aligned16(z_b)))) return CSA_E_ARG;
  const size_t need = stream_state_bytes(dtype == CSA_BF16 ? 2 : 4, m, overlap ? 1 : 0, f.c,
                                         z_cols);
  if (state_stride < need || (state_stride & 15)) return CSA_E_ARG;
  if (!ws || ws_bytes < kWsScratch) return CSA_E_WORKSPACE;
  StreamParams p{};
  p.kv_a = kv_a;
  p.kv_b = kv_b;
  p.z_a = z_a;
  p.z_b = z_b;
  p.z_cols = z_cols;
  p.m = m;
  p.overlap = overlap ? 1 : 0;
  p.f = f;
  p.pos0 = pos0;
  p.state = static_cast<uint8_t*>(state);
  p.stride = state_stride;
  p.entries = entries;
  p.n_cap = n_cap;
  p.win = win_out;
  p.status = status_word(ws);
  g_launches.fetch_add(1);
  return cuda_status(launch_stream_append(dtype, p, B, S(stream)));
}

csa_status csa_compress_append(int32_t dtype, int64_t B, int32_t m, const csa_fmt* fmt,
                               const void* kv_a, const void* kv_b, const void* z_a,
                               const void* z_b, int32_t z_cols, int64_t pos0, void* state,
                               size_t state_stride, void* entries, int64_t n_cap, void* win_out,
                               void* ws, size_t ws_bytes, void* stream) {
  return append_common(dtype, B, m, true, fmt, kv_a, kv_b, z_a, z_b, z_cols, pos0, state,
                       state_stride, entries, n_cap, win_out, ws, ws_bytes, stream);
}

csa_status hca_compress_append(int32_t dtype, int64_t B, int32_t m_prime, const csa_fmt* fmt,
                               const void* kv, const void* z, int32_t z_cols, int64_t pos0,
                               void* state, size_t state_stride, void* entries, int64_t n_cap,
                               void* win_out, void* ws, size_t ws_bytes, void* stream) {
  return append_common(dtype, B, m_prime, false, fmt, kv, nullptr, z, nullptr, z_cols, pos0,
                       state, state_stride, entries, n_cap, win_out, ws, ws_bytes, stream);
}

size_t csa_mixed_record_bytes(int32_t c, int32_t rope_dims) {
  if (c <= 0 || rope_dims < 0 || rope_dims > c || (c - rope_dims) % 32 != 0) return 0;
  return mixed_record_bytes(c, rope_dims);
}

csa_status csa_store_mixed(int32_t dtype, int64_t B, int64_t N, const csa_fmt* fmt,
                           const void* entries, void* records, void* stream) {
  Fmt f;
  csa_status st = check_fmt(dtype, fmt, &f);
  if (st != CSA_OK) return st;
  if (B < 0 || N < 0) return CSA_E_ARG;
  if ((f.c - f.r) % 32 != 0 || f.c - f.r > 1024) return CSA_E_UNSUPPORTED;
  if (B == 0 || N == 0) return CSA_OK;
  if (!entries || !records || !aligned16(entries) || !aligned16(records)) return CSA_E_ARG;
  g_launches.fetch_add(1);
  return cuda_status(launch_mixed_store(dtype, entries, records, B * N, f.c, f.r, S(stream)));
}

static csa_status mx_quantize(int fmt, int32_t dtype, int64_t B, int64_t rows, int32_t d,
                              const void* x, void* codes, void* scales, void* stream) {
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_E_ARG;
  if (B < 0 || rows < 0 || d <= 0) return CSA_E_ARG;
  if (d != 128) return CSA_E_UNSUPPORTED;
  if (B > 65535 || rows > 0x7fffffffLL) return CSA_E_UNSUPPORTED;
  if (B == 0 || rows == 0) return CSA_OK;
  if (!x || !codes || !scales) return CSA_E_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return CSA_E_ARG;
  g_launches.fetch_add(1);
  return cuda_status(fmt == 2 ? launch_mxfp4_quantize(dtype, x, codes, scales, B, rows, S(stream))
                              : launch_mxfp8_quantize(dtype, x, codes, scales, B, rows, S(stream)));
}

csa_status indexer_mxfp8_quantize(int32_t dtype, int64_t B, int64_t rows, int32_t d,
                                  const void* x, void* codes, void* scales, void* stream) {
  return mx_quantize(1, dtype, B, rows, d, x, codes, scales, stream);
}

csa_status indexer_mxfp4_quantize(int32_t dtype, int64_t B, int64_t rows, int32_t d,
                                  const void* x, void* codes, void* scales, void* stream) {
  return mx_quantize(2, dtype, B, rows, d, x, codes, scales, stream);
}

static csa_status scores_mx(int fmt, int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                            const void* q_codes, const void* q_scales, const float* w,
                            const void* k_codes, const void* k_scales, int64_t N,
                            const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                            float* score_out, void* ws, size_t ws_bytes, void* stream) {
  if (B < 0 || Tq < 0 || N < 0 || H_I <= 0 || d_I <= 0 || m < 1 || k < 1) return CSA_E_ARG;
  if (H_I != 64 || d_I != 128) return CSA_E_UNSUPPORTED;
  if (B > 65535 || Tq > 65535 || N > 0x7fffffffLL) return CSA_E_UNSUPPORTED;
  if (B == 0 || Tq == 0) return CSA_OK;
  if (!q_codes || !q_scales || !w || !idx_out || (N > 0 && (!k_codes || !k_scales)))
    return CSA_E_ARG;
  if (!aligned16(q_codes) || !aligned16(q_scales) ||
      (N > 0 && (!aligned16(k_codes) || !aligned16(k_scales))))
    return CSA_E_ARG;
  if (!ws || ws_bytes < csa_workspace_bytes(CSA_OP_INDEXER_MX, CSA_BF16, B, Tq, 0, 0, N, k, 0))
    return CSA_E_WORKSPACE;
  IndexerParams p{};
  p.B = B;
  p.Tq = Tq;
  p.HI = H_I;
  p.dI = d_I;
  p.q_I = q_codes;
  p.w = w;
  p.k_I = k_codes;
  p.N = N;
  p.q_pos = q_pos;
  p.m = m;
  p.k = k;
  p.idx_out = idx_out;
  p.score_out = score_out;
  p.status = status_word(ws);
  p.scratch = static_cast<char*>(ws) + kWsScratch;
  p.scratch_bytes = ws_bytes - kWsScratch;
  unsigned long long n = 0;
  cudaError_t e = launch_indexer_mx(p, fmt, q_scales, k_scales, S(stream), &n);
  g_launches.fetch_add(n);
  return cuda_status(e);
}

csa_status indexer_scores_topk_mxfp8(int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                                     const void* q_codes, const void* q_scales, const float* w,
                                     const void* k_codes, const void* k_scales, int64_t N,
                                     const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                                     float* score_out, void* ws, size_t ws_bytes, void* stream) {
  return scores_mx(1, B, Tq, H_I, d_I, q_codes, q_scales, w, k_codes, k_scales, N, q_pos, m, k,
                   idx_out, score_out, ws, ws_bytes, stream);
}

csa_status indexer_scores_topk_mxfp4(int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                                     const void* q_codes, const void* q_scales, const float* w,
                                     const void* k_codes, const void* k_scales, int64_t N,
                                     const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                                     float* score_out, void* ws, size_t ws_bytes, void* stream) {
  return scores_mx(2, B, Tq, H_I, d_I, q_codes, q_scales, w, k_codes, k_scales, N, q_pos, m, k,
                   idx_out, score_out, ws, ws_bytes, stream);
}

csa_status grouped_output_projection(int32_t dtype, int64_t T, int32_t H, int32_t c, int32_t g,
                                     int32_t d_g, int32_t d, const void* o, const void* w_group,
                                     const void* w_out, void* y, void* ws, size_t ws_bytes,
                                     void* stream) {
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_E_ARG;
  if (T < 0 || H <= 0 || c <= 0 || g <= 0 || d_g <= 0 || d <= 0) return CSA_E_ARG;
  ProjParams p{};
  p.T = T;
  p.H = H;
  p.c = c;
  p.g = g;
  p.dg = d_g;
  p.d = d;
  if (dtype != CSA_BF16 || !proj_supported(p)) return CSA_E_UNSUPPORTED;
  if (T == 0) return CSA_OK;
  if (!o || !w_group || !w_out || !y) return CSA_E_ARG;
  if (!aligned16(o) || !aligned16(w_group) || !aligned16(w_out) || !aligned16(y))
    return CSA_E_ARG;
  if (!ws || ws_bytes < csa_workspace_bytes(CSA_OP_OUT_PROJ, dtype, 1, T, 0, 0,
                                            (int64_t)g * d_g, 0, 0))
    return CSA_E_WORKSPACE;
  p.o = o;
  p.w_group = w_group;
  p.w_out = w_out;
  p.v = static_cast<char*>(ws) + kWsScratch;
  p.y = y;
  p.status = status_word(ws);
  unsigned long long n = 0;
  cudaError_t e = launch_proj(p, S(stream), &n);
  g_launches.fetch_add(n);
  return cuda_status(e);
}

size_t csa_workspace_bytes(int32_t op, int32_t dtype, int64_t B, int64_t Tq, int32_t H, int32_t c,
                           int64_t N, int32_t k, int32_t n_win) {
  if (B < 0 || Tq < 0 || N < 0) return 0;
  switch (op) {
    case CSA_OP_COMPRESS:
      return kWsScratch;
    case CSA_OP_INDEXER_MX:
      return kWsScratch + indexer_mx_scratch(B, Tq, N, k);
    case CSA_OP_OUT_PROJ:
      return kWsScratch + (size_t)B * (size_t)Tq * (size_t)N * 2;
    case CSA_OP_INDEXER:
      return kWsScratch + (dtype == CSA_BF16 ? indexer_tc_scratch(B, Tq, N, k)
                                             : indexer_portable_scratch(B, Tq, N, k));
    case CSA_OP_SPARSE_ATTN:
    case CSA_OP_DENSE_ATTN: {
      int64_t max_keys = (op == CSA_OP_SPARSE_ATTN ? (int64_t)k : N) + n_win;
      size_t b = dtype == CSA_BF16 ? attn_tc_scratch(B, Tq, H, c, max_keys) : 0;
      return kWsScratch + b;
    }
    default:
      return 0;
  }
}

csa_status indexer_scores_topk(int32_t dtype, int64_t B, int64_t Tq, int32_t H_I, int32_t d_I,
                               const void* q_I, const float* w, const void* k_I, int64_t N,
                               const int64_t* q_pos, int32_t m, int32_t k, int32_t* idx_out,
                               float* score_out, void* ws, size_t ws_bytes, void* stream) {
  IndexerParams p{};
  bool tc = false;
  csa_status st = indexer_prepare(dtype, B, Tq, H_I, d_I, q_I, w, k_I, N, q_pos, m, k, idx_out,
                                  score_out, &p, &tc);
  if (st != CSA_OK || B == 0 || Tq == 0) return st;
  if (!ws) return CSA_E_WORKSPACE;
  if (ws_bytes < kWsScratch + indexer_scratch(tc, p)) return CSA_E_WORKSPACE;
  p.status = status_word(ws);
  p.scratch = static_cast<char*>(ws) + kWsScratch;
  p.scratch_bytes = ws_bytes - kWsScratch;
  return indexer_launch(dtype, tc, p, S(stream));
}

static csa_status attn_common(int32_t dtype, int64_t B, int64_t Tq, int32_t H, const csa_fmt* fmt,
                              bool sparse, const void* q, const int64_t* q_pos, const void* entries, int64_t N,
                              const int32_t* idx, int32_t k, int32_t m_dense, const void* win,
                              int64_t Tw, const int64_t* win_pos0, int32_t n_win,
                              const float* sink, float scale, void* out, void* ws,
                              size_t ws_bytes, void* stream) {
  Fmt f;
  csa_status st = check_fmt(dtype, fmt, &f);
  if (st != CSA_OK) return st;
  if (B < 0 || Tq < 0 || H <= 0 || N < 0 || Tw < 0 || n_win < 0) return CSA_E_ARG;
  if (sparse ? k < 0 : m_dense < 1) return CSA_E_ARG;
  if (B > 65535 || Tq > 0x7fffffffLL) return CSA_E_UNSUPPORTED;
  if (f.c % 64 != 0 || f.c > 512) return CSA_E_UNSUPPORTED;
  if (B == 0 || Tq == 0) return CSA_OK;
  if (!q || !out || (N > 0 && !entries) || (Tw > 0 && !win)) return CSA_E_ARG;
  if (!aligned16(q) || !aligned16(out) || (entries && !aligned16(entries)) ||
      (win && !aligned16(win)))
    return CSA_E_ARG;
  AttnParams p{};
  if (f.flags & CSA_F_MIXED) {
    if ((f.c - f.r) % 32 != 0 || f.c - f.r > 1024) return CSA_E_UNSUPPORTED;
    p.mixed = 1;
    p.rec_bytes = (int)mixed_record_bytes(f.c, f.r);
  }
  p.B = B;
  p.Tq = Tq;
  p.H = H;
  p.f = f;
  p.q = q;
  p.entries = entries;
  p.N = N;
  p.sparse = sparse ? 1 : 0;
  p.k = sparse ? k : 0;
  p.Tw = Tw;
  p.out = out;
  p.win = win;
  // bf16 runs on the tensor cores unless CSA_F_PORTABLE asks for the CUDA-core
  // kernel; shapes outside the tensor-core kernel's envelope are rejected
  if (dtype == CSA_BF16 && !(f.flags & CSA_F_PORTABLE) && !attn_tc_supported(p))
    return CSA_E_UNSUPPORTED;
  if (!ws) return CSA_E_WORKSPACE;
  const int op = sparse ? CSA_OP_SPARSE_ATTN : CSA_OP_DENSE_ATTN;
  if (ws_bytes < csa_workspace_bytes(op, dtype, B, Tq, H, f.c, N, k, n_win)) return CSA_E_WORKSPACE;
  p.q_pos = q_pos;
  p.idx = idx;
  p.m_dense = m_dense;
  p.win_pos0 = win_pos0;
  p.n_win = n_win;
  p.sink = sink;
  p.scale = scale;
  p.out = out;
  p.status = status_word(ws);
  p.scratch = static_cast<char*>(ws) + kWsScratch;
  p.scratch_bytes = ws_bytes - kWsScratch;
  if (dtype == CSA_BF16 && !(f.flags & CSA_F_PORTABLE)) {
    unsigned long long n_launch = 0;
    cudaError_t e = launch_attn_tc(p, S(stream), &n_launch);
    g_launches.fetch_add(n_launch);
    return cuda_status(e);
  }
  g_launches.fetch_add(1);
  return cuda_status(launch_attn_portable(dtype, p, S(stream)));
}

csa_status sparse_mqa_attn(int32_t dtype, int64_t B, int64_t Tq, int32_t H, const csa_fmt* fmt,
                           const void* q, const int64_t* q_pos, const void* entries, int64_t N,
                           const int32_t* idx, int32_t k, const void* win, int64_t Tw,
                           const int64_t* win_pos0, int32_t n_win, const float* sink, float scale,
                           void* out, void* ws, size_t ws_bytes, void* stream) {
  if (k < 0 || (!idx && k > 0)) return CSA_E_ARG;
  return attn_common(dtype, B, Tq, H, fmt, true, q, q_pos, entries, N, idx, k, 1, win, Tw,
                     win_pos0, n_win, sink, scale, out, ws, ws_bytes, stream);
}

csa_status dense_hca_attn(int32_t dtype, int64_t B, int64_t Tq, int32_t H, const csa_fmt* fmt,
                          const void* q, const int64_t* q_pos, const void* entries, int64_t N,
                          int32_t m_prime, const void* win, int64_t Tw, const int64_t* win_pos0,
                          int32_t n_win, const float* sink, float scale, void* out, void* ws,
                          size_t ws_bytes, void* stream) {
  return attn_common(dtype, B, Tq, H, fmt, false, q, q_pos, entries, N, nullptr, 0, m_prime, win,
                     Tw, win_pos0, n_win, sink, scale, out, ws, ws_bytes, stream);
}

namespace {
// One thread waits, bounded, on a barrier that no thread ever arrives on.
__global__ void selftest_wait_kernel(unsigned* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0u, limit_ns))
    report(status, CSA_DEV_TIMEOUT, 0x5e1fu);
}
}  // namespace

csa_status csa_selftest_wait(int64_t limit_ns, void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kWsScratch || limit_ns < 1000 || limit_ns > 10000000000LL)
    return CSA_E_ARG;
  selftest_wait_kernel<<<1, 32, 0, S(stream)>>>(status_word(ws), (uint64_t)limit_ns);
  g_launches.fetch_add(1);
  return cuda_status(cudaGetLastError());
}

csa_status csa_check_status(void* ws, void* stream, uint32_t* detail) {
  if (!ws) return CSA_E_ARG;
  cudaError_t e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) return CSA_E_CUDA;
  unsigned word[2] = {0u, 0u};
  e = cudaMemcpy(word, ws, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return CSA_E_CUDA;
  if (detail) *detail = word[0];
  if (word[0] == 0u) return CSA_OK;
  e = cudaMemset(ws, 0, sizeof(word));
  if (e != cudaSuccess) return CSA_E_CUDA;
  return CSA_E_DEVICE;
}

const char* csa_status_string(csa_status s) {
  switch (s) {
    case CSA_OK: return "ok";
    case CSA_E_ARG: return "invalid argument";
    case CSA_E_UNSUPPORTED: return "unsupported shape or format";
    case CSA_E_CUDA: return "CUDA error";
    case CSA_E_DEVICE: return "device-side error (see status word)";
    case CSA_E_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

unsigned long long csa_launch_count(void) { return g_launches.load(); }

}  // extern "C"

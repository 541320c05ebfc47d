// C ABI of libmla.so: argument validation, workspace carving and launches.
// Every step of the path runs in the kernels included below; this file only
// checks arguments, computes workspace offsets and launches.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "append_f64.cuh"
#include "common.cuh"
#include "decode_plan.cuh"
#include "decode_simt.cuh"
#include "decode_pair.cuh"
#include "elementwise.cuh"
#include "gemm_simt.cuh"
#include "out_combine.cuh"
#include "qhead_tc.cuh"
#include "wgemm_tc.cuh"

using namespace mla;

namespace {

mla_status check_cfg(const mla_config* c) {
  if (!c) return MLA_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->n_heads <= 0 || c->d_c <= 0 || c->d_r <= 0 || c->qk_nope <= 0 ||
      c->v_head <= 0 || c->q_lora < 0 || c->block_size <= 0 || (c->d_r & 1) ||
      !(c->rope_theta > 0.0) || c->softmax_scale < 0.f)
    return MLA_ERR_INVALID_ARG;
  if (c->dtype != MLA_F32 && c->dtype != MLA_BF16) return MLA_ERR_INVALID_ARG;
  if (c->flags & ~(MLA_FLAG_SPLIT_QUERY | MLA_FLAG_FP8_CACHE)) return MLA_ERR_INVALID_ARG;
  if ((c->flags & MLA_FLAG_FP8_CACHE) && c->dtype != MLA_BF16) return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

inline bool fp8_cache(const mla_config* c) { return (c->flags & MLA_FLAG_FP8_CACHE) != 0; }

// The bf16 tensor-core decode (pair kernel, packed query): bf16 pages only.
inline bool tc_decode(const mla_config* c) { return c->dtype == MLA_BF16 && !fp8_cache(c); }

mla_status check_cache(const mla_cache* k) {
  if (!k || !k->pool || !k->block_table || k->num_blocks <= 0 || k->batch <= 0 ||
      k->max_blocks_per_seq <= 0)
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

mla_status check_cache(const mla_config* c, const mla_cache* k) {
  const mla_status st0 = check_cache(k);
  if (st0 != MLA_OK) return st0;
  if (fp8_cache(c) && (k->row_scale == nullptr || (reinterpret_cast<uintptr_t>(k->row_scale) & 3u)))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
template <typename... P>
inline bool all_aligned16(const P*... p) {
  return (aligned16(p) && ...);
}

inline mla_status st(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

#define MLA_TRY(expr)                          \
  do {                                         \
    mla_status _s = (expr);                    \
    if (_s != MLA_OK) return _s;               \
  } while (0)
#define MLA_CUDA(expr) MLA_TRY(st(expr))

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// ---------------------------------------------------------------- append
// The latent projection is accumulated in fp64 (exact products of bf16
// values, fp64 sums), so rounding it once gives the bf16 of the real-number
// dot product.  K is cut into `append_splits` chunks (more parallel work for
// a skinny GEMM) whose fp64 sums are added into one zeroed fp64 buffer.
int append_splits(const mla_config* c) {
  int S = 1;
  for (int cand = 32; cand > 1; --cand)
    if (c->hidden % cand == 0 && c->hidden / cand >= 128) {
      S = cand;
      break;
    }
  return S;
}

size_t append_ws(const mla_config* c, int n_tok) {
  return align_up(sizeof(double) * (size_t)n_tok * (c->d_c + c->d_r), 256);
}

template <typename T>
mla_status append_impl(const mla_config* c, const void* x, int n, const void* W_DKV, const void* W_KR,
                       const int32_t* seq_idx, const int32_t* pos, const mla_cache* k, void* ws,
                       cudaStream_t s) {
  const int row = c->d_c + c->d_r;
  double* C = static_cast<double*>(ws);
  MLA_CUDA(cudaMemsetAsync(C, 0, sizeof(double) * (size_t)n * row, s));
  if (apf64::supports<T>(x, c->hidden, W_DKV, c->d_c, W_KR, c->d_r, c->d_c, c->d_r, c->hidden)) {
    const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
    const int tiles = (row / apf64::BN) * ((n + apf64::BM - 1) / apf64::BM);
    const int S = apf64::choose_splits(c->hidden, tiles, sms);
    apf64::Args<T> a{static_cast<const T*>(x), c->hidden, static_cast<const T*>(W_DKV), c->d_c,
                     static_cast<const T*>(W_KR), c->d_r, c->d_c, C, row, n, c->hidden / S};
    MLA_CUDA(apf64::launch<T>(a, row, S, s));
  } else {
    const int S = append_splits(c), Kc = c->hidden / S;
    GemmSimtArgs g1{x, W_DKV, C, n, c->d_c, Kc, S, c->hidden, 1, Kc, c->d_c, 1, (long long)Kc * c->d_c, row, 1, 0};
    MLA_CUDA((gemm_simt<T, T, double, true>(g1, s)));
    GemmSimtArgs g2{x, W_KR, C + c->d_c, n, c->d_r, Kc, S, c->hidden, 1, Kc, c->d_r, 1, (long long)Kc * c->d_r,
                    row, 1, 0};
    MLA_CUDA((gemm_simt<T, T, double, true>(g2, s)));
  }
  if (c->flags & MLA_FLAG_FP8_CACHE) {
    const size_t smem = sizeof(double) * (size_t)row;
    if (smem > 48 * 1024) return MLA_ERR_UNSUPPORTED;
    return st(launch_chained(append_finish_fp8_kernel, dim3(n), dim3(256), smem, s, (const double*)C, n, c->d_c,
                             c->d_r, c->rope_theta, seq_idx, pos, static_cast<__nv_fp8_e4m3*>(k->pool), k->row_scale,
                             k->block_table, k->batch, k->max_blocks_per_seq, k->num_blocks, c->block_size));
  }
  const long long total = (long long)n * (c->d_c + c->d_r / 2);
  return st(launch_chained(append_finish_kernel<T>, dim3(grid_for(total)), dim3(256), 0, s, (const double*)C, 1, n,
                            c->d_c, c->d_r, c->rope_theta, seq_idx, pos, static_cast<T*>(k->pool), k->block_table,
                            k->batch, k->max_blocks_per_seq, k->num_blocks, c->block_size));
}

// ---------------------------------------------------------------- absorb
// Query intermediates stay in fp32: with bf16 weights and fp32 activations the
// only rounding left on the query side is fp32 accumulation.
struct AbsorbWs {
  size_t cq_f, q_f, qn_f, total;
};
AbsorbWs absorb_ws(const mla_config* c, int n) {
  const size_t H = c->n_heads, qw = H * (c->qk_nope + c->d_r);
  AbsorbWs w{};
  size_t o = 0;
  w.cq_f = o; o = align_up(o + 4 * (size_t)n * c->q_lora, 256);
  w.q_f = o;  o = align_up(o + 4 * (size_t)n * qw, 256);
  w.qn_f = o; o = align_up(o + 4 * (size_t)n * H * c->qk_nope, 256);
  w.total = o;
  return w;
}

template <typename T>
mla_status absorb_impl(const mla_config* c, const void* x, int n, const void* W_DQ, const void* W_UQ,
                       const void* W_UK, const int32_t* pos, float* q_lat, float* q_rope, void* ws,
                       cudaStream_t s) {
  const AbsorbWs w = absorb_ws(c, n);
  char* base = static_cast<char*>(ws);
  float* cq_f = reinterpret_cast<float*>(base + w.cq_f);
  float* q_f = reinterpret_cast<float*>(base + w.q_f);
  float* qn_f = reinterpret_cast<float*>(base + w.qn_f);
  const int H = c->n_heads, nope = c->qk_nope, qw = H * (nope + c->d_r);
  if (c->q_lora > 0) {
    MLA_CUDA((gemm_rm<T, T, float>(x, c->hidden, W_DQ, c->q_lora, cq_f, c->q_lora, n, c->q_lora, c->hidden, s)));
    MLA_CUDA((gemm_rm<float, T, float>(cq_f, c->q_lora, W_UQ, qw, q_f, qw, n, qw, c->q_lora, s)));
  } else {
    MLA_CUDA((gemm_rm<T, T, float>(x, c->hidden, W_UQ, qw, q_f, qw, n, qw, c->hidden, s)));
  }
  const long long tot = (long long)n * H * (nope + c->d_r / 2);
  query_split_kernel<float><<<grid_for(tot), 256, 0, s>>>(q_f, n, H, nope, c->d_r, c->rope_theta, pos,
                                                          qn_f, q_rope);
  note_launch();
  MLA_CUDA(cudaGetLastError());
  // q_lat[t, h, :] = q_nope[t, h, :] W_UK_h^T, batched over heads
  GemmSimtArgs g{qn_f, W_UK, q_lat, n, c->d_c, nope, H,
                 (long long)H * nope, 1, nope,
                 1, (long long)H * nope, nope,
                 (long long)H * c->d_c, 1, c->d_c};
  MLA_CUDA((gemm_simt<float, T, float>(g, s)));
  return MLA_OK;
}

// ---------------------------------------------------------------- out proj
struct OutWs {
  size_t oh_f, y_f, total;
};
OutWs out_ws(const mla_config* c, int n) {
  const size_t H = c->n_heads;
  OutWs w{};
  size_t o = 0;
  w.oh_f = o; o = align_up(o + 4 * (size_t)n * H * c->v_head, 256);
  w.y_f = o;  o = align_up(o + 4 * (size_t)n * c->hidden, 256);
  w.total = o;
  return w;
}

template <typename T>
mla_status out_impl(const mla_config* c, const float* o_lat, int n, const void* W_UV, const void* W_O,
                    void* y, void* ws, cudaStream_t s) {
  const OutWs w = out_ws(c, n);
  char* base = static_cast<char*>(ws);
  float* oh_f = reinterpret_cast<float*>(base + w.oh_f);
  float* y_f = reinterpret_cast<float*>(base + w.y_f);
  const int H = c->n_heads, dv = c->v_head;
  // o_h[t, h, :] = o_lat[t, h, :] W_UV_h, batched over heads
  GemmSimtArgs g{o_lat, W_UV, oh_f, n, dv, c->d_c, H,
                 (long long)H * c->d_c, 1, c->d_c,
                 (long long)H * dv, 1, dv,
                 (long long)H * dv, 1, dv};
  MLA_CUDA((gemm_simt<float, T, float>(g, s)));
  MLA_CUDA((gemm_rm<float, T, float>(oh_f, (long long)H * dv, W_O, c->hidden, y_f, c->hidden, n, c->hidden, H * dv, s)));
  MLA_CUDA(round_store<T>(y_f, static_cast<T*>(y), (long long)n * c->hidden, s));
  return MLA_OK;
}

// Time limit of every bounded wait in the tensor-core kernels (process-wide).
std::atomic<unsigned long long> g_wait_limit_ns{sm100::kWaitLimitNs};

// ---------------------------------------------------------------- bf16 projections
// Tensor-core path of the query and output projections (weights bf16; see
// wgemm_tc.cuh).  Activations enter the MMAs in bf16; with the split-query
// flag the fp32 query intermediates enter as a bf16 hi + lo pair.
bool proj_tc_supported(const mla_config* c) {
  const long long qw = (long long)c->n_heads * (c->qk_nope + c->d_r);
  return c->hidden % 128 == 0 && (c->q_lora == 0 || c->q_lora % 128 == 0) && qw % 128 == 0 &&
         c->qk_nope % 64 == 0 && c->d_c % 128 == 0 && c->v_head % 128 == 0;
}

const bf16* const kSizeOnly = reinterpret_cast<const bf16*>(256);  // placeholder pointer for size queries

struct ProjSpecs {
  wg::Spec dq, uq, uk, uv, o;
};

ProjSpecs proj_specs(const mla_config* c, int n, bool split, const void* W_DQ, const void* W_UQ,
                     const void* W_UK, const void* W_UV, const void* W_O, const bf16* x, const bf16* cq_hi,
                     const bf16* cq_lo, const bf16* qn_hi, const bf16* qn_lo, const bf16* ol, const bf16* oh) {
  const int H = c->n_heads, nope = c->qk_nope, qw = H * (c->qk_nope + c->d_r);
  ProjSpecs p{};
  p.dq = wg::Spec{static_cast<const bf16*>(W_DQ), c->hidden, c->q_lora, 0, 1, c->q_lora, c->hidden, 0,
                  x, nullptr, c->hidden, 0, n};
  const int kq = c->q_lora > 0 ? c->q_lora : c->hidden;
  p.uq = wg::Spec{static_cast<const bf16*>(W_UQ), kq, qw, 0, 1, qw, kq, 0,
                  c->q_lora > 0 ? cq_hi : x, c->q_lora > 0 && split ? cq_lo : nullptr, kq, 0, n};
  p.uk = wg::Spec{static_cast<const bf16*>(W_UK), c->d_c, (long long)H * nope, 1, H, c->d_c, nope, nope,
                  qn_hi, split ? qn_lo : nullptr, (long long)H * nope, nope, n};
  p.uv = wg::Spec{static_cast<const bf16*>(W_UV), c->d_c, (long long)H * c->v_head, 0, H, c->v_head, c->d_c,
                  c->v_head, ol, nullptr, (long long)H * c->d_c, c->d_c, n};
  p.o = wg::Spec{static_cast<const bf16*>(W_O), (long long)H * c->v_head, c->hidden, 0, 1, c->hidden,
                 H * c->v_head, 0, oh, nullptr, (long long)H * c->v_head, 0, n};
  return p;
}

struct AbsorbTcWs {
  size_t part, cq_hi, cq_lo, q_f, qn_hi, qn_lo, total;
};
AbsorbTcWs absorb_tc_ws(const mla_config* c, int n) {
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  const ProjSpecs ps = proj_specs(c, n, split, nullptr, nullptr, nullptr, nullptr, nullptr, kSizeOnly, kSizeOnly,
                                  kSizeOnly, kSizeOnly, kSizeOnly, kSizeOnly, kSizeOnly);
  const size_t H = c->n_heads, qw = H * (c->qk_nope + c->d_r);
  size_t part = wg::run_partial_bytes(ps.uq);
  part = std::max(part, wg::run_partial_bytes(ps.uk));
  if (c->q_lora > 0) part = std::max(part, wg::run_partial_bytes(ps.dq));
  AbsorbTcWs w{};
  size_t o = 0;
  w.part = o;  o = align_up(o + part, 256);
  w.cq_hi = o; o = align_up(o + 2 * (size_t)n * c->q_lora, 256);
  w.cq_lo = o; o = align_up(o + (split ? 2 * (size_t)n * c->q_lora : 0), 256);
  w.q_f = o;   o = align_up(o + 4 * (size_t)n * qw, 256);
  w.qn_hi = o; o = align_up(o + 2 * (size_t)n * H * c->qk_nope, 256);
  w.qn_lo = o; o = align_up(o + (split ? 2 * (size_t)n * H * c->qk_nope : 0), 256);
  w.total = o;
  return w;
}

// Query side on the tensor cores.  Outputs either fp32 q_lat / q_rope, or
// (q_packed != nullptr) the decode's packed bf16 rows [n][H][d_c + d_r]
// (q_lat then the rotated q_R), followed in split-query mode by a second
// such array with the bf16 remainders.
mla_status absorb_tc(const mla_config* c, const void* x, int n, const void* W_DQ, const void* W_UQ,
                     const void* W_UK, const int32_t* pos, float* q_lat, float* q_rope, bf16* q_packed, void* ws,
                     cudaStream_t s) {
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  const AbsorbTcWs w = absorb_tc_ws(c, n);
  char* base = static_cast<char*>(ws);
  float* part = reinterpret_cast<float*>(base + w.part);
  bf16* cq_hi = reinterpret_cast<bf16*>(base + w.cq_hi);
  bf16* cq_lo = split ? reinterpret_cast<bf16*>(base + w.cq_lo) : nullptr;
  float* q_f = reinterpret_cast<float*>(base + w.q_f);
  bf16* qn_hi = reinterpret_cast<bf16*>(base + w.qn_hi);
  bf16* qn_lo = split ? reinterpret_cast<bf16*>(base + w.qn_lo) : nullptr;
  const ProjSpecs ps = proj_specs(c, n, split, W_DQ, W_UQ, W_UK, nullptr, nullptr, static_cast<const bf16*>(x),
                                  cq_hi, cq_lo, qn_hi, qn_lo, nullptr, nullptr);
  // W_UQ head slice, RoPE and W_UK in one kernel; its rotation table (in the
  // q_f region) depends on the positions only and is made first
  const bool fused = qh::supports(c, n);
  static_assert(sizeof(double) * 64 <= 4 * 192, "rotation table larger than the fp32 query it replaces");
  if (fused) MLA_TRY(qh::launch_rope_table(c, n, pos, reinterpret_cast<double*>(q_f), s));
  if (c->q_lora > 0) MLA_TRY(wg::run(ps.dq, part, nullptr, cq_hi, cq_lo, s));
  const int H = c->n_heads, nope = c->qk_nope, row = c->d_c + c->d_r;
  bf16* qp_lo = q_packed && split ? q_packed + (long long)n * H * row : nullptr;
  if (fused) {
    return qh::launch(c, n, cq_hi, cq_lo, static_cast<const bf16*>(W_UQ), static_cast<const bf16*>(W_UK), pos,
                      reinterpret_cast<double*>(q_f), q_packed, qp_lo, q_packed ? nullptr : q_lat,
                      q_packed ? nullptr : q_rope, g_wait_limit_ns.load(std::memory_order_relaxed), s);
  }
  MLA_TRY(wg::run(ps.uq, part, q_f, nullptr, nullptr, s));
  const dim3 qgrid(n, (H + kHeadGroup - 1) / kHeadGroup);
  MLA_CUDA(launch_chained(query_split_bf16_kernel, qgrid, dim3(256), sizeof(double) * c->d_r, s, (const float*)q_f, n, H,
                          nope, c->d_r, c->rope_theta, pos, qn_hi, qn_lo, q_rope, q_packed, qp_lo, row, c->d_c));
  if (q_packed == nullptr) return wg::run(ps.uk, part, q_lat, nullptr, nullptr, s);
  wg::Spec uk = ps.uk;  // q_lat of head h of token t -> packed row t H + h, columns [0, d_c)
  uk.o_ts = (long long)H * row;
  uk.o_gs = row;
  return wg::run(uk, part, nullptr, q_packed, qp_lo, s);
}

struct OutTcWs {
  size_t part, ol, oh, total;
};
OutTcWs out_tc_ws(const mla_config* c, int n) {
  const ProjSpecs ps = proj_specs(c, n, false, nullptr, nullptr, nullptr, nullptr, nullptr, kSizeOnly, kSizeOnly,
                                  kSizeOnly, kSizeOnly, kSizeOnly, kSizeOnly, kSizeOnly);
  const size_t H = c->n_heads;
  OutTcWs w{};
  size_t o = 0;
  w.part = o; o = align_up(o + std::max(wg::run_partial_bytes(ps.uv), wg::run_partial_bytes(ps.o)), 256);
  w.ol = o;   o = align_up(o + 2 * (size_t)n * H * c->d_c, 256);
  w.oh = o;   o = align_up(o + 2 * (size_t)n * H * c->v_head, 256);
  w.total = o;
  return w;
}

mla_status out_tc(const mla_config* c, const float* o_lat, int n, const void* W_UV, const void* W_O, void* y,
                  void* ws, cudaStream_t s) {
  const OutTcWs w = out_tc_ws(c, n);
  char* base = static_cast<char*>(ws);
  float* part = reinterpret_cast<float*>(base + w.part);
  bf16* ol = reinterpret_cast<bf16*>(base + w.ol);
  bf16* oh = reinterpret_cast<bf16*>(base + w.oh);
  const long long cnt = (long long)n * c->n_heads * c->d_c;
  MLA_CUDA(launch_chained(wg::split_bf16_kernel, dim3(grid_for(cnt / 4)), dim3(256), 0, s, o_lat, cnt, ol,
                          (bf16*)nullptr));
  const ProjSpecs ps = proj_specs(c, n, false, nullptr, nullptr, nullptr, W_UV, W_O, nullptr, nullptr, nullptr,
                                  nullptr, nullptr, ol, oh);
  MLA_TRY(wg::run(ps.uv, part, nullptr, oh, nullptr, s));
  return wg::run(ps.o, part, nullptr, static_cast<bf16*>(y), nullptr, s);
}

// ---------------------------------------------------------------- decode
// Parallel workers of the decode: one CTA pair per two SMs on the
// tensor-core path (bf16), two warps-worth of CTAs per SM on the CUDA-core path.
int default_workers(const mla_config* c) {
  const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
  if (tc_decode(c)) return std::max(1, sms / 2);
  return std::max(1, 2 * sms);
}

// The tensor-core decode reads the query as bf16 rows [H, d_c + d_r] that a
// first kernel packs from the fp32 inputs into the workspace.
size_t qpack_row_bytes(const mla_config* c) {
  return tc_decode(c) ? pairdec::qpack_row_bytes(c) : 0;
}

// Partial outputs of the split decode: bf16 from the tensor-core decode
// (they feed bf16 MMAs next), fp32 from the CUDA-core one.
int part_elem(const mla_config* c) { return tc_decode(c) ? 2 : 4; }


int resolve_workers(const mla_config* c, int max_workers) {
  return max_workers > 0 ? max_workers : default_workers(c);
}

template <typename T, int DPL>
void launch_decode_simt(const mla_config* c, const float* q_lat, const float* q_rope, int n_q,
                        const mla_cache* k, const int32_t* seq_lens, void* ws, const DecodeLayout& L,
                        cudaStream_t s) {
  const float scale_log2 = scale_of(c) * 1.4426950408889634f;
  dim3 grid(L.max_segments, (c->n_heads + 3) / 4);
  decode_simt_kernel<T, DPL><<<grid, 128, 0, s>>>(
      q_lat, q_rope, static_cast<const T*>(k->pool), fp8_cache(c) ? k->row_scale : nullptr,
      k->block_table, k->max_blocks_per_seq, k->num_blocks, seq_lens, n_q, c->n_heads, c->d_c, c->d_r,
      c->block_size, scale_log2, ws, L);
  note_launch();
}

template <typename T>
mla_status decode_simt_dispatch(const mla_config* c, const float* q_lat, const float* q_rope, int n_q,
                                const mla_cache* k, const int32_t* seq_lens, void* ws,
                                const DecodeLayout& L, cudaStream_t s) {
  const int row = c->d_c + c->d_r;
  if (row <= 96) launch_decode_simt<T, 3>(c, q_lat, q_rope, n_q, k, seq_lens, ws, L, s);
  else if (row <= 576) launch_decode_simt<T, 18>(c, q_lat, q_rope, n_q, k, seq_lens, ws, L, s);
  else if (row <= kSimtDecodeMaxRow) launch_decode_simt<T, 32>(c, q_lat, q_rope, n_q, k, seq_lens, ws, L, s);
  else return MLA_ERR_UNSUPPORTED;
  return st(cudaGetLastError());
}

// ------------------------------------------------- append without allocation
// Scratch of mla_cache_append_noalloc: a fixed device array that every GPU
// loading the library holds until the process exits.  In host code the name
// g_append_scratch is only a host-side stand-in for the device symbol, never a
// usable device address: the address comes from cudaGetSymbolAddress, taken
// once per device (with that device current) and cached below.
static __device__ __align__(256) unsigned char g_append_scratch[MLA_APPEND_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::atomic<void*> g_append_scratch_addr[kMaxDevices];
std::mutex g_append_scratch_mutex;

// Device address of this device's scratch array, looked up on first use.
mla_status append_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  void* p = g_append_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_append_scratch_mutex);
    p = g_append_scratch_addr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_append_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
      g_append_scratch_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return MLA_OK;
}

// A barrier that expects two arrivals and gets one: the bounded wait on it
// must give up after `limit_ns`, record MLA_ERR_TIMEOUT (where = 1) and return.
__global__ void wait_timeout_check_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 2);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    sm100::mbar_arrive(&bar);  // the second arrival never comes
    sm100::mbar_wait(&bar, 0, 1, limit_ns);
  }
}

}  // namespace

namespace {
mla_status combine_impl(const mla_config* cfg, const void* workspace, size_t ws_bytes, int32_t batch, int32_t n_q,
                        float* o_lat, float* lse, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (batch < 0 || n_q <= 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!workspace || !o_lat) return MLA_ERR_INVALID_ARG;
  if (ws_bytes < sizeof(DecodeHeader)) return MLA_ERR_WORKSPACE;
  if (!all_aligned16(workspace, o_lat)) return MLA_ERR_INVALID_ARG;
  if (lse != nullptr && ((uintptr_t)lse & 3u)) return MLA_ERR_INVALID_ARG;
  if (cfg->d_c % 8 != 0 || cfg->d_c / 8 > 256) return MLA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int per_head = cfg->d_c / 8, heads_per_block = 256 / per_head;
  dim3 grid(batch * n_q, (cfg->n_heads + heads_per_block - 1) / heads_per_block);
  return st(launch_chained(combine_kernel, grid, dim3(256), 0, s, (const void*)workspace, (long long)ws_bytes, batch,
                            n_q, cfg->n_heads, cfg->d_c, o_lat, lse));
}
}  // namespace

extern "C" {

int32_t mla_abi_version(void) { return MLA_ABI_VERSION; }

int64_t mla_kernel_launches(void) { return launch_counter().load(std::memory_order_relaxed); }

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported dimensions";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_BOUNDS: return "index out of bounds (device)";
    case MLA_ERR_TIMEOUT: return "bounded wait timed out (device)";
    case MLA_ERR_WORKSPACE: return "workspace too small or not written by mla_decode";
  }
  return "unknown status";
}

size_t mla_cache_append_workspace_size(const mla_config* cfg, int32_t n_tok) {
  if (check_cfg(cfg) != MLA_OK || n_tok < 0) return 0;
  return append_ws(cfg, n_tok);
}

mla_status mla_cache_append(const mla_config* cfg, const void* x, int32_t n_tok, const void* W_DKV,
                            const void* W_KR, const int32_t* seq_idx, const int32_t* pos,
                            const mla_cache* cache, void* workspace, size_t ws_bytes, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (n_tok < 0) return MLA_ERR_INVALID_ARG;
  if (n_tok == 0) return MLA_OK;
  if (!x || !W_DKV || !W_KR || !seq_idx || !pos || !workspace) return MLA_ERR_INVALID_ARG;
  MLA_TRY(check_cache(cfg, cache));
  if (ws_bytes < append_ws(cfg, n_tok)) return MLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == MLA_BF16)
    return append_impl<bf16>(cfg, x, n_tok, W_DKV, W_KR, seq_idx, pos, cache, workspace, s);
  return append_impl<float>(cfg, x, n_tok, W_DKV, W_KR, seq_idx, pos, cache, workspace, s);
}

mla_status mla_cache_append_noalloc(const mla_config* cfg, const void* x, int32_t n_tok, const void* W_DKV,
                                    const void* W_KR, const int32_t* seq_idx, const int32_t* pos,
                                    const mla_cache* cache, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (n_tok < 0) return MLA_ERR_INVALID_ARG;
  if (n_tok == 0) return MLA_OK;
  if (!x || !W_DKV || !W_KR || !seq_idx || !pos) return MLA_ERR_INVALID_ARG;
  MLA_TRY(check_cache(cfg, cache));
  const size_t need = append_ws(cfg, n_tok);
  if (need > (size_t)MLA_APPEND_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  MLA_TRY(append_scratch_address(&scratch));
  // The append clears the part of the scratch it accumulates into at the start
  // of every call, so nothing left over from an earlier call leaks in.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == MLA_BF16)
    return append_impl<bf16>(cfg, x, n_tok, W_DKV, W_KR, seq_idx, pos, cache, scratch, s);
  return append_impl<float>(cfg, x, n_tok, W_DKV, W_KR, seq_idx, pos, cache, scratch, s);
}

size_t mla_absorb_q_workspace_size(const mla_config* cfg, int32_t n_tok) {
  if (check_cfg(cfg) != MLA_OK || n_tok < 0) return 0;
  if (cfg->dtype == MLA_BF16) return proj_tc_supported(cfg) ? absorb_tc_ws(cfg, n_tok).total : 0;
  return absorb_ws(cfg, n_tok).total;
}

mla_status mla_absorb_q(const mla_config* cfg, const void* x, int32_t n_tok, const void* W_DQ,
                        const void* W_UQ, const void* W_UK, const int32_t* pos, float* q_lat,
                        float* q_rope, void* workspace, size_t ws_bytes, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (n_tok < 0) return MLA_ERR_INVALID_ARG;
  if (n_tok == 0) return MLA_OK;
  if (!x || !W_UQ || !W_UK || !pos || !q_lat || !q_rope || !workspace) return MLA_ERR_INVALID_ARG;
  if ((cfg->q_lora > 0) != (W_DQ != nullptr)) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == MLA_BF16) {
    if (!proj_tc_supported(cfg)) return MLA_ERR_UNSUPPORTED;
    if (!all_aligned16(x, W_DQ, W_UQ, W_UK, q_lat, q_rope, workspace)) return MLA_ERR_INVALID_ARG;
    if (ws_bytes < absorb_tc_ws(cfg, n_tok).total) return MLA_ERR_WORKSPACE;
    return absorb_tc(cfg, x, n_tok, W_DQ, W_UQ, W_UK, pos, q_lat, q_rope, nullptr, workspace, s);
  }
  if (ws_bytes < absorb_ws(cfg, n_tok).total) return MLA_ERR_WORKSPACE;
  return absorb_impl<float>(cfg, x, n_tok, W_DQ, W_UQ, W_UK, pos, q_lat, q_rope, workspace, s);
}

size_t mla_fp8_scratch_bytes(const mla_config* cfg, int32_t batch, int32_t max_blocks_per_seq) {
  if (check_cfg(cfg) != MLA_OK || !fp8_cache(cfg) || batch < 0 || max_blocks_per_seq <= 0) return 0;
  const size_t slots = (size_t)batch * max_blocks_per_seq;
  return align_up(4 * slots, 256) + slots * cfg->block_size * (cfg->d_c + cfg->d_r) * 2;
}

mla_status mla_cache_dequant_fp8(const mla_config* cfg, const mla_cache* cache, int32_t batch,
                                 const int32_t* seq_lens, void* scratch, size_t scratch_bytes, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (!fp8_cache(cfg) || batch < 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!seq_lens || !scratch) return MLA_ERR_INVALID_ARG;
  MLA_TRY(check_cache(cfg, cache));
  if (cache->batch < batch) return MLA_ERR_INVALID_ARG;
  const int row = cfg->d_c + cfg->d_r;
  if (row % 16 != 0) return MLA_ERR_UNSUPPORTED;
  if (!all_aligned16(cache->pool, scratch)) return MLA_ERR_INVALID_ARG;
  if (scratch_bytes < mla_fp8_scratch_bytes(cfg, batch, cache->max_blocks_per_seq)) return MLA_ERR_WORKSPACE;
  const size_t slots = (size_t)batch * cache->max_blocks_per_seq;
  int32_t* table = static_cast<int32_t*>(scratch);
  bf16* pages = reinterpret_cast<bf16*>(static_cast<char*>(scratch) + align_up(4 * slots, 256));
  return st(launch_chained(dequant_fp8_pages_kernel, dim3(cache->max_blocks_per_seq, batch), dim3(256), 0,
                           static_cast<cudaStream_t>(stream), static_cast<const uint8_t*>(cache->pool),
                           (const float*)cache->row_scale, cache->block_table, cache->num_blocks, seq_lens,
                           cache->max_blocks_per_seq, cfg->block_size, row, pages, table));
}

size_t mla_query_packed_bytes(const mla_config* cfg, int32_t n_tok) {
  if (check_cfg(cfg) != MLA_OK || n_tok < 0 || !tc_decode(cfg)) return 0;
  return (size_t)n_tok * pairdec::qpack_row_bytes(cfg);
}

mla_status mla_absorb_q_packed(const mla_config* cfg, const void* x, int32_t n_tok, const void* W_DQ,
                               const void* W_UQ, const void* W_UK, const int32_t* pos, void* q_packed,
                               void* workspace, size_t ws_bytes, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (n_tok < 0) return MLA_ERR_INVALID_ARG;
  if (n_tok == 0) return MLA_OK;
  if (!x || !W_UQ || !W_UK || !pos || !q_packed || !workspace) return MLA_ERR_INVALID_ARG;
  if ((cfg->q_lora > 0) != (W_DQ != nullptr)) return MLA_ERR_INVALID_ARG;
  if (cfg->dtype != MLA_BF16 || !proj_tc_supported(cfg) || !pairdec::supports(cfg)) return MLA_ERR_UNSUPPORTED;
  if (!all_aligned16(x, W_DQ, W_UQ, W_UK, q_packed, workspace)) return MLA_ERR_INVALID_ARG;
  if (ws_bytes < absorb_tc_ws(cfg, n_tok).total) return MLA_ERR_WORKSPACE;
  return absorb_tc(cfg, x, n_tok, W_DQ, W_UQ, W_UK, pos, nullptr, nullptr, static_cast<bf16*>(q_packed), workspace,
                   static_cast<cudaStream_t>(stream));
}

static mla_status decode_packed_impl(const mla_config* cfg, const void* q_packed, int32_t batch, int32_t n_q,
                                     const mla_cache* cache, const int32_t* seq_lens, int32_t max_workers,
                                     void* workspace, size_t ws_bytes, void* stream, bool planned) {
  MLA_TRY(check_cfg(cfg));
  if (batch < 0 || n_q <= 0 || max_workers < 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!q_packed || !seq_lens || !workspace) return MLA_ERR_INVALID_ARG;
  if ((long long)batch * n_q > kPlanMaxRows) return MLA_ERR_UNSUPPORTED;
  MLA_TRY(check_cache(cfg, cache));
  if (cache->batch < batch) return MLA_ERR_INVALID_ARG;
  if (cfg->dtype != MLA_BF16 || !pairdec::supports(cfg)) return MLA_ERR_UNSUPPORTED;
  if (!all_aligned16(q_packed, cache->pool, workspace)) return MLA_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(batch, n_q, cfg->n_heads, cfg->d_c, resolve_workers(cfg, max_workers),
                                       qpack_row_bytes(cfg), part_elem(cfg));
  if (ws_bytes < (size_t)L.total) return MLA_ERR_WORKSPACE;
  return pairdec::launch(cfg, nullptr, nullptr, static_cast<const bf16*>(q_packed), n_q, cache, seq_lens, workspace,
                         L, scale_of(cfg), g_wait_limit_ns.load(std::memory_order_relaxed),
                         static_cast<cudaStream_t>(stream), planned);
}

mla_status mla_decode_packed(const mla_config* cfg, const void* q_packed, int32_t batch, int32_t n_q,
                             const mla_cache* cache, const int32_t* seq_lens, int32_t max_workers, void* workspace,
                             size_t ws_bytes, void* stream) {
  return decode_packed_impl(cfg, q_packed, batch, n_q, cache, seq_lens, max_workers, workspace, ws_bytes, stream,
                            false);
}

mla_status mla_decode_packed_planned(const mla_config* cfg, const void* q_packed, int32_t batch, int32_t n_q,
                                     const mla_cache* cache, const int32_t* seq_lens, int32_t max_workers,
                                     void* workspace, size_t ws_bytes, void* stream) {
  return decode_packed_impl(cfg, q_packed, batch, n_q, cache, seq_lens, max_workers, workspace, ws_bytes, stream,
                            true);
}

mla_status mla_decode_plan(const mla_config* cfg, int32_t batch, int32_t n_q, const mla_cache* cache,
                           const int32_t* seq_lens, int32_t max_workers, void* workspace, size_t ws_bytes,
                           void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (batch < 0 || n_q <= 0 || max_workers < 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!seq_lens || !workspace) return MLA_ERR_INVALID_ARG;
  if ((long long)batch * n_q > kPlanMaxRows) return MLA_ERR_UNSUPPORTED;
  MLA_TRY(check_cache(cfg, cache));
  if (cache->batch < batch) return MLA_ERR_INVALID_ARG;
  if (!all_aligned16(workspace)) return MLA_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(batch, n_q, cfg->n_heads, cfg->d_c, resolve_workers(cfg, max_workers),
                                       qpack_row_bytes(cfg), part_elem(cfg));
  if (ws_bytes < (size_t)L.total) return MLA_ERR_WORKSPACE;
  const size_t plan_smem = sizeof(int) * ((size_t)batch * n_q + 1);
  static std::atomic<uint64_t> attr{0};
  if (plan_smem > 48 * 1024 && pairdec::set_smem_once((const void*)decode_plan_kernel, plan_smem, attr) != MLA_OK)
    return MLA_ERR_CUDA;
  MLA_CUDA(launch_chained(decode_plan_kernel, dim3(1), dim3(1024), plan_smem, static_cast<cudaStream_t>(stream),
                          seq_lens, cfg->block_size, cache->max_blocks_per_seq, workspace, L));
  return MLA_OK;
}

size_t mla_decode_workspace_size(const mla_config* cfg, int32_t batch, int32_t n_q, int32_t max_workers) {
  if (check_cfg(cfg) != MLA_OK || batch < 0 || n_q <= 0 || max_workers < 0) return 0;
  return (size_t)decode_layout(batch, n_q, cfg->n_heads, cfg->d_c, resolve_workers(cfg, max_workers),
                               qpack_row_bytes(cfg), part_elem(cfg))
      .total;
}

mla_status mla_decode(const mla_config* cfg, const float* q_lat, const float* q_rope, int32_t batch,
                      int32_t n_q, const mla_cache* cache, const int32_t* seq_lens, int32_t max_workers,
                      void* workspace, size_t ws_bytes, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (batch < 0 || n_q <= 0 || max_workers < 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!q_lat || !q_rope || !seq_lens || !workspace) return MLA_ERR_INVALID_ARG;
  if ((long long)batch * n_q > kPlanMaxRows) return MLA_ERR_UNSUPPORTED;
  MLA_TRY(check_cache(cfg, cache));
  if (cache->batch < batch) return MLA_ERR_INVALID_ARG;
  if (tc_decode(cfg) && !pairdec::supports(cfg)) return MLA_ERR_UNSUPPORTED;
  if (tc_decode(cfg) && !all_aligned16(q_lat, q_rope, cache->pool, workspace)) return MLA_ERR_INVALID_ARG;
  const DecodeLayout L =
      decode_layout(batch, n_q, cfg->n_heads, cfg->d_c, resolve_workers(cfg, max_workers), qpack_row_bytes(cfg),
                    part_elem(cfg));
  if (ws_bytes < (size_t)L.total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tc_decode(cfg))
    return pairdec::launch(cfg, q_lat, q_rope, nullptr, n_q, cache, seq_lens, workspace, L, scale_of(cfg),
                           g_wait_limit_ns.load(std::memory_order_relaxed), s);
  const size_t plan_smem = sizeof(int) * ((size_t)batch * n_q + 1);
  if (plan_smem > 48 * 1024 &&
      cudaFuncSetAttribute(decode_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan_smem) !=
          cudaSuccess)
    return MLA_ERR_CUDA;
  MLA_CUDA(launch_chained(decode_plan_kernel, dim3(1), dim3(1024), plan_smem, s, seq_lens, cfg->block_size,
                          cache->max_blocks_per_seq, workspace, L));
  if (fp8_cache(cfg))
    return decode_simt_dispatch<__nv_fp8_e4m3>(cfg, q_lat, q_rope, n_q, cache, seq_lens, workspace, L, s);
  return decode_simt_dispatch<float>(cfg, q_lat, q_rope, n_q, cache, seq_lens, workspace, L, s);
}

mla_status mla_combine(const mla_config* cfg, const void* workspace, size_t ws_bytes, int32_t batch,
                       int32_t n_q, float* o_lat, void* stream) {
  return combine_impl(cfg, workspace, ws_bytes, batch, n_q, o_lat, nullptr, stream);
}

mla_status mla_combine_lse(const mla_config* cfg, const void* workspace, size_t ws_bytes, int32_t batch,
                           int32_t n_q, float* o_lat, float* lse, void* stream) {
  if (lse == nullptr) return MLA_ERR_INVALID_ARG;
  return combine_impl(cfg, workspace, ws_bytes, batch, n_q, o_lat, lse, stream);
}

mla_status mla_merge_shards(const mla_config* cfg, int32_t n_shards, int32_t rows, const float* o_parts,
                            const float* lse_parts, float* o_lat, float* lse, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (n_shards <= 0 || rows < 0) return MLA_ERR_INVALID_ARG;
  if (rows == 0) return MLA_OK;
  if (!o_parts || !lse_parts || !o_lat) return MLA_ERR_INVALID_ARG;
  if (!all_aligned16(o_parts, o_lat) || ((uintptr_t)lse_parts & 3u) || (lse != nullptr && ((uintptr_t)lse & 3u)))
    return MLA_ERR_INVALID_ARG;
  if (cfg->d_c % 8 != 0 || cfg->d_c / 8 > 256) return MLA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int per_head = cfg->d_c / 8, heads_per_block = 256 / per_head;
  dim3 grid(rows, (cfg->n_heads + heads_per_block - 1) / heads_per_block);
  return st(launch_chained(merge_shards_kernel, grid, dim3(256), 0, s, o_parts, lse_parts, (int)n_shards, (int)rows,
                            cfg->n_heads, cfg->d_c, o_lat, lse));
}

size_t mla_combine_out_proj_workspace_size(const mla_config* cfg, int32_t batch, int32_t n_q) {
  if (check_cfg(cfg) != MLA_OK || batch < 0 || n_q <= 0 || cfg->dtype != MLA_BF16 || !proj_tc_supported(cfg))
    return 0;
  if ((long long)batch * n_q > kPlanMaxRows) return 0;
  // the merge takes up to ocomb::kMaxN segments (rows plus the plan's extra cuts) in one launch
  const DecodeLayout L = decode_layout(batch, n_q, cfg->n_heads, cfg->d_c, resolve_workers(cfg, 0),
                                       qpack_row_bytes(cfg), part_elem(cfg));
  if (!pairdec::supports(cfg) || !ocomb::supports(cfg, L.max_segments)) return 0;
  const int n = batch * n_q;
  const ProjSpecs ps = proj_specs(cfg, n, false, nullptr, nullptr, nullptr, nullptr, nullptr, kSizeOnly, kSizeOnly,
                                  kSizeOnly, kSizeOnly, kSizeOnly, kSizeOnly, kSizeOnly);
  return align_up(2 * (size_t)n * cfg->n_heads * cfg->v_head, 256) + align_up(wg::run_partial_bytes(ps.o), 256);
}

mla_status mla_combine_out_proj(const mla_config* cfg, const void* decode_ws, size_t decode_ws_bytes, int32_t batch,
                                int32_t n_q, int32_t max_workers, const void* W_UV, const void* W_O, void* y,
                                void* workspace, size_t ws_bytes, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (batch < 0 || n_q <= 0 || max_workers < 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  if (!decode_ws || !W_UV || !W_O || !y || !workspace) return MLA_ERR_INVALID_ARG;
  if (cfg->dtype != MLA_BF16 || !proj_tc_supported(cfg) || !pairdec::supports(cfg)) return MLA_ERR_UNSUPPORTED;
  if (!all_aligned16(decode_ws, W_UV, W_O, y, workspace)) return MLA_ERR_INVALID_ARG;
  if ((long long)batch * n_q > kPlanMaxRows) return MLA_ERR_UNSUPPORTED;
  const DecodeLayout L = decode_layout(batch, n_q, cfg->n_heads, cfg->d_c, resolve_workers(cfg, max_workers),
                                       qpack_row_bytes(cfg), part_elem(cfg));
  if (decode_ws_bytes < (size_t)L.total) return MLA_ERR_WORKSPACE;
  if (!ocomb::supports(cfg, L.max_segments)) return MLA_ERR_UNSUPPORTED;
  if (ws_bytes < mla_combine_out_proj_workspace_size(cfg, batch, n_q)) return MLA_ERR_WORKSPACE;
  const int n = batch * n_q;
  char* base = static_cast<char*>(workspace);
  bf16* oh = reinterpret_cast<bf16*>(base);
  float* part = reinterpret_cast<float*>(base + align_up(2 * (size_t)n * cfg->n_heads * cfg->v_head, 256));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MLA_TRY(ocomb::launch(cfg, W_UV, decode_ws, decode_ws_bytes, L, oh, s));
  const ProjSpecs ps = proj_specs(cfg, n, false, nullptr, nullptr, nullptr, W_UV, W_O, nullptr, nullptr, nullptr,
                                  nullptr, nullptr, nullptr, oh);
  return wg::run(ps.o, part, nullptr, static_cast<bf16*>(y), nullptr, s);
}

size_t mla_out_proj_workspace_size(const mla_config* cfg, int32_t n_tok) {
  if (check_cfg(cfg) != MLA_OK || n_tok < 0) return 0;
  if (cfg->dtype == MLA_BF16) return proj_tc_supported(cfg) ? out_tc_ws(cfg, n_tok).total : 0;
  return out_ws(cfg, n_tok).total;
}

mla_status mla_out_proj(const mla_config* cfg, const float* o_lat, int32_t n_tok, const void* W_UV,
                        const void* W_O, void* y, void* workspace, size_t ws_bytes, void* stream) {
  MLA_TRY(check_cfg(cfg));
  if (n_tok < 0) return MLA_ERR_INVALID_ARG;
  if (n_tok == 0) return MLA_OK;
  if (!o_lat || !W_UV || !W_O || !y || !workspace) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->dtype == MLA_BF16) {
    if (!proj_tc_supported(cfg)) return MLA_ERR_UNSUPPORTED;
    if (!all_aligned16(o_lat, W_UV, W_O, y, workspace)) return MLA_ERR_INVALID_ARG;
    if (ws_bytes < out_tc_ws(cfg, n_tok).total) return MLA_ERR_WORKSPACE;
    return out_tc(cfg, o_lat, n_tok, W_UV, W_O, y, workspace, s);
  }
  if (ws_bytes < out_ws(cfg, n_tok).total) return MLA_ERR_WORKSPACE;
  return out_impl<float>(cfg, o_lat, n_tok, W_UV, W_O, y, workspace, s);
}

mla_status mla_check_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > 10000000000LL) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  wait_timeout_check_kernel<<<1, 32, 0, s>>>((unsigned long long)limit_ns);
  note_launch();
  return st(cudaGetLastError());
}

mla_status mla_get_device_error(void* stream, int32_t* detail) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
  int h[4] = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbol(h, g_err, sizeof(h)) != cudaSuccess) return MLA_ERR_CUDA;
  if (h[0] != 0) {
    const int zero[4] = {0, 0, 0, 0};
    if (cudaMemcpyToSymbol(g_err, zero, sizeof(zero)) != cudaSuccess) return MLA_ERR_CUDA;
  }
  if (detail) {
    detail[0] = h[1];
    detail[1] = h[2];
    detail[2] = h[3];
  }
  return static_cast<mla_status>(h[0]);
}

}  // extern "C"

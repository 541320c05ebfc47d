// Epilogue kernels of the projection steps: storage rounding, decoupled RoPE,
// the paged-cache scatter of new latent rows, and the query split.
#pragma once

#include "common.cuh"

namespace mla {

// Round an fp32 buffer to the storage type.
template <typename T>
__global__ void round_store_kernel(const float* __restrict__ src, T* __restrict__ dst, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    Store<T>::st(dst + i, src[i]);
}

template <typename T>
static cudaError_t round_store(const float* src, T* dst, long long n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int blocks = (int)std::min<long long>((n + 255) / 256, 4096);
  round_store_kernel<T><<<blocks, 256, 0, s>>>(src, dst, n);
  note_launch();
  return cudaGetLastError();
}

// Where token t's cache row goes, or -1 after recording a bounds error.
__device__ __forceinline__ long long cache_row_slot(const int32_t* seq_idx, const int32_t* pos, int t,
                                                    const int32_t* block_table, int batch,
                                                    int max_blocks, int num_blocks, int bs) {
  const int b = seq_idx[t], p = pos[t];
  if (b < 0 || b >= batch || p < 0) {
    report(MLA_ERR_BOUNDS, 1, t, p);
    return -1;
  }
  const int page = p / bs;
  if (page >= max_blocks) {
    report(MLA_ERR_BOUNDS, 2, t, p);
    return -1;
  }
  const int phys = block_table[(long long)b * max_blocks + page];
  if (phys < 0 || phys >= num_blocks) {
    report(MLA_ERR_BOUNDS, 3, t, phys);
    return -1;
  }
  return (long long)phys * bs + (p % bs);
}

// New latent rows from exact (fp64) projections C = x [W_DKV | W_KR] (the sum
// of `splits` fp64 partials over K):
// c = C[:, :d_c], k_R = RoPE(C[:, d_c:], pos); each value rounded once to T
// and written to its paged slot.  One thread per latent value or rotary pair.
template <typename T>
__global__ void append_finish_kernel(const double* __restrict__ C, int splits, int n_tok, int d_c, int d_r,
                                     double theta, const int32_t* __restrict__ seq_idx,
                                     const int32_t* __restrict__ pos, T* __restrict__ pool,
                                     const int32_t* __restrict__ block_table, int batch,
                                     int max_blocks, int num_blocks, int bs) {
  pdl_wait();
  pdl_trigger();
  const int per_tok = d_c + d_r / 2;
  const long long total = (long long)n_tok * per_tok;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_tok), k = (int)(i % per_tok);
    const long long slot = cache_row_slot(seq_idx, pos, t, block_table, batch, max_blocks, num_blocks, bs);
    if (slot < 0) continue;
    const int row = d_c + d_r;
    const long long split_stride = (long long)n_tok * row;
    const double* src = C + (long long)t * row;
    auto total = [&](int col) {
      double acc = 0.0;
      for (int s = 0; s < splits; ++s) acc += src[s * split_stride + col];
      return acc;
    };
    T* dst = pool + slot * row;
    if (k < d_c) {
      Store<T>::st64(dst + k, total(k));
    } else {
      const int pr = k - d_c;  // rotary pair index
      const double ang = (double)pos[t] * rope_inv_freq(theta, pr, d_r);
      double sn, cs;
      sincos(ang, &sn, &cs);
      const double r0 = total(d_c + 2 * pr), r1 = total(d_c + 2 * pr + 1);
      Store<T>::st64(dst + d_c + 2 * pr, r0 * cs - r1 * sn);
      Store<T>::st64(dst + d_c + 2 * pr + 1, r0 * sn + r1 * cs);
    }
  }
}

// The same epilogue into an FP8 cache: one CTA per new token assembles its
// exact row [c | RoPE(k_R)] in fp64 (shared memory), takes the row's largest
// magnitude m, the scale s = the smallest power of two with m / s <= 448 (1
// if m is 0) and writes the E4M3 codes of row / s (nearest, ties to even)
// and s.  A power-of-two scale keeps code * s exact in bf16.
__global__ void __launch_bounds__(256) append_finish_fp8_kernel(
    const double* __restrict__ C, int n_tok, int d_c, int d_r, double theta, const int32_t* __restrict__ seq_idx,
    const int32_t* __restrict__ pos, __nv_fp8_e4m3* __restrict__ pool, float* __restrict__ row_scale,
    const int32_t* __restrict__ block_table, int batch, int max_blocks, int num_blocks, int bs) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ double v[];  // [d_c + d_r]
  __shared__ double warp_max[8];
  __shared__ long long slot_s;
  const int t = blockIdx.x, row = d_c + d_r;
  if (t >= n_tok) return;
  if (threadIdx.x == 0) slot_s = cache_row_slot(seq_idx, pos, t, block_table, batch, max_blocks, num_blocks, bs);
  const double* src = C + (long long)t * row;
  for (int k = threadIdx.x; k < d_c + d_r / 2; k += blockDim.x) {
    if (k < d_c) {
      v[k] = src[k];
    } else {
      const int pr = k - d_c;  // rotary pair index
      double sn, cs;
      sincos((double)pos[t] * rope_inv_freq(theta, pr, d_r), &sn, &cs);
      const double r0 = src[d_c + 2 * pr], r1 = src[d_c + 2 * pr + 1];
      v[d_c + 2 * pr] = r0 * cs - r1 * sn;
      v[d_c + 2 * pr + 1] = r0 * sn + r1 * cs;
    }
  }
  __syncthreads();
  double m = 0.0;
  for (int k = threadIdx.x; k < row; k += blockDim.x) m = fmax(m, fabs(v[k]));
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  const long long slot = slot_s;
  if (slot < 0) return;
  m = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmax(m, warp_max[w]);
  // the smallest power of two s with m / s <= 448 (1 for a zero row)
  int e = 0;
  const double f = frexp(m / 448.0, &e);  // m / 448 = f 2^e, 0.5 <= f < 1
  float scale = m > 0.0 ? (float)ldexp(1.0, f == 0.5 ? e - 1 : e) : 1.f;
  if (scale == 0.f) scale = 1.f;
  __nv_fp8_e4m3* dst = pool + slot * row;
  for (int k = threadIdx.x; k < row; k += blockDim.x) Store<__nv_fp8_e4m3>::st64(dst + k, v[k] / (double)scale);
  if (threadIdx.x == 0) row_scale[slot] = scale;
}

// FP8 cache pages -> bf16 pages for the tensor-core decode: page k of
// sequence b (if visible) becomes scratch page b * max_blocks + k, each value
// code * row scale rounded once to bf16, and the scratch block table entry
// (b, k) = b * max_blocks + k.  Grid (max_blocks, batch); 16 codes per step.
__global__ void __launch_bounds__(256) dequant_fp8_pages_kernel(
    const uint8_t* __restrict__ pool, const float* __restrict__ row_scale, const int32_t* __restrict__ block_table,
    int num_blocks, const int32_t* __restrict__ seq_lens, int max_blocks, int bs, int row,
    bf16* __restrict__ out_pool, int32_t* __restrict__ out_table) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y, k = blockIdx.x;
  const long long slot = (long long)b * max_blocks + k;
  if (threadIdx.x == 0) out_table[slot] = (int32_t)slot;
  const int len = seq_lens[b];
  if (len < 0 || len > max_blocks * bs) {
    if (k == 0 && threadIdx.x == 0) report(MLA_ERR_BOUNDS, 6, b, len);
    return;
  }
  const int rows = min(bs, len - k * bs);
  if (rows <= 0) return;
  const int phys = block_table[slot];
  if (phys < 0 || phys >= num_blocks) {
    if (threadIdx.x == 0) report(MLA_ERR_BOUNDS, 7, b, phys);
    return;
  }
  const uint8_t* src = pool + (long long)phys * bs * row;
  const float* sc = row_scale + (long long)phys * bs;
  bf16* dst = out_pool + slot * bs * row;
  const int per_row = row / 16, chunks = rows * per_row;
  // kAhead 16-byte loads in flight per thread before any conversion
  constexpr int kAhead = 4;
  for (int c0 = threadIdx.x; c0 < chunks; c0 += kAhead * blockDim.x) {
    uint4 buf[kAhead];
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      const int c = c0 + j * blockDim.x;
      if (c < chunks) buf[j] = __ldcs(reinterpret_cast<const uint4*>(src + (long long)c * 16));
    }
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      const int c = c0 + j * blockDim.x;
      if (c >= chunks) break;
      const float s = sc[c / per_row];
      const uint4 in = buf[j];
      const uint32_t w[4] = {in.x, in.y, in.z, in.w};
      uint32_t out[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        __nv_fp8_e4m3 lo, hi;
        lo.__x = (__nv_fp8_storage_t)((w[i >> 1] >> (16 * (i & 1))) & 0xFFu);
        hi.__x = (__nv_fp8_storage_t)((w[i >> 1] >> (16 * (i & 1) + 8)) & 0xFFu);
        // code * scale is exact in fp64 (4 + 24 significant bits): one rounding to bf16
        const bf16 va = __double2bfloat16((double)static_cast<float>(lo) * (double)s);
        const bf16 vb = __double2bfloat16((double)static_cast<float>(hi) * (double)s);
        out[i] = (uint32_t)__bfloat16_as_ushort(va) | ((uint32_t)__bfloat16_as_ushort(vb) << 16);
      }
      uint4* o = reinterpret_cast<uint4*>(dst + (long long)c * 16);
      o[0] = make_uint4(out[0], out[1], out[2], out[3]);
      o[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
  }
}

// Split q [n, H, nope + d_r] (fp32) into q_nope (storage type) and the rotated
// q_rope (storage type).  The RoPE angle and rotation are evaluated in fp64.
template <typename T>
__global__ void query_split_kernel(const float* __restrict__ q, int n_tok, int H, int nope, int d_r,
                                   double theta, const int32_t* __restrict__ pos,
                                   T* __restrict__ q_nope, T* __restrict__ q_rope) {
  const int w = nope + d_r;
  const int per_head = nope + d_r / 2;
  const long long total = (long long)n_tok * H * per_head;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long th = i / per_head;  // t * H + h
    const int k = (int)(i % per_head);
    const int t = (int)(th / H);
    const float* src = q + th * w;
    if (k < nope) {
      Store<T>::st(q_nope + th * nope + k, src[k]);
    } else {
      const int pr = k - nope;
      const double ang = (double)pos[t] * rope_inv_freq(theta, pr, d_r);
      double sn, cs;
      sincos(ang, &sn, &cs);
      const double r0 = src[nope + 2 * pr], r1 = src[nope + 2 * pr + 1];
      Store<T>::st(q_rope + th * d_r + 2 * pr, (float)(r0 * cs - r1 * sn));
      Store<T>::st(q_rope + th * d_r + 2 * pr + 1, (float)(r0 * sn + r1 * cs));
    }
  }
}

// Split q [n, H, nope + d_r] (fp32): q_nope to bf16 (and its bf16 remainder
// when lo != nullptr), the rotated q_rope (angle and rotation in fp64) kept
// in fp32 (q_rope) and/or written as bf16 (and its remainder) into columns
// [rope_col, rope_col + d_r) of the packed query rows of `row` values
// (qp_hi / qp_lo).  One block per (token, group of kHeadGroup heads): the
// token's d_r/2 rotation angles are evaluated once into shared memory and
// shared by every head.  Needs even nope and d_r (pairs are read and written
// together).
constexpr int kHeadGroup = 8;
__global__ void query_split_bf16_kernel(const float* __restrict__ q, int n_tok, int H, int nope, int d_r,
                                        double theta, const int32_t* __restrict__ pos, bf16* __restrict__ q_nope,
                                        bf16* __restrict__ q_nope_lo, float* __restrict__ q_rope,
                                        bf16* __restrict__ qp_hi, bf16* __restrict__ qp_lo, int row, int rope_col) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ double rot[];  // [d_r/2][cos, sin]
  const int t = blockIdx.x, half = d_r / 2, w = nope + d_r;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    double sn, cs;
    sincos((double)pos[t] * rope_inv_freq(theta, i, d_r), &sn, &cs);
    rot[2 * i] = cs;
    rot[2 * i + 1] = sn;
  }
  __syncthreads();
  const int h0 = blockIdx.y * kHeadGroup, nh = min(kHeadGroup, H - h0);
  const int np = nope / 2;
  for (int e = threadIdx.x; e < nh * np; e += blockDim.x) {
    const long long th = (long long)t * H + h0 + e / np;
    const int k = 2 * (e % np);
    const float2 v = *reinterpret_cast<const float2*>(q + th * w + k);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(v.x, v.y);
    *reinterpret_cast<__nv_bfloat162*>(q_nope + th * nope + k) = hi;
    if (q_nope_lo)
      *reinterpret_cast<__nv_bfloat162*>(q_nope_lo + th * nope + k) =
          __floats2bfloat162_rn(v.x - __bfloat162float(hi.x), v.y - __bfloat162float(hi.y));
  }
  for (int e = threadIdx.x; e < nh * half; e += blockDim.x) {
    const long long th = (long long)t * H + h0 + e / half;
    const int pr = e % half;
    const float2 r = *reinterpret_cast<const float2*>(q + th * w + nope + 2 * pr);
    const double cs = rot[2 * pr], sn = rot[2 * pr + 1];
    const float2 rr =
        make_float2((float)((double)r.x * cs - (double)r.y * sn), (float)((double)r.x * sn + (double)r.y * cs));
    if (q_rope) *reinterpret_cast<float2*>(q_rope + th * d_r + 2 * pr) = rr;
    if (qp_hi) {
      const __nv_bfloat162 hi = __floats2bfloat162_rn(rr.x, rr.y);
      const long long o = th * row + rope_col + 2 * pr;
      *reinterpret_cast<__nv_bfloat162*>(qp_hi + o) = hi;
      if (qp_lo)
        *reinterpret_cast<__nv_bfloat162*>(qp_lo + o) =
            __floats2bfloat162_rn(rr.x - __bfloat162float(hi.x), rr.y - __bfloat162float(hi.y));
    }
  }
}

static inline int grid_for(long long n, int threads = 256, int cap = 8192) {
  long long b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  return (int)(b > cap ? cap : b);
}

}  // namespace mla

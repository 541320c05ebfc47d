// Latent-space decode on CUDA cores: one warp per (segment, head).
// Used for the fp32 storage path (small shapes, exact fp32 arithmetic) and
// for the FP8 cache (E4M3 codes times the row's fp32 scale, `row_scale`
// [num_blocks, block]; null for the other storage types).
//
// For the rows u of its segment (all visible to the segment's query row):
//   s_u = (q_lat . c_u + q_R . kR_u) * scale * log2(e)
// with an online (running-max) softmax, O = sum_u 2^(s_u - m) c_u / l.
#pragma once

#include "decode_plan.cuh"

namespace mla {

constexpr int kSimtDecodeMaxRow = 1024;  // d_c + d_r handled by one warp (32 lanes x 32 values)

template <typename T, int DPL>
__global__ void __launch_bounds__(128) decode_simt_kernel(
    const float* __restrict__ q_lat, const float* __restrict__ q_rope, const T* __restrict__ pool,
    const float* __restrict__ row_scale, const int32_t* __restrict__ block_table, int max_blocks, int num_blocks,
    const int32_t* __restrict__ seq_lens, int n_q, int H, int d_c, int d_r, int bs,
    float scale_log2, void* ws, DecodeLayout L) {
  const DecodeHeader* hd = ws_at<DecodeHeader>(ws, 0);
  const int sidx = blockIdx.x;
  if (sidx >= hd->num_segments) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 4 + warp;
  if (h >= H) return;
  const int4 sg = ws_at<int4>(ws, L.off_seg)[sidx];
  const int v = sg.x, b = v / n_q, j = v % n_q;
  const int len_v = seq_lens[b] - n_q + j + 1;  // rows this query sees
  const int row = d_c + d_r;

  float q[DPL], o[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    const int d = lane + 32 * i;
    float val = 0.f;
    if (d < d_c) val = q_lat[((long long)v * H + h) * d_c + d];
    else if (d < row) val = q_rope[((long long)v * H + h) * d_r + (d - d_c)];
    q[i] = val;
    o[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int blk = sg.y; blk < sg.z; ++blk) {
    const int nrows = min(bs, len_v - blk * bs);
    if (nrows <= 0) break;
    const int phys = block_table[(long long)b * max_blocks + blk];
    if (phys < 0 || phys >= num_blocks) {
      if (lane == 0) report(MLA_ERR_BOUNDS, 5, b, phys);
      continue;
    }
    const T* base = pool + (long long)phys * bs * row;
    for (int r = 0; r < nrows; ++r) {
      const T* kv = base + (long long)r * row;
      const float sc = row_scale != nullptr ? row_scale[(long long)phys * bs + r] : 1.f;
      float part = 0.f;
      float c[DPL];
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const int d = lane + 32 * i;
        c[i] = d < row ? Store<T>::ld(kv + d) * sc : 0.f;
        part = fmaf(q[i], c[i], part);
      }
      const float s = warp_sum(part) * scale_log2;
      const float m_new = fmaxf(m, s);
      const float corr = exp2f(m - m_new);
      const float pw = exp2f(s - m_new);
      l = l * corr + pw;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const int d = lane + 32 * i;
        o[i] = o[i] * corr + (d < d_c ? pw * c[i] : 0.f);
      }
      m = m_new;
    }
  }
  const long long r_out = (long long)sidx * H + h;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  float* out = ws_at<float>(ws, L.off_o) + r_out * d_c;  // [segment][h][d]
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    const int d = lane + 32 * i;
    if (d < d_c) out[d] = o[i] * inv;
  }
  if (lane == 0) ws_at<float>(ws, L.off_lse)[r_out] = l > 0.f ? m + log2f(l) : -INFINITY;
}

}  // namespace mla

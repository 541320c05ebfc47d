// Split-KV work plan shared by every decode kernel, and the split combine.
//
// The unit of work is a query row v = b * n_q + j (query j of sequence b).
// Row v sees the cache rows 0 .. len_v - 1 of sequence b, with
// len_v = seq_lens[b] - n_q + j + 1 (causal, its own row included), i.e.
// ceil(len_v / block) pages (none for an empty sequence, seq_lens[b] = 0).  The pages of all query rows, laid end to end,
// are cut into `workers` contiguous ranges of about equal cost (pages plus a
// fixed charge per row for the segment's setup); where a range crosses a row
// boundary it is cut again, so every piece - a "segment" - covers pages
// [blk_begin, blk_end) of one query row.  There are
// at most workers + rows - 1 segments, and they are ordered by query row.
// Each segment's decode writes, per head, its output normalised over its own
// rows ([segment][h][d], bf16 from the tensor-core decode, fp32 from the
// CUDA-core one) plus the log2-sum-exp of its scaled scores; the combine
// merges the segments of a row.  The plan is computed on the device from
// seq_lens, so a decode step never waits on the host.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kPlanMagic = 0x4D4C4131;  // "MLA1"

struct DecodeLayout {
  int batch, n_q, H, d_c, workers, max_segments;
  int part_elem;               // bytes per partial-output value: 2 (bf16) or 4 (fp32)
  long long off_prefix;        // int32 [rows + 1]    pages before query row v
  long long off_worker_first;  // int32 [workers + 1] first segment of worker w
  long long off_seq_first;     // int32 [rows]        first segment of query row v
  long long off_seq_nseg;      // int32 [rows]        number of segments of query row v
  long long off_seg;           // int4  [max_segments] (v, blk_begin, blk_end, worker)
  long long off_lse;           // f32   [max_segments, H]        log2-sum-exp
  long long off_o;             // bf16 / f32 [max_segments, H, d_c]  normalised partial output
  long long off_qpack;         // bf16  [rows, H, d_c + d_r]     the query in bf16 (tensor-core path)
  long long total;
};

// Written by the plan kernel at offset 0 of the workspace; read by the combine.
struct DecodeHeader {
  int magic, batch, n_q, H, d_c, workers, max_segments, num_segments;
  DecodeLayout layout;
};

static inline DecodeLayout decode_layout(int batch, int n_q, int H, int d_c, int workers,
                                         size_t qpack_row_bytes, int part_elem) {
  DecodeLayout L{};
  const size_t rows = (size_t)batch * n_q;
  L.part_elem = part_elem;
  L.batch = batch;
  L.n_q = n_q;
  L.H = H;
  L.d_c = d_c;
  L.workers = workers;
  L.max_segments = workers + (int)rows;
  size_t o = align_up(sizeof(DecodeHeader), 256);
  L.off_prefix = o;        o = align_up(o + sizeof(int) * (rows + 1), 256);
  L.off_worker_first = o;  o = align_up(o + sizeof(int) * (size_t)(workers + 1), 256);
  L.off_seq_first = o;     o = align_up(o + sizeof(int) * rows, 256);
  L.off_seq_nseg = o;      o = align_up(o + sizeof(int) * rows, 256);
  L.off_seg = o;           o = align_up(o + sizeof(int4) * (size_t)L.max_segments, 256);
  L.off_lse = o;           o = align_up(o + sizeof(float) * (size_t)L.max_segments * H, 256);
  L.off_o = o;             o = align_up(o + (size_t)part_elem * L.max_segments * H * d_c, 256);
  L.off_qpack = o;         o = align_up(o + qpack_row_bytes * rows, 256);
  L.total = o;
  return L;
}

template <typename T> __device__ __forceinline__ T* ws_at(void* ws, long long off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}
template <typename T> __device__ __forceinline__ const T* ws_at(const void* ws, long long off) {
  return reinterpret_cast<const T*>(static_cast<const char*>(ws) + off);
}

// Exclusive prefix sum of value_of(0..n-1) into dst[0..n] (dst[n] = total), one CTA.
template <typename F>
__device__ int block_scan_exclusive(F value_of, int* dst, int n) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int v = i < n ? value_of(i) : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int w = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < nw) warp_tot[lane] = w;
    }
    __syncthreads();
    const int excl = carry + (wid > 0 ? warp_tot[wid - 1] : 0) + x - v;
    if (i < n) dst[i] = excl;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = excl + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) dst[n] = carry;
  __syncthreads();
  return carry;
}

// Largest v in [0, rows) with P[v] <= g (requires 0 <= g < P[rows]).
__device__ __forceinline__ int seq_of_page(const int* P, int rows, long long g) {
  int lo = 0, hi = rows - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)P[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Page prefix of the query rows lives in shared memory (the searches below
// are chains of dependent loads); one CTA computes the whole plan.
constexpr int kPlanMaxRows = 49152;
constexpr int kSegCost = 10;  // per-segment overhead of the decode, in quarter pages

// The plan, computed by one CTA of 1024 threads with (rows + 1) ints of
// dynamic shared memory.
__device__ __forceinline__ void plan_body(const int32_t* __restrict__ seq_lens, int bs, int max_blocks, void* ws,
                                          const DecodeLayout& L) {
  extern __shared__ int P[];  // [rows + 1]
  int* wfirst = ws_at<int>(ws, L.off_worker_first);
  int* sfirst = ws_at<int>(ws, L.off_seq_first);
  int* snseg = ws_at<int>(ws, L.off_seq_nseg);
  int4* seg = ws_at<int4>(ws, L.off_seg);
  const int n_q = L.n_q, W = L.workers;
  const int rows = L.batch * n_q;  // query rows

  auto pages_of = [&](int v) -> int {
    const int b = v / n_q, j = v % n_q;
    const int len = seq_lens[b];
    // 0: an empty sequence (e.g. a shard of another GPU's pages holding none
    // of this one's), whose query rows see no row
    if (len < 0 || (len > 0 && len < n_q) || len > max_blocks * bs) {
      if (j == 0) report(MLA_ERR_BOUNDS, 4, b, len);
      return 0;
    }
    return (len - n_q + j + 1 + bs - 1) / bs;
  };
  const int NB = block_scan_exclusive(pages_of, P, rows);

  // Workers get equal shares of cost, not of pages: a segment costs a
  // query reload and an epilogue on top of its pages (about kSegCost / 4
  // pages), so every row is charged that much once.  Cost positions are in
  // quarter pages; row v occupies [Pc(v), Pc(v + 1)) with Pc(v) = 4 P[v] +
  // kSegCost v, its first kSegCost quarters being the overhead.
  const long long NC = 4LL * NB + (long long)kSegCost * rows;
  auto page_at = [&](long long x) -> long long {
    int lo = 0, hi = rows - 1;  // largest v with Pc(v) <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (4LL * P[mid] + (long long)kSegCost * mid <= x) lo = mid; else hi = mid - 1;
    }
    const long long o = x - (4LL * P[lo] + (long long)kSegCost * lo) - kSegCost;
    const long long pages = P[lo + 1] - P[lo];
    return P[lo] + (o <= 0 ? 0 : (o / 4 < pages ? o / 4 : pages));
  };
  auto range_of = [&](int w, long long& s, long long& e) {
    s = page_at((long long)w * NC / W);
    e = page_at((long long)(w + 1) * NC / W);
  };
  auto segs_of = [&](int w) -> int {
    long long s, e;
    range_of(w, s, e);
    if (s >= e) return 0;
    return seq_of_page(P, rows, e - 1) - seq_of_page(P, rows, s) + 1;
  };
  const int nsegs = block_scan_exclusive(segs_of, wfirst, W);

  for (int w = threadIdx.x; w < W; w += blockDim.x) {
    long long s, e;
    range_of(w, s, e);
    if (s >= e) continue;
    const int b0 = seq_of_page(P, rows, s), b1 = seq_of_page(P, rows, e - 1);
    int k = wfirst[w];
    for (int b = b0; b <= b1; ++b, ++k) {
      const long long lo = s > P[b] ? s : P[b];
      const long long hi = e < P[b + 1] ? e : P[b + 1];
      seg[k] = make_int4(b, (int)(lo - P[b]), (int)(hi - P[b]), w);
    }
  }
  for (int b = threadIdx.x; b < rows; b += blockDim.x) {
    sfirst[b] = 0;
    snseg[b] = 0;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < nsegs; k += blockDim.x) {
    const int b = seg[k].x;
    if (k == 0 || seg[k - 1].x != b) sfirst[b] = k;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < nsegs; k += blockDim.x) {
    const int b = seg[k].x;
    if (k == nsegs - 1 || seg[k + 1].x != b) snseg[b] = k - sfirst[b] + 1;
  }
  if (threadIdx.x == 0) {
    DecodeHeader* h = ws_at<DecodeHeader>(ws, 0);
    h->magic = kPlanMagic;
    h->batch = L.batch;
    h->n_q = n_q;
    h->H = L.H;
    h->d_c = L.d_c;
    h->workers = W;
    h->max_segments = L.max_segments;
    h->num_segments = nsegs;
    h->layout = L;
  }
}

__global__ void __launch_bounds__(1024) decode_plan_kernel(const int32_t* __restrict__ seq_lens, int bs,
                                                           int max_blocks, void* ws, DecodeLayout L) {
  pdl_wait();
  pdl_trigger();
  plan_body(seq_lens, bs, max_blocks, ws, L);
}

// Weight of segment `first + s` in the merge of query row v for head h:
// 2^(lse_s - M) / sum_s' 2^(lse_s' - M) with M the largest lse of the row.
struct RowMerge {
  float M, Z, invZ;
  // the n log2-sum-exps at lse[(first + s) * stride + h], s < n
  __device__ RowMerge(const float* lse, long long first, int n, long long stride, int h)
      : M(-INFINITY), Z(0.f), invZ(0.f) {
    for (int s = 0; s < n; ++s) M = fmaxf(M, lse[(first + s) * stride + h]);
    if (M == -INFINITY) return;
    for (int s = 0; s < n; ++s) Z += exp2f(lse[(first + s) * stride + h] - M);
    invZ = 1.f / Z;
  }
  __device__ float weight(float lse_s) const { return invZ > 0.f ? exp2f(lse_s - M) * invZ : 0.f; }
  // log2-sum-exp of the merged pieces (-inf when none holds a key)
  __device__ float lse() const { return M == -INFINITY ? -INFINITY : M + log2f(Z); }
};

__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(p)), b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void load8(const bf16* p, float (&x)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    x[2 * k] = __uint_as_float(w[k] << 16);
    x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

// o_lat[v, h, d] = sum_s w_s,h O_s[h, d] over the segments s of query row v.
// Grid (query rows, head blocks); a thread owns 8 consecutive d of one head
// (d_c / 8 threads per head), so every load and store is a 16- or 32-byte
// vector and a warp covers whole rows.
// With `valid` false (a workspace no decode wrote) the row is written as zeros.
template <typename P>
__device__ void combine_rows(const void* ws, const DecodeLayout& L, bool valid, int v, int H, int d_c,
                             float* __restrict__ o_lat, float* __restrict__ lse_out) {
  const int per_head = d_c / 8;
  const int hb = blockDim.x / per_head;
  const int h = blockIdx.y * hb + threadIdx.x / per_head, d0 = 8 * (threadIdx.x % per_head);
  if (h >= H || threadIdx.x >= hb * per_head) return;
  const int first = valid ? ws_at<int>(ws, L.off_seq_first)[v] : 0;
  const int n = valid ? ws_at<int>(ws, L.off_seq_nseg)[v] : 0;
  const float* lse = ws_at<float>(ws, L.off_lse);
  const P* part = ws_at<P>(ws, L.off_o);
  const RowMerge rm(lse, first, n, H, h);
  if (lse_out != nullptr && d0 == 0) lse_out[(long long)v * H + h] = rm.lse();
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < n; ++s) {
    const float w = rm.weight(lse[(long long)(first + s) * H + h]);
    if (w == 0.f) continue;  // no rows in this piece: its output was never written
    float x[8];
    load8(part + ((long long)(first + s) * H + h) * d_c + d0, x);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = fmaf(w, x[k], acc[k]);
  }
  float* out = o_lat + ((long long)v * H + h) * d_c + d0;
  *reinterpret_cast<float4*>(out) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  *reinterpret_cast<float4*>(out + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

__global__ void __launch_bounds__(256) combine_kernel(const void* ws, long long ws_bytes, int batch, int n_q, int H,
                                                      int d_c, float* __restrict__ o_lat, float* __restrict__ lse_out) {
  pdl_wait();
  pdl_trigger();
  const DecodeHeader* hd = ws_at<DecodeHeader>(ws, 0);
  const bool bad = hd->magic != kPlanMagic || hd->batch != batch || hd->n_q != n_q || hd->H != H ||
                   hd->d_c != d_c || hd->layout.total > ws_bytes;
  const int v = blockIdx.x;
  if (bad && v == 0 && blockIdx.y == 0 && threadIdx.x == 0) report(MLA_ERR_WORKSPACE, 0, batch, n_q);
  const DecodeLayout L = hd->layout;
  if (!bad && L.part_elem == 2) combine_rows<bf16>(ws, L, true, v, H, d_c, o_lat, lse_out);
  else combine_rows<float>(ws, L, !bad, v, H, d_c, o_lat, lse_out);
}

// The same merge one level up: o_parts[r] and lse_parts[r] are the
// (o_lat, log2-sum-exp) of query rows over shard r of every sequence's keys
// (e.g. the pages held by GPU r), all shards of a row together are its whole
// key set.  o_lat[v, h] = sum_r 2^(lse_r - M) o_r / sum_r 2^(lse_r - M), and
// lse_out (optional) the merged log2-sum-exp.  Grid and threads as combine.
__global__ void __launch_bounds__(256) merge_shards_kernel(const float* __restrict__ o_parts,
                                                           const float* __restrict__ lse_parts, int n_shards,
                                                           int rows, int H, int d_c, float* __restrict__ o_lat,
                                                           float* __restrict__ lse_out) {
  pdl_wait();
  pdl_trigger();
  const int per_head = d_c / 8;
  const int hb = blockDim.x / per_head;
  const int v = blockIdx.x;
  const int h = blockIdx.y * hb + threadIdx.x / per_head, d0 = 8 * (threadIdx.x % per_head);
  if (h >= H || threadIdx.x >= hb * per_head) return;
  const long long stride = (long long)rows * H;  // between shards, in lse entries
  const RowMerge rm(lse_parts, 0, n_shards, stride, v * H + h);
  if (lse_out != nullptr && d0 == 0) lse_out[(long long)v * H + h] = rm.lse();
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int r = 0; r < n_shards; ++r) {
    const float w = rm.weight(lse_parts[r * stride + (long long)v * H + h]);
    if (w == 0.f) continue;  // a shard without keys for this row
    float x[8];
    load8(o_parts + (r * stride + (long long)v * H + h) * d_c + d0, x);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = fmaf(w, x[k], acc[k]);
  }
  float* out = o_lat + ((long long)v * H + h) * d_c + d0;
  *reinterpret_cast<float4*>(out) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  *reinterpret_cast<float4*>(out + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

}  // namespace mla

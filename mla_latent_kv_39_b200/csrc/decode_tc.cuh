// Latent-space split-KV decode on the sm_100 tensor cores (tcgen05 + TMEM + TMA).
//
// Shape: 128 heads, latent d_c = 512, rotary d_r = 64, 64-token cache pages,
// bf16 cache.  All heads share one latent row per token, so for one query
// row the scores S = [q_lat | q_R] [c | k_R]^T (M = 128 heads, K = 576) and
// the output O = P c (K = tokens, N = 512) are real GEMMs
// ("MLA · latent KV, decoupled RoPE và matrix absorption", section 2 "Luồng":
// scores and output from the merged matrices or an equivalent kernel).
//
// One worker is a cluster of two CTAs on two SMs.  TMEM (512 columns x 128
// lanes) cannot hold the 128 x 512 fp32 output, the scores and the query of
// one head block at once, so the pair splits the latent width:
//   CTA 0 owns dims [0, 256)   : scores over c[0:256],         O[:, 0:256]
//   CTA 1 owns dims [256, 576) : scores over c[256:512] + k_R, O[:, 256:512]
// Each CTA loads only its columns of every page (TMA, 128-byte swizzle, no
// byte loaded twice), keeps its query half in TMEM as the MMA A operand, and
// after every page sends its fp32 partial scores to the peer through
// distributed shared memory.  Both CTAs then hold identical full scores and
// run the identical online softmax; P (bf16) goes to TMEM as the A operand of
// the P V MMA, whose B operand is the same staged page read MN-major.
//
// TMEM columns: [0, 256) O, [256, 320) S (64 tokens), [320, 352) P (bf16
// pairs), [352, 512) query half (bf16 pairs: 128 or 160 columns).
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM
// and issues MMAs (one thread), warps 2-5 run the softmax, one thread per
// head (TMEM lane).  The running max is kept stale until it grows by more
// than 2^8, so the output in TMEM is rescaled only on such jumps.
//
// Split-query variant (kSplit): the fp32 query is held as bf16 hi (TMEM, A
// operand) + bf16 lo (shared memory, A operand of a second MMA into the same
// scores), about 16 significant bits instead of 8.  It needs the shared
// memory of one page stage, so it runs with two stages instead of three.
#pragma once

#include "decode_plan.cuh"
#include "decode_tc3.cuh"
#include "sm100.cuh"

namespace mla {
namespace tcdec {

using namespace sm100;

constexpr int kH = 128, kDc = 512, kDr = 64, kRow = 576, kBS = 64;
constexpr int kSlabBytes = 64 * 128;                 // 64 rows x 64 bf16 (128 B), swizzled
constexpr int kMaxSlabs = 5;
constexpr int kStageBytes = kMaxSlabs * kSlabBytes;  // 40 KiB
constexpr int kQloSlabBytes = 128 * 128;             // 128 rows x 64 bf16, swizzled
constexpr int kTmemO = 0, kTmemS = 256, kTmemP = 320, kTmemQ = 352, kTmemCols = 512;
constexpr int kThreads = 192;
constexpr float kRescaleLog2 = 8.f;

template <bool kSplit> struct Cfg {
  static constexpr int kStages = kSplit ? 2 : 3;
  static constexpr int kQloBytes = kSplit ? kMaxSlabs * kQloSlabBytes : 16;
};

// Exchanged score rows are 64 floats; the 16-byte chunk c of row r is stored
// at chunk position c ^ (r & 15), so a quarter warp touches 8 distinct bank groups.
template <bool kSplit> struct Smem {
  uint8_t kv[Cfg<kSplit>::kStages][kStageBytes];  // first member: 1024-byte aligned
  uint8_t qlo[Cfg<kSplit>::kQloBytes];            // split variant: query lo part (A operand)
  float xbuf[2][kH][64];
  uint64_t full[Cfg<kSplit>::kStages], empty[Cfg<kSplit>::kStages];
  uint64_t s_full, s_free, p_ready, pv_done, q_ready, mma_done;
  uint64_t xfull[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <bool kSplit> constexpr size_t smem_bytes() { return sizeof(Smem<kSplit>) + 1024; }

struct Params {
  const float* q_lat;      // [rows, 128, 512]
  const float* q_rope;     // [rows, 128, 64]
  const int32_t* block_table;
  const int32_t* seq_lens;
  int max_blocks, num_blocks, n_q;
  float scale_log2;
  void* ws;
  DecodeLayout L;
};

template <class S> __device__ __forceinline__ void set_abort(S& sm) { *(volatile int*)&sm.abort_flag = 1; }
template <class S> __device__ __forceinline__ bool aborted(S& sm) { return *(volatile int*)&sm.abort_flag != 0; }

// ---------------------------------------------------------------- TMA producer
template <bool kSplit>
__device__ void producer(Smem<kSplit>& sm, const CUtensorMap* tmap, const Params& p, int seg_begin, int seg_end,
                         uint32_t crank, int nslab) {
  constexpr int kStages = Cfg<kSplit>::kStages;
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  int k = 0;
  for (int si = seg_begin; si < seg_end && !aborted(sm); ++si) {
    const int4 sg = segs[si];
    const int b = sg.x / p.n_q;
    for (int blk = sg.y; blk < sg.z; ++blk, ++k) {
      const int stage = k % kStages;
      if (k >= kStages && !mbar_wait(&sm.empty[stage], ((k / kStages) - 1) & 1, 10)) {
        set_abort(sm);
        goto drain;
      }
      int phys = p.block_table[(long long)b * p.max_blocks + blk];
      if (phys < 0 || phys >= p.num_blocks) {
        report(MLA_ERR_BOUNDS, 5, b, phys);
        phys = 0;  // keep the pipeline moving; the error word marks the result invalid
      }
      mbar_arrive_expect_tx(&sm.full[stage], (uint32_t)(nslab * kSlabBytes));
      for (int s = 0; s < nslab; ++s)
        tma_load_2d(sm.kv[stage] + s * kSlabBytes, tmap, (int)crank * 256 + s * 64, phys * kBS,
                    &sm.full[stage]);
    }
  }
drain:
  // Never leave a copy in flight into shared memory that is about to be released.
  for (int kk = k - kStages < 0 ? 0 : k - kStages; kk < k; ++kk)
    mbar_wait(&sm.full[kk % kStages], (kk / kStages) & 1, 11);
}

// ---------------------------------------------------------------- MMA issuer
template <bool kSplit>
__device__ __forceinline__ bool issue_scores(Smem<kSplit>& sm, uint32_t tmem, int kk, int ksteps) {
  constexpr int kStages = Cfg<kSplit>::kStages;
  const int stage = kk % kStages;
  if (!mbar_wait(&sm.full[stage], (kk / kStages) & 1, 20)) return false;
  if (kk > 0 && !mbar_wait(&sm.s_free, (kk - 1) & 1, 21)) return false;
  tc_fence_after();
  constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
  const uint32_t base = smem_u32(sm.kv[stage]);
  const uint32_t qlo = smem_u32(sm.qlo);
  for (int j = 0; j < ksteps; ++j) {
    // K-major page slab: rows (tokens) 128 B apart, 8-row groups 1024 B apart;
    // the 16-value K step j sits at byte (j % 4) * 32 of slab j / 4.
    const uint64_t bdesc = smem_desc(base + (j >> 2) * kSlabBytes + (j & 3) * 32, 16, 1024, kSwizzle128B);
    mma_ts(tmem + kTmemS, tmem + kTmemQ + j * 8, bdesc, idesc, j > 0 ? 1u : 0u);
    if constexpr (kSplit) {
      // query lo part: K-major, 128 rows 128 B apart, 8-row groups 1024 B apart
      const uint64_t adesc = smem_desc(qlo + (j >> 2) * kQloSlabBytes + (j & 3) * 32, 16, 1024, kSwizzle128B);
      mma_ss(tmem + kTmemS, adesc, bdesc, idesc, 1u);
    }
  }
  mma_commit(&sm.s_full);
  return true;
}

template <bool kSplit>
__device__ void mma_issuer(Smem<kSplit>& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end,
                           int ksteps) {
  constexpr int kStages = Cfg<kSplit>::kStages;
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
  int k = 0, seg_i = 0;
  for (int si = seg_begin; si < seg_end; ++si, ++seg_i) {
    const int4 sg = segs[si];
    const int T = sg.z - sg.y;
    if (!mbar_wait(&sm.q_ready, seg_i & 1, 22) || !issue_scores(sm, tmem, k, ksteps)) goto fail;
    for (int i = 0; i < T; ++i) {
      const int kk = k + i;
      if (i + 1 < T && !issue_scores(sm, tmem, kk + 1, ksteps)) goto fail;
      if (!mbar_wait(&sm.p_ready, kk & 1, 23)) goto fail;
      tc_fence_after();
      const uint32_t base = smem_u32(sm.kv[kk % kStages]);
      for (int j = 0; j < 4; ++j) {
        // MN-major page slabs: 64-dim chunks 8 KiB apart (LBO), 8-token groups
        // 1 KiB apart (SBO); the 16-token K step j starts 2 KiB further.
        const uint64_t bdesc = smem_desc(base + j * 2048, kSlabBytes, 1024, kSwizzle128B);
        mma_ts(tmem + kTmemO, tmem + kTmemP + j * 8, bdesc, idesc_pv, (i > 0 || j > 0) ? 1u : 0u);
      }
      mma_commit(&sm.pv_done);
      mma_commit(&sm.empty[kk % kStages]);
    }
    k += T;
  }
  mma_commit(&sm.mma_done);
  mbar_wait(&sm.mma_done, 0, 24);
  return;
fail:
  set_abort(sm);
  mma_commit(&sm.mma_done);
  mbar_wait(&sm.mma_done, 0, 25);
}

// ---------------------------------------------------------------- softmax
// bf16 pair (hi) of two floats and the bf16 pair of what hi leaves out (lo).
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(a, b);
  const float ha = __uint_as_float(hi << 16), hb = __uint_as_float(hi & 0xFFFF0000u);
  lo = pack_bf16x2(a - ha, b - hb);
}

// Row r of this CTA's query half: bf16 hi into TMEM (A operand); in the split
// variant also the bf16 lo part into shared memory, K-major with 128-byte swizzle.
template <bool kSplit>
__device__ __forceinline__ void load_query_half(const Params& p, int v, int r, uint32_t crank, uint32_t taddr,
                                                uint8_t* qlo) {
  const float* ql = p.q_lat + ((long long)v * kH + r) * kDc + crank * 256;
  const float* qr = p.q_rope + ((long long)v * kH + r) * kDr;
  const int chunks = crank == 0 ? 8 : 10;  // 32 values per chunk
  for (int ch = 0; ch < chunks; ++ch) {
    const float4* src = reinterpret_cast<const float4*>(ch < 8 ? ql + ch * 32 : qr + (ch - 8) * 32);
    uint32_t w[16], lo[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 f = __ldg(src + i);
      split_pair(f.x, f.y, w[2 * i], lo[2 * i]);
      split_pair(f.z, f.w, w[2 * i + 1], lo[2 * i + 1]);
    }
    tmem_st16(taddr + ch * 16, w);
    if constexpr (kSplit) {
      // values [32 ch, 32 ch + 32) = slab ch / 2, 16-byte chunks 4 (ch % 2) .. + 3
      uint8_t* row = qlo + (ch >> 1) * kQloSlabBytes + r * 128;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int chunk = (ch & 1) * 4 + q4;
        *reinterpret_cast<uint4*>(row + ((chunk ^ (r & 7)) * 16)) =
            make_uint4(lo[4 * q4], lo[4 * q4 + 1], lo[4 * q4 + 2], lo[4 * q4 + 3]);
      }
    }
  }
}

// All 32 lanes agree on a wait's outcome (the tcgen05 loads and stores that
// follow must be executed by the whole warp).
#define MLA_WARP_WAIT(expr) (__all_sync(0xffffffffu, (expr)))

template <bool kSplit>
__device__ void softmax_role(Smem<kSplit>& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end,
                             uint32_t crank, int warp, int lane) {
  constexpr int kStages = Cfg<kSplit>::kStages;
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const int qw = warp & 3;
  const int r = qw * 32 + lane;                          // head row == TMEM lane
  const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);  // this warp's lane quarter
  const uint32_t peer = crank ^ 1u;
  const uint32_t x_row_local = smem_u32(&sm.xbuf[0][r][0]);
  const uint32_t x_row_peer = mapa(x_row_local, peer);
  constexpr uint32_t kXStageBytes = kH * 64 * 4;
  const int xsw = r & 15;
  const uint32_t xfull_peer0 = mapa(smem_u32(&sm.xfull[0]), peer);
  const uint32_t xfull_peer1 = mapa(smem_u32(&sm.xfull[1]), peer);
  float* part_o = ws_at<float>(p.ws, p.L.off_o);
  float* part_lse = ws_at<float>(p.ws, p.L.off_lse);
  const int tid = (warp - 2) * 32 + lane;               // 0..127

  int k = 0;
  for (int si = seg_begin; si < seg_end; ++si) {
    const int4 sg = segs[si];
    const int v = sg.x, b = v / p.n_q, jq = v % p.n_q;
    const int len_v = p.seq_lens[b] - p.n_q + jq + 1;
    const int T = sg.z - sg.y;

    load_query_half<kSplit>(p, v, r, crank, tl + kTmemQ, sm.qlo);
    tmem_wait_st();
    if constexpr (kSplit) fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(&sm.q_ready);

    float m_used = -INFINITY, l = 0.f;
    for (int i = 0; i < T; ++i) {
      const int kk = k + i, blk = sg.y + i;
      if (!MLA_WARP_WAIT(mbar_wait(&sm.s_full, kk & 1, 30))) goto fail;
      tc_fence_after();
      float s[64];
      {
        uint32_t a[32];
        tmem_ld32(tl + kTmemS, a);
        uint32_t c[32];
        tmem_ld32(tl + kTmemS + 32, c);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          s[t] = __uint_as_float(a[t]);
          s[32 + t] = __uint_as_float(c[t]);
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.s_free);

      // exchange partial scores with the peer CTA
      const int xs = kk & 1;
      const uint32_t dst = x_row_peer + xs * kXStageBytes;
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4)
        st_cluster_v4(dst + ((c4 ^ xsw) * 16), s[4 * c4], s[4 * c4 + 1], s[4 * c4 + 2], s[4 * c4 + 3]);
      mbar_arrive_cluster(xs ? xfull_peer1 : xfull_peer0);
      if (!MLA_WARP_WAIT(mbar_wait<true>(&sm.xfull[xs], (kk >> 1) & 1, 31))) goto fail;
      {
        const float4* mine = reinterpret_cast<const float4*>(&sm.xbuf[xs][r][0]);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 t4 = mine[c4 ^ xsw];
          s[4 * c4] += t4.x;
          s[4 * c4 + 1] += t4.y;
          s[4 * c4 + 2] += t4.z;
          s[4 * c4 + 3] += t4.w;
        }
      }

      const int valid = min(kBS, len_v - blk * kBS);
      float mx = -INFINITY;
#pragma unroll
      for (int t = 0; t < 64; ++t) {
        s[t] = t < valid ? s[t] * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[t]);
      }
      bool rescale = false;
      float alpha = 1.f;
      if (i == 0) {
        m_used = mx;
      } else if (mx > m_used + kRescaleLog2) {
        alpha = exp2f(m_used - mx);
        m_used = mx;
        rescale = true;
      }
      uint32_t pk[32];
      float psum = 0.f;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float p0 = exp2f(s[2 * t] - m_used), p1 = exp2f(s[2 * t + 1] - m_used);
        psum += p0 + p1;
        pk[t] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + psum;

      if (i > 0) {
        if (!MLA_WARP_WAIT(mbar_wait(&sm.pv_done, (kk - 1) & 1, 32))) goto fail;
        tc_fence_after();
        // tcgen05.ld / st are warp-collective: the whole warp rescales when any
        // of its rows needs it (rows that do not use alpha = 1).
        if (__any_sync(0xffffffffu, rescale)) {
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t o[32];
            tmem_ld32(tl + kTmemO + ch * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
            tmem_st32(tl + kTmemO + ch * 32, o);
          }
        }
      }
      if (valid < kBS) {
        // Rows past the sequence end hold whatever the pool holds (maybe NaN);
        // P is 0 there, but 0 x NaN is NaN, so clear them in the V slabs.
        uint8_t* stage = sm.kv[kk % kStages];
        const int nrow = kBS - valid, per_slab = nrow * 8;
        for (int c = tid; c < 4 * per_slab; c += 128) {
          const int slab = c / per_slab, rem = c % per_slab;
          *reinterpret_cast<uint4*>(stage + slab * kSlabBytes + (valid + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tmem_st32(tl + kTmemP, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_ready);
    }
    // epilogue of the segment: O / l and the log2-sum-exp
    {
      const int kl = k + T - 1;
      if (!MLA_WARP_WAIT(mbar_wait(&sm.pv_done, kl & 1, 33))) goto fail;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      // head-minor partial output: the warp's 32 heads of one column are one 128-byte line
      float* out = part_o + ((long long)si * kDc + crank * 256) * kH + r;
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t o[32];
        tmem_ld32(tl + kTmemO + ch * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) out[(long long)(ch * 32 + t) * kH] = __uint_as_float(o[t]) * inv;
      }
      if (crank == 0) part_lse[(long long)si * kH + r] = l > 0.f ? m_used + log2f(l) : -INFINITY;
    }
    k += T;
  }
  return;
fail:
  set_abort(sm);
}

// ---------------------------------------------------------------- kernel
template <bool kSplit>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap, const Params p) {
  constexpr int kStages = Cfg<kSplit>::kStages;
  extern __shared__ uint8_t smem_raw[];
  Smem<kSplit>& sm =
      *reinterpret_cast<Smem<kSplit>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const int worker = blockIdx.x >> 1;
  const int nslab = crank == 0 ? 4 : 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 128);
    mbar_init(&sm.p_ready, 128);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.q_ready, 128);
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.xfull[0], 128);
    mbar_init(&sm.xfull[1], 128);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // the peer's barriers exist before anyone arrives on them
  const uint32_t tmem = sm.tmem_base;

  int seg_begin = 0, seg_end = 0;
  if (worker < p.L.workers) {
    const int* wfirst = ws_at<int>(p.ws, p.L.off_worker_first);
    seg_begin = wfirst[worker];
    seg_end = wfirst[worker + 1];
  }

  if (warp == 0) {
    if (lane == 0) producer<kSplit>(sm, &tmap, p, seg_begin, seg_end, crank, nslab);
  } else if (warp == 1) {
    if (lane == 0) mma_issuer<kSplit>(sm, tmem, p, seg_begin, seg_end, nslab * 4);
  } else {
    softmax_role<kSplit>(sm, tmem, p, seg_begin, seg_end, crank, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync();  // the peer no longer writes into this CTA's shared memory
}

}  // namespace tcdec
}  // namespace mla

// ================================================================ host side
namespace mla {
namespace tcdec {

inline bool supports(const mla_config* c) {
  return c->dtype == MLA_BF16 && c->n_heads == kH && c->d_c == kDc && c->d_r == kDr && c->block_size == kBS;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load(std::memory_order_acquire);
  if (f == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && p != nullptr) {
      f = reinterpret_cast<EncodeTiledFn>(p);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

// The pool as a 2-D bf16 tensor [num_blocks * 64 rows, 576 values], row
// stride 1152 B, read in 64 x 64 boxes with the 128-byte swizzle.
inline mla_status pool_tensor_map(const mla_cache* k, CUtensorMap* map) {
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return MLA_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)kRow, (cuuint64_t)k->num_blocks * kBS};
  const cuuint64_t strides[1] = {(cuuint64_t)kRow * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k->pool, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// The packed query (bf16 [rows * 128, 576], row stride 1152 B) read in boxes
// of 128 heads x 64 values with the 128-byte swizzle: one box is one
// shared-memory query slab of the decode.
inline mla_status qpack_tensor_map(void* qpack, long long rows, CUtensorMap* map) {
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return MLA_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)kRow, (cuuint64_t)rows * kH};
  const cuuint64_t strides[1] = {(cuuint64_t)kRow * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kH};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qpack, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

template <bool kSplit>
inline mla_status set_smem_attr() {
  static std::atomic<uint64_t> done_mask{0};  // one bit per device (devices 0..63)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done_mask.load(std::memory_order_acquire) & bit)) return MLA_OK;
  if (cudaFuncSetAttribute(decode_tc_kernel<kSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_bytes<kSplit>()) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (bit) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return MLA_OK;
}

// Launch the tensor-core decode.  With `with_plan` (the non-split path) the
// split plan is computed in the same launch as the query packing; otherwise
// the caller has launched the plan already.
inline mla_status launch(const mla_config* c, const float* q_lat, const float* q_rope, int n_q,
                         const mla_cache* k, const int32_t* seq_lens, void* ws, const DecodeLayout& L,
                         float scale, cudaStream_t s, size_t plan_smem) {
  if (((uintptr_t)k->pool & 15u) != 0 || ((uintptr_t)q_lat & 15u) != 0 || ((uintptr_t)q_rope & 15u) != 0)
    return MLA_ERR_INVALID_ARG;
  CUtensorMap map;
  const mla_status ms = pool_tensor_map(k, &map);
  if (ms != MLA_OK) return ms;
  Params p{q_lat, q_rope, k->block_table, seq_lens, k->max_blocks_per_seq, k->num_blocks, n_q,
           scale * 1.4426950408889634f, ws, L};
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  const dim3 grid(2 * L.workers), block(kThreads);
  if (split) {
    if (set_smem_attr<true>() != MLA_OK) return MLA_ERR_CUDA;
    decode_tc_kernel<true><<<grid, block, smem_bytes<true>(), s>>>(map, p);
  } else {
    static std::atomic<uint64_t> done_mask{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
    if (!bit || !(done_mask.load(std::memory_order_acquire) & bit)) {
      if (cudaFuncSetAttribute(tcdec3::decode_tc3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)tcdec3::kSmemBytes) != cudaSuccess)
        return MLA_ERR_CUDA;
      if (bit) done_mask.fetch_or(bit, std::memory_order_acq_rel);
    }
    const long long rows = (long long)L.batch * L.n_q;
    bf16* qpack = reinterpret_cast<bf16*>(static_cast<char*>(ws) + L.off_qpack);
    CUtensorMap qmap;
    const mla_status qs = qpack_tensor_map(qpack, rows, &qmap);
    if (qs != MLA_OK) return qs;
    const long long groups = rows * kH * (kRow / 8);
    const int qblocks = (int)std::min<long long>((groups + 1023) / 1024, 4096);
    if (plan_smem > 48 * 1024 && cudaFuncSetAttribute(tcdec3::plan_pack_kernel,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      (int)plan_smem) != cudaSuccess)
      return MLA_ERR_CUDA;
    if (launch_chained(tcdec3::plan_pack_kernel, dim3(1 + qblocks), dim3(1024), plan_smem, s, seq_lens, c->block_size,
                       k->max_blocks_per_seq, ws, L, q_lat, q_rope, rows * kH, qpack) != cudaSuccess)
      return MLA_ERR_CUDA;
    const tcdec3::Params p3{q_lat, q_rope, k->block_table, seq_lens, k->max_blocks_per_seq, k->num_blocks, n_q,
                            scale * 1.4426950408889634f, ws, L};
    return launch_chained(tcdec3::decode_tc3_kernel, grid, dim3(tcdec3::kThreads), tcdec3::kSmemBytes, s, map, qmap,
                          p3) == cudaSuccess
               ? MLA_OK
               : MLA_ERR_CUDA;
  }
  note_launch();
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace tcdec
}  // namespace mla

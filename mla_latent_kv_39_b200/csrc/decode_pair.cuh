// Latent-space split-KV decode on pairs of SMs (tcgen05 .cta_group::2).
//
// "MLA · latent KV, decoupled RoPE và matrix absorption" (openarchlab),
// section 1 "Định nghĩa" and section 2 "Luồng": with W_UK absorbed into the
// query and W_UV into the output side, for every head h of query row v
//   s_t = q_lat[h] . c_t + q_R[h] . k_R,t          (t over the visible rows)
//   o_lat[h] = sum_t softmax(scale * s)_t c_t        (the latent output)
// The split-KV plan (decode_plan.cuh) hands every worker one contiguous run
// of pages (one or more query rows, "segments"); per segment the worker
// writes the normalised partial output and its log2-sum-exp.
//
// A worker is a cluster of two CTAs on two SMs.  CTA r owns heads
// [64 r, 64 r + 64): its shared memory holds those heads' query rows and its
// TMEM their scores and their whole 512-wide latent output.  The pages are
// walked two at a time (a 128-token tile); the scores of a tile are one pair
// MMA per 16-value K step, M = 128 heads (A split by heads), N = 128 tokens
// (B split by pages: CTA r holds page r of the tile, all 576 values), so
// every page is read from memory once and every score is computed once.
// P V is a pair MMA per 16 tokens with N = 256 latent columns (B split by
// columns: CTA r loads columns [128 r, 128 r + 128) of each 256-column
// chunk of both pages).  The rows of D that a pair MMA leaves in one CTA's
// TMEM sit in 128 lanes x N/2 columns: lane l holds head 64 r + (l mod 64),
// lanes 0..63 the first half of the N columns and lanes 64..127 the second.
//
// Warp roles (192 threads per CTA): warp 0 issues the TMA loads (both CTAs,
// counted on the leader's barriers); warp 1 of the leader issues every MMA
// of the pair; warps 2..5 run the online softmax, one TMEM lane per thread
// (a head and one page of the tile), and write the segment's partial output.
//
// TMEM (512 columns): [0,64) and [64,128) two score tiles, [128,384) the
// latent output (two 128-column chunks), the rest unused.
//
// Shared memory: the query (9 slabs of 64 heads x 64 values, 128-byte
// swizzle, K-major), a double-buffered P (2 pages x 64 heads x 64 tokens),
// a ring of 8 KiB page slabs for the score MMAs (in split-query mode the
// low query slabs go through the same ring) and a ring of 16 KiB value units
// (one page x 128 latent columns) for P V.
//
// The last page of a row may be partial: it is loaded with its row
// coordinate shifted down by the missing rows, so the rows past the visible
// length arrive as zeros (out-of-range fill) at the top of the tile and the
// pool's contents there (maybe NaN) are never read.  A tile with only one
// page skips the second page's loads and its P V steps.
//
// Every wait gives up after a time limit, records MLA_ERR_TIMEOUT and makes
// the roles wind down.
#pragma once

#include "decode_plan.cuh"
#include "sm100.cuh"

namespace mla {
namespace pairdec {

using namespace sm100;

constexpr int kH = 128, kHalfH = 64, kDc = 512, kDr = 64, kBS = 64, kRow = kDc + kDr;
constexpr int kSlabs = kRow / 64;  // 9 K slabs of 64 values
constexpr int kSlab = 64 * 128;    // 64 rows x 64 bf16, 128-byte swizzle
constexpr int kVUnit = 2 * kSlab;  // one page x 128 latent columns
constexpr int kKcStages = 7, kVcStages = 4;
constexpr int kTmemS = 0, kTmemO = 128, kTmemCols = 512;
constexpr int kSoftmaxWarps = 4;
constexpr int kThreads = 32 * (2 + kSoftmaxWarps);
constexpr float kRescaleLog2 = 8.f;
constexpr uint16_t kBoth = 3;  // multicast mask: both CTAs of the pair

struct Smem {
  uint8_t q[kSlabs][kSlab];      // first member: 1024-byte aligned
  uint8_t p[2][2][kSlab];        // [buffer][page of the tile]
  uint8_t kc[kKcStages][kSlab];  // page slabs (and low query slabs)
  uint8_t vc[kVcStages][kVUnit];
  uint64_t kc_full[kKcStages], kc_empty[kKcStages];
  uint64_t vc_full[kVcStages], vc_empty[kVcStages];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint64_t o_free, fin, xbar[2], lbar;
  float xm[2][128];  // tile max of each TMEM lane (exchanged between lanes l and l ^ 64)
  float xl[128];     // row sums at the end of a segment
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the 227 KiB per-block limit");

struct Params {
  const int32_t* block_table;
  const int32_t* seq_lens;
  int max_blocks, num_blocks, n_q, split;
  float scale_log2;
  unsigned long long wait_ns;
  void* ws;
  DecodeLayout L;
};

__device__ __forceinline__ void set_abort(Smem& sm) { *(volatile int*)&sm.abort_flag = 1; }
__device__ __forceinline__ bool aborted(Smem& sm) { return *(volatile int*)&sm.abort_flag != 0; }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The same barrier in the leader CTA (rank 0), as a shared::cluster address.
__device__ __forceinline__ uint32_t leader(const uint64_t* bar) { return mapa(smem_u32(bar), 0); }

__device__ __forceinline__ uint64_t kmajor_desc(const void* p, uint32_t byte_off) {
  return smem_desc(smem_u32(p) + byte_off, 16, 1024, kSwizzle128B);
}

// Descriptors differ only in the start address (bits 0-13, 16-byte units).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t byte_offset) { return d + (byte_offset >> 4); }

// ---------------------------------------------------------------- tiles
// Walks the worker's tiles in order: segment, first page of the tile.
struct Tiles {
  const int4* segs;
  int si, seg_end, pg, nseg;  // nseg: segments started so far (this one included)
  __device__ Tiles(const int4* s, int b, int e) : segs(s), si(b), seg_end(e), pg(b < e ? s[b].y : 0), nseg(1) {}
  __device__ bool valid() const { return si < seg_end; }
  __device__ int4 seg() const { return segs[si]; }
  __device__ bool first() const { return pg == segs[si].y; }
  __device__ bool last() const { return pg + 2 >= segs[si].z; }
  __device__ bool has_b() const { return pg + 1 < segs[si].z; }
  __device__ void next() {
    pg += 2;
    if (pg >= segs[si].z && ++si < seg_end) {
      pg = segs[si].y;
      ++nseg;
    }
  }
};

// Visible rows of query row v: its sequence's rows up to and including its own.
__device__ __forceinline__ int visible_len(const Params& p, int v) {
  const int b = v / p.n_q, j = v % p.n_q;
  return p.seq_lens[b] - p.n_q + j + 1;
}

__device__ __forceinline__ int page_valid(int len_v, int blk) { return max(0, min(kBS, len_v - blk * kBS)); }

__device__ __forceinline__ int phys_block(const Params& p, int v, int blk, bool report_err) {
  const int b = v / p.n_q;
  int phys = p.block_table[(long long)b * p.max_blocks + blk];
  if (phys < 0 || phys >= p.num_blocks) {
    if (report_err) report(MLA_ERR_BOUNDS, 5, b, phys);
    phys = 0;  // keep the pipeline moving; the error word marks the result invalid
  }
  return phys;
}

// ---------------------------------------------------------------- TMA producer
struct Ring {
  uint32_t n = 0;  // items issued
  template <int S>
  __device__ __forceinline__ bool acquire(uint64_t (&empty)[S], int& slot, int where, uint64_t wait_ns) {
    slot = (int)(n % S);
    const uint32_t use = n / S;
    return use == 0 || mbar_wait<true>(&empty[slot], (use - 1) & 1, where, wait_ns);
  }
};

__device__ void producer(Smem& sm, const CUtensorMap* pool, const CUtensorMap* qmap, const CUtensorMap* qlomap,
                         const Params& p, int seg_begin, int seg_end, uint32_t rank) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const bool lead = rank == 0;
  Ring kc, vc;
  Tiles t(segs, seg_begin, seg_end), tv(segs, seg_begin, seg_end);
  int nq = 0;  // query loads issued
  for (int i = 0;; ++i) {
    if (aborted(sm)) break;
    const bool do_k = t.valid(), do_v = i >= 1 && tv.valid();
    if (!do_k && !do_v) break;
    if (do_k) {
      const int4 sg = t.seg();
      const int v = sg.x;
      if (t.first()) {  // this segment's query rows (64 heads per CTA)
        if (nq >= 1 && !mbar_wait<true>(&sm.q_empty, (nq - 1) & 1, 70, p.wait_ns)) goto fail;
        if (lead) mbar_arrive_expect_tx(&sm.q_full, 2 * kSlabs * kSlab);
        for (int e = 0; e < kSlabs; ++e)
          tma_load_2d_pair(sm.q[e], qmap, 64 * e, v * kH + kHalfH * (int)rank, leader(&sm.q_full));
        ++nq;
      }
      const int len_v = visible_len(p, v);
      const bool has = rank == 0 || t.has_b();
      const int blk = t.pg + (int)rank;
      const int phys = has ? phys_block(p, v, blk, true) : 0;
      const int y = has ? page_valid(len_v, blk) - kBS : 0;
      const uint32_t page_bytes = (t.has_b() ? 2 : 1) * kSlab;
      for (int e = 0; e < kSlabs; ++e) {
        int slot;
        if (!kc.acquire(sm.kc_empty, slot, 71, p.wait_ns)) goto fail;
        if (lead) mbar_arrive_expect_tx(&sm.kc_full[slot], page_bytes);
        if (has) tma_load_3d_pair(sm.kc[slot], pool, 64 * e, y, phys, leader(&sm.kc_full[slot]));
        ++kc.n;
        if (p.split) {  // the low part of the query for the same K slab
          if (!kc.acquire(sm.kc_empty, slot, 72, p.wait_ns)) goto fail;
          if (lead) mbar_arrive_expect_tx(&sm.kc_full[slot], 2 * kSlab);
          tma_load_2d_pair(sm.kc[slot], qlomap, 64 * e, v * kH + kHalfH * (int)rank, leader(&sm.kc_full[slot]));
          ++kc.n;
        }
      }
      t.next();
    }
    if (do_v) {
      const int4 sg = tv.seg();
      const int v = sg.x, len_v = visible_len(p, v);
      const int npg = tv.has_b() ? 2 : 1;
      for (int c = 0; c < 2; ++c)
        for (int q = 0; q < npg; ++q) {
          const int blk = tv.pg + q;
          const int phys = phys_block(p, v, blk, false);
          const int y = page_valid(len_v, blk) - kBS;
          const int x = 256 * c + 128 * (int)rank;
          int slot;
          if (!vc.acquire(sm.vc_empty, slot, 73, p.wait_ns)) goto fail;
          if (lead) mbar_arrive_expect_tx(&sm.vc_full[slot], 2 * kVUnit);
          tma_load_3d_pair(sm.vc[slot], pool, x, y, phys, leader(&sm.vc_full[slot]));
          tma_load_3d_pair(sm.vc[slot] + kSlab, pool, x + 64, y, phys, leader(&sm.vc_full[slot]));
          ++vc.n;
        }
      tv.next();
    }
  }
  return;
fail:
  set_abort(sm);
}

// ---------------------------------------------------------------- MMA issuer (leader CTA)
__device__ void mma_issuer(Smem& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, 256, 0, 1);
  const uint64_t wns = p.wait_ns;
  uint32_t nk = 0, nv = 0;
  Tiles t(segs, seg_begin, seg_end), tv(segs, seg_begin, seg_end);
  for (int i = 0;; ++i) {
    const bool do_k = t.valid(), do_v = i >= 1 && tv.valid();
    if (!do_k && !do_v) break;
    if (do_k) {
      if (t.first() && !mbar_wait<true>(&sm.q_full, (t.nseg - 1) & 1, 80, wns)) goto fail;
      if (i >= 2 && !mbar_wait<true>(&sm.s_free[i & 1], ((i - 2) >> 1) & 1, 81, wns)) goto fail;
      tc_fence_after();
      const uint32_t d = tmem + kTmemS + (i & 1) * 64;
      for (int e = 0; e < kSlabs; ++e) {
        const int slot = (int)(nk % kKcStages);
        if (!mbar_wait<true>(&sm.kc_full[slot], (nk / kKcStages) & 1, 82, wns)) goto fail;
        int lo_slot = 0;
        if (p.split) {
          lo_slot = (int)((nk + 1) % kKcStages);
          if (!mbar_wait<true>(&sm.kc_full[lo_slot], ((nk + 1) / kKcStages) & 1, 83, wns)) goto fail;
        }
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_ss_pair(d, kmajor_desc(sm.q[e], 32 * j), kmajor_desc(sm.kc[slot], 32 * j), idesc_s, (e | j) ? 1u : 0u);
        if (p.split) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_ss_pair(d, kmajor_desc(sm.kc[lo_slot], 32 * j), kmajor_desc(sm.kc[slot], 32 * j), idesc_s, 1u);
          mma_commit_pair(&sm.kc_empty[lo_slot], kBoth);
        }
        mma_commit_pair(&sm.kc_empty[slot], kBoth);
        nk += p.split ? 2 : 1;
      }
      mma_commit_pair(&sm.s_full[i & 1], kBoth);
      if (t.last()) mma_commit_pair(&sm.q_empty, kBoth);
      t.next();
    }
    if (do_v) {
      const int j = i - 1;  // the tile whose P V this is
      if (tv.first() && tv.nseg >= 2 && !mbar_wait<true>(&sm.o_free, (tv.nseg - 2) & 1, 84, wns)) goto fail;
      if (!mbar_wait<true>(&sm.p_full[j & 1], (j >> 1) & 1, 85, wns)) goto fail;
      tc_fence_after();
      const int npg = tv.has_b() ? 2 : 1;
      for (int c = 0; c < 2; ++c)
        for (int q = 0; q < npg; ++q) {
          const int slot = (int)(nv % kVcStages);
          if (!mbar_wait<true>(&sm.vc_full[slot], (nv / kVcStages) & 1, 86, wns)) goto fail;
          tc_fence_after();
          // value unit as an MN-major B operand: 64-column halves 8 KiB apart
          // (LBO), 8-token groups 1 KiB apart (SBO), 16 tokens per K step
          const uint64_t vd = smem_desc(smem_u32(sm.vc[slot]), kSlab, 1024, kSwizzle128B);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss_pair(tmem + kTmemO + 128 * c, kmajor_desc(sm.p[j & 1][q], 32 * kk), desc_add(vd, 2048 * kk),
                        idesc_o, (tv.first() && q == 0 && kk == 0) ? 0u : 1u);
          mma_commit_pair(&sm.vc_empty[slot], kBoth);
          ++nv;
        }
      mma_commit_pair(&sm.pv_done[j & 1], kBoth);
      tv.next();
    }
  }
  mma_commit_pair(&sm.fin, 1);
  mbar_wait(&sm.fin, 0, 87, wns);
  return;
fail:
  set_abort(sm);
  mma_commit_pair(&sm.fin, 1);
  mbar_wait(&sm.fin, 0, 88, wns);
}

// ---------------------------------------------------------------- softmax
#define MLA_WARP_WAIT(expr) (__all_sync(0xffffffffu, (expr)))

__device__ void softmax_role(Smem& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end, uint32_t rank,
                             int warp, int lane) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const int qw = warp & 3;                                 // TMEM lane quarter
  const int l = qw * 32 + lane;                            // TMEM lane
  const int half = l >> 6;                                 // page of the tile / latent half of O
  const int hl = l & 63, head = kHalfH * (int)rank + hl;   // head of this lane
  const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);  // this warp's lane quarter
  const uint64_t wns = p.wait_ns;
  float* part_o = ws_at<float>(p.ws, p.L.off_o);
  float* part_lse = ws_at<float>(p.ws, p.L.off_lse);

  float m_used = -INFINITY, lsum = 0.f;
  int nseg_done = 0;
  Tiles t(segs, seg_begin, seg_end);
  for (int i = 0; t.valid(); ++i, t.next()) {
    const int4 sg = t.seg();
    const int v = sg.x, len_v = visible_len(p, v);
    const bool first = t.first(), last = t.last();
    if (first) {
      m_used = -INFINITY;
      lsum = 0.f;
    }
    if (!MLA_WARP_WAIT(mbar_wait<true>(&sm.s_full[i & 1], (i >> 1) & 1, 90, wns))) goto fail;
    tc_fence_after();
    float s[64];
    {
      uint32_t a[32], b[32];
      tmem_ld32(tl + kTmemS + (i & 1) * 64, a);
      tmem_ld32(tl + kTmemS + (i & 1) * 64 + 32, b);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = __uint_as_float(a[c]);
        s[32 + c] = __uint_as_float(b[c]);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(leader(&sm.s_free[i & 1]));

    // this lane's page: rows past the visible length sit at the top of the tile
    const int blk = t.pg + half;
    const int shift = kBS - ((half == 0 || t.has_b()) ? page_valid(len_v, blk) : 0);
    float m8[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) m8[c] = -INFINITY;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      s[c] = c >= shift ? s[c] * p.scale_log2 : -INFINITY;
      m8[c & 7] = fmaxf(m8[c & 7], s[c]);
    }
    const float m_loc =
        fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    sm.xm[i & 1][l] = m_loc;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.xbar[i & 1]);
    if (!MLA_WARP_WAIT(mbar_wait(&sm.xbar[i & 1], (i >> 1) & 1, 91, wns))) goto fail;
    const float m_tile = fmaxf(m_loc, sm.xm[i & 1][l ^ 64]);

    bool rescale = false;
    float alpha = 1.f;
    if (first) {
      m_used = m_tile;
    } else if (m_tile > m_used + kRescaleLog2) {  // lazy: rescale only when P could grow past 2^8
      alpha = fast_exp2(m_used - m_tile);
      m_used = m_tile;
      rescale = true;
    }
    const float mbase = m_used == -INFINITY ? 0.f : m_used;
    uint32_t pk[32];
    float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float p0 = fast_exp2(s[2 * c] - mbase), p1 = fast_exp2(s[2 * c + 1] - mbase);
      ps[c & 3] += p0 + p1;
      pk[c] = pack_bf16x2(p0, p1);
    }
    lsum = lsum * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));

    // tcgen05.ld / st are warp-collective: the warp rescales when any lane needs it
    const bool warp_rescale = __any_sync(0xffffffffu, rescale);
    if (warp_rescale) {
      // O must hold every earlier tile before it is scaled: wait for P V of tile i - 1
      if (!MLA_WARP_WAIT(mbar_wait<true>(&sm.pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, 92, wns))) goto fail;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        const uint32_t a = tl + kTmemO + c * 32;
        tmem_ld32(a, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
        tmem_st32(a, o);
      }
      tmem_wait_st();
    }
    // P buffer i & 1 is free once P V of tile i - 2 is done
    if (i >= 2 && !MLA_WARP_WAIT(mbar_wait<true>(&sm.pv_done[i & 1], ((i - 2) >> 1) & 1, 93, wns))) goto fail;
    {
      // row hl of this page's P slab, K-major with the 128-byte swizzle
      uint8_t* row = sm.p[i & 1][half] + hl * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(row + ((c ^ (hl & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(leader(&sm.p_full[i & 1]));

    if (last) {
      // epilogue of the segment: O / l and the log2-sum-exp
      sm.xl[l] = lsum;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.lbar);
      if (!MLA_WARP_WAIT(mbar_wait(&sm.lbar, nseg_done & 1, 94, wns))) goto fail;
      const float ltot = lsum + sm.xl[l ^ 64];
      if (!MLA_WARP_WAIT(mbar_wait<true>(&sm.pv_done[i & 1], (i >> 1) & 1, 95, wns))) goto fail;
      tc_fence_after();
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      const int si = t.si;
      // head-minor partial output: the warp's 32 heads of one column are one 128-byte line
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        tmem_ld32(tl + kTmemO + c * 32, o);
        tmem_wait_ld();
        const int d0 = 256 * (c >> 2) + 128 * half + 32 * (c & 3);
        float* out = part_o + ((long long)si * kDc + d0) * kH + head;
#pragma unroll
        for (int k = 0; k < 32; ++k) out[(long long)k * kH] = __uint_as_float(o[k]) * inv;
      }
      if (half == 0) part_lse[(long long)si * kH + head] = ltot > 0.f ? m_used + log2f(ltot) : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader(&sm.o_free));
      ++nseg_done;
    }
  }
  return;
fail:
  set_abort(sm);
}

#undef MLA_WARP_WAIT

// ---------------------------------------------------------------- plan + query pack
// The split plan (block 0) and the query packing (the other blocks) in one
// launch.  The fp32 query rows are packed into bf16 rows [H][d_c + d_r]
// (q_lat then q_rope) so the decode loads them with TMA; in split-query mode
// a second copy holds the bf16 remainder q - bf16(q).
__global__ void __launch_bounds__(1024) pair_plan_pack_kernel(const int32_t* __restrict__ seq_lens, int bs,
                                                              int max_blocks, void* ws, DecodeLayout L,
                                                              const float* __restrict__ q_lat,
                                                              const float* __restrict__ q_rope, long long heads,
                                                              bf16* __restrict__ qpack, bf16* __restrict__ qlo) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0) {
    plan_body(seq_lens, bs, max_blocks, ws, L);
    return;
  }
  constexpr int kPer = kRow / 8;
  for (long long i = (blockIdx.x - 1) * (long long)blockDim.x + threadIdx.x; i < heads * kPer;
       i += (long long)(gridDim.x - 1) * blockDim.x) {
    const long long hrow = i / kPer;
    const int g = (int)(i % kPer);
    const float* src = g < kDc / 8 ? q_lat + hrow * kDc + g * 8 : q_rope + hrow * kDr + (g - kDc / 8) * 8;
    const float4 a = __ldg(reinterpret_cast<const float4*>(src)), b = __ldg(reinterpret_cast<const float4*>(src) + 1);
    const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      hi[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
      const float h0 = __uint_as_float(hi[k] << 16), h1 = __uint_as_float(hi[k] & 0xFFFF0000u);
      lo[k] = pack_bf16x2(x[2 * k] - h0, x[2 * k + 1] - h1);
    }
    *reinterpret_cast<uint4*>(qpack + hrow * kRow + g * 8) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    if (qlo != nullptr)
      *reinterpret_cast<uint4*>(qlo + hrow * kRow + g * 8) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// ---------------------------------------------------------------- kernel
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_pair_kernel(const __grid_constant__ CUtensorMap pool, const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap qlomap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int worker = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKcStages; ++s) {
      mbar_init(&sm.kc_full[s], 1);
      mbar_init(&sm.kc_empty[s], 1);
    }
    for (int s = 0; s < kVcStages; ++s) {
      mbar_init(&sm.vc_full[s], 1);
      mbar_init(&sm.vc_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_free[b], 2 * kSoftmaxWarps);
      mbar_init(&sm.p_full[b], 2 * kSoftmaxWarps);
      mbar_init(&sm.pv_done[b], 1);
      mbar_init(&sm.xbar[b], kSoftmaxWarps);
    }
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    mbar_init(&sm.o_free, 2 * kSoftmaxWarps);
    mbar_init(&sm.fin, 1);
    mbar_init(&sm.lbar, kSoftmaxWarps);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&pool);
    prefetch_tensormap(&qmap);
    if (p.split) prefetch_tensormap(&qlomap);
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive or load
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();  // the plan, the packed query and the appended rows come from the kernels before
  pdl_trigger();

  int seg_begin = 0, seg_end = 0;
  if (worker < p.L.workers) {
    const int* wfirst = ws_at<int>(p.ws, p.L.off_worker_first);
    seg_begin = wfirst[worker];
    seg_end = wfirst[worker + 1];
  }

  // The single-thread roles keep their warp's other lanes parked at a warp
  // barrier (not at the CTA barrier below) while lane 0 works.
  if (warp == 0) {
    if (lane == 0) producer(sm, &pool, &qmap, &qlomap, p, seg_begin, seg_end, rank);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) mma_issuer(sm, tmem, p, seg_begin, seg_end);
    __syncwarp();
  } else {
    softmax_role(sm, tmem, p, seg_begin, seg_end, rank, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs and remote arrives are over before TMEM and shared memory go away
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ================================================================ host side
inline bool supports(const mla_config* c) {
  return c->dtype == MLA_BF16 && c->n_heads == kH && c->d_c == kDc && c->d_r == kDr && c->block_size == kBS;
}

// Bytes of packed query the decode keeps in its workspace per query row
// (the bf16 query, and its bf16 remainder in split-query mode).
inline size_t qpack_row_bytes(const mla_config* c) {
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  return (size_t)kH * kRow * sizeof(bf16) * (split ? 2 : 1);
}

// The pool as a 3-D bf16 tensor [num_blocks][64 rows][576 values] (row
// stride 1152 B, page stride 73,728 B), read in boxes of 64 values x 64 rows
// of one page with the 128-byte swizzle; rows outside the page read as zero.
inline mla_status pool_map(const mla_cache* k, CUtensorMap* map) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return MLA_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)kRow, (cuuint64_t)kBS, (cuuint64_t)k->num_blocks};
  const cuuint64_t strides[2] = {(cuuint64_t)kRow * 2, (cuuint64_t)kRow * 2 * kBS};
  const cuuint32_t box[3] = {64, (cuuint32_t)kBS, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k->pool, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// A packed query (bf16 [rows * 128 heads, 576]) read in boxes of 64 values x
// 64 heads: one box is one shared-memory query slab of one CTA.
inline mla_status query_map(const void* q, long long rows, CUtensorMap* map) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return MLA_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)kRow, (cuuint64_t)rows * kH};
  const cuuint64_t strides[1] = {(cuuint64_t)kRow * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kHalfH};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

inline mla_status set_smem_once(const void* fn, size_t bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done_mask.load(std::memory_order_acquire) & bit)) return MLA_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (bit) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return MLA_OK;
}

// Plan + query pack, then the pair decode (two chained launches).
inline mla_status launch(const mla_config* c, const float* q_lat, const float* q_rope, int n_q, const mla_cache* k,
                         const int32_t* seq_lens, void* ws, const DecodeLayout& L, float scale,
                         unsigned long long wait_ns, cudaStream_t s) {
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  const long long rows = (long long)L.batch * L.n_q;
  bf16* qpack = reinterpret_cast<bf16*>(static_cast<char*>(ws) + L.off_qpack);
  bf16* qlo = split ? qpack + rows * kH * kRow : nullptr;
  CUtensorMap pmap, qmap, qlomap;
  mla_status st = pool_map(k, &pmap);
  if (st == MLA_OK) st = query_map(qpack, rows, &qmap);
  if (st == MLA_OK) st = query_map(split ? qlo : qpack, rows, &qlomap);
  if (st != MLA_OK) return st;

  static std::atomic<uint64_t> plan_attr{0}, dec_attr{0};
  const size_t plan_smem = sizeof(int) * ((size_t)rows + 1);
  if (plan_smem > 48 * 1024 && set_smem_once((const void*)pair_plan_pack_kernel, plan_smem, plan_attr) != MLA_OK)
    return MLA_ERR_CUDA;
  if (set_smem_once((const void*)decode_pair_kernel, kSmemBytes, dec_attr) != MLA_OK) return MLA_ERR_CUDA;

  const long long groups = rows * kH * (kRow / 8);
  const int qblocks = (int)std::min<long long>((groups + 1023) / 1024, 4096);
  if (launch_chained(pair_plan_pack_kernel, dim3(1 + qblocks), dim3(1024), plan_smem, s, seq_lens, c->block_size,
                     k->max_blocks_per_seq, ws, L, q_lat, q_rope, rows * kH, qpack, qlo) != cudaSuccess)
    return MLA_ERR_CUDA;
  const Params p{k->block_table, seq_lens, k->max_blocks_per_seq, k->num_blocks, n_q, split ? 1 : 0,
                 scale * 1.4426950408889634f, wait_ns, ws, L};
  return launch_chained(decode_pair_kernel, dim3(2 * L.workers), dim3(kThreads), kSmemBytes, s, pmap, qmap, qlomap,
                        p) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace pairdec
}  // namespace mla

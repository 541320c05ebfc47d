// Latent-space split-KV decode on the sm_100 tensor cores, pipelined form.
//
// Same work split as decode_tc.cuh (a 2-CTA cluster per worker, the 576-wide
// latent row split by columns, partial scores exchanged through distributed
// shared memory) with the per-page latency chain broken up:
//  * two score tiles in TMEM; P (bf16) is written over the score tile it came
//    from, so the MMA warp computes the scores of page k+1 (and k+2) while the
//    softmax works on page k, and a P store never waits for the previous P V;
//  * the partial scores of page k+1 go to the peer as soon as they exist -
//    before page k is processed when the MMA warp is ahead - through st.async
//    stores into the peer's shared memory, counted in bytes on the peer's
//    mbarrier (no fence); each CTA tells the peer when it has read a buffer
//    (xempty, a relaxed remote arrive) before the peer refills it;
//  * eight softmax warps: the two warps of a TMEM lane quarter split the 64
//    tokens of a page (32 each) and meet once per page to agree on the row max;
//  * the producer prefetches pages into L2 several pages ahead of the shared
//    memory stages, so a stage load mostly hits L2;
//  * one mbarrier per score buffer, so no wait ever runs more than one phase
//    behind its barrier.
//
// TMEM columns: [0, 256) O, [256, 320) and [320, 384) score/P tiles, [384,
// 512) this CTA's half of q_lat (bf16 pairs).  CTA 1 also holds the rotary
// query (bf16, 128 x 64) in shared memory as the A operand of its last four
// score K-steps.
#pragma once

#include "decode_plan.cuh"
#include "sm100.cuh"

namespace mla {
namespace tcdec2 {

using namespace sm100;

constexpr int kH = 128, kDc = 512, kDr = 64, kBS = 64;
constexpr int kSlabBytes = 64 * 128;                 // 64 rows x 64 bf16 (128 B), swizzled
constexpr int kStages = 3;
constexpr int kPrefetch = 8;                         // pages prefetched into L2 ahead of the stages
constexpr int kStageBytes = 5 * kSlabBytes;          // 40 KiB (CTA 0 uses 4 slabs)
constexpr int kQropeBytes = 128 * 128;               // 128 rows x 64 bf16, swizzled
constexpr int kTmemO = 0, kTmemSP = 256, kTmemQ = 384, kTmemCols = 512;
constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr int kThreads = 64 + kSoftmaxThreads;       // producer warp, MMA warp, softmax warps
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kXStageBytes = kH * 64 * 4;       // one exchanged score tile

struct Smem {
  uint8_t kv[kStages][kStageBytes];  // first member: 1024-byte aligned
  uint8_t qrope[kQropeBytes];        // CTA 1: rotary query, K-major, 128-byte swizzle
  // Exchanged partial scores: one 4 KiB block per softmax warp (32 rows x 32
  // tokens); the 16-byte chunk c of a row sits at chunk position c ^ (row & 7).
  float xrecv[2][kSoftmaxWarps][32][32];  // from the peer, per score buffer
  float rowx[2][4][2][32];           // per page parity, lane quarter, column half: partial max
  float rowl[4][2][32];              // partial row sums at a segment's end
  uint64_t full[kStages], empty[kStages];
  uint64_t s_full[2], p_ready[2], pv_done[2], xfull[2], xempty[2];
  uint64_t q_ready, mma_done;
  uint64_t rowsync[4];               // the two softmax warps of a lane quarter
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

struct Params {
  const float* q_lat;   // [rows, 128, 512]
  const float* q_rope;  // [rows, 128, 64]
  const int32_t* block_table;
  const int32_t* seq_lens;
  int max_blocks, num_blocks, n_q;
  float scale_log2;
  void* ws;
  DecodeLayout L;
};

__device__ __forceinline__ void set_abort(Smem& sm) { *(volatile int*)&sm.abort_flag = 1; }
__device__ __forceinline__ bool aborted(Smem& sm) { return *(volatile int*)&sm.abort_flag != 0; }

// 16-byte store into the peer CTA's shared memory, counted in bytes on the
// peer's mbarrier (no fence: the barrier's transaction count orders it).
__device__ __forceinline__ void st_async_v4(uint32_t addr, float a, float b, float c, float d, uint32_t mbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
               ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d), "r"(mbar)
               : "memory");
}

// Arrive on a barrier of the peer CTA without ordering earlier memory
// operations (the shared-memory reads it reports have already been consumed).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void prefetch_l2_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}


__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- TMA producer
// Walks the worker's pages in order: (segment, page) -> physical block.
struct PageCursor {
  const int4* segs;
  int si, seg_end, blk;
  __device__ bool valid() const { return si < seg_end; }
  __device__ void next() {
    if (++blk >= segs[si].z) {
      if (++si < seg_end) blk = segs[si].y;
    }
  }
};

__device__ __forceinline__ int phys_block(const Params& p, const int4* segs, const PageCursor& c, bool report_err) {
  const int b = segs[c.si].x / p.n_q;
  int phys = p.block_table[(long long)b * p.max_blocks + c.blk];
  if (phys < 0 || phys >= p.num_blocks) {
    if (report_err) report(MLA_ERR_BOUNDS, 5, b, phys);
    phys = 0;  // keep the pipeline moving; the error word marks the result invalid
  }
  return phys;
}

__device__ void producer(Smem& sm, const CUtensorMap* tmap, const Params& p, int seg_begin, int seg_end,
                         uint32_t crank, int nslab) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  PageCursor cur{segs, seg_begin, seg_end, seg_begin < seg_end ? segs[seg_begin].y : 0};
  PageCursor ahead = cur;
  // skip empty segments (cannot happen: every segment has >= 1 page)
  for (int i = 0; i < kPrefetch && ahead.valid(); ++i, ahead.next())
    for (int s = 0; s < nslab; ++s)
      prefetch_l2_2d(tmap, (int)crank * 256 + s * 64, phys_block(p, segs, ahead, false) * kBS);
  int k = 0;
  for (; cur.valid() && !aborted(sm); cur.next(), ++k) {
    const int stage = k % kStages;
    if (k >= kStages && !mbar_wait(&sm.empty[stage], ((k / kStages) - 1) & 1, 40)) {
      set_abort(sm);
      break;
    }
    if (ahead.valid()) {
      for (int s = 0; s < nslab; ++s)
        prefetch_l2_2d(tmap, (int)crank * 256 + s * 64, phys_block(p, segs, ahead, false) * kBS);
      ahead.next();
    }
    const int phys = phys_block(p, segs, cur, true);
    mbar_arrive_expect_tx(&sm.full[stage], (uint32_t)(nslab * kSlabBytes));
    for (int s = 0; s < nslab; ++s)
      tma_load_2d(sm.kv[stage] + s * kSlabBytes, tmap, (int)crank * 256 + s * 64, phys * kBS, &sm.full[stage]);
  }
  // never leave a copy in flight into shared memory that is about to be released
  for (int kk = k - kStages < 0 ? 0 : k - kStages; kk < k; ++kk)
    mbar_wait(&sm.full[kk % kStages], (kk / kStages) & 1, 41);
}

// ---------------------------------------------------------------- MMA issuer
struct MmaDescs {
  uint64_t kv0;     // K-major view of stage 0, slab 0, K step 0
  uint64_t pv0;     // MN-major view of stage 0 (V slabs)
  uint64_t qrope0;  // K-major rotary query
};

// Descriptors differ only in the start address (bits 0-13, in 16-byte units).
__device__ __forceinline__ uint64_t desc_at(uint64_t d, uint32_t byte_offset) { return d + (byte_offset >> 4); }

// Scores of global page kk into score buffer kk % 2.
__device__ __forceinline__ bool issue_scores(Smem& sm, const MmaDescs& md, uint32_t tmem, int kk, uint32_t crank) {
  const int stage = kk % kStages, buf = kk & 1;
  if (!mbar_wait(&sm.full[stage], (kk / kStages) & 1, 50)) return false;
  // the buffer's previous P (page kk - 2) must have been consumed
  if (kk >= 2 && !mbar_wait(&sm.pv_done[buf], ((kk - 2) >> 1) & 1, 51)) return false;
  tc_fence_after();
  constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
  const uint32_t d = tmem + kTmemSP + buf * 64;
  const uint64_t b0 = desc_at(md.kv0, stage * kStageBytes);
#pragma unroll
  for (int j = 0; j < 16; ++j)
    mma_ts(d, tmem + kTmemQ + j * 8, desc_at(b0, (j >> 2) * kSlabBytes + (j & 3) * 32), idesc, j > 0 ? 1u : 0u);
  if (crank == 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      mma_ss(d, desc_at(md.qrope0, j * 32), desc_at(b0, 4 * kSlabBytes + j * 32), idesc, 1u);
  }
  mma_commit(&sm.s_full[buf]);
  return true;
}

__device__ void mma_issuer(Smem& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end, uint32_t crank) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
  // K-major page slab: tokens 128 B apart, 8-token groups 1 KiB apart (SBO).
  // MN-major page slabs (P V): 64-dim chunks 8 KiB apart (LBO), 8-token
  // groups 1 KiB apart (SBO); K step j (16 tokens) starts 2 KiB further.
  const MmaDescs md{smem_desc(smem_u32(sm.kv[0]), 16, 1024, kSwizzle128B),
                    smem_desc(smem_u32(sm.kv[0]), kSlabBytes, 1024, kSwizzle128B),
                    smem_desc(smem_u32(sm.qrope), 16, 1024, kSwizzle128B)};
  int k = 0, seg_i = 0;
  for (int si = seg_begin; si < seg_end; ++si, ++seg_i) {
    const int4 sg = segs[si];
    const int T = sg.z - sg.y;
    if (!mbar_wait(&sm.q_ready, seg_i & 1, 52)) goto fail;
    for (int i = 0; i < T && i < 2; ++i)
      if (!issue_scores(sm, md, tmem, k + i, crank)) goto fail;
    for (int i = 0; i < T; ++i) {
      const int kk = k + i, buf = kk & 1;
      if (!mbar_wait(&sm.p_ready[buf], (kk >> 1) & 1, 53)) goto fail;
      tc_fence_after();
      const uint64_t v0 = desc_at(md.pv0, (kk % kStages) * kStageBytes);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        mma_ts(tmem + kTmemO, tmem + kTmemSP + buf * 64 + j * 8, desc_at(v0, j * 2048), idesc_pv,
               (i > 0 || j > 0) ? 1u : 0u);
      mma_commit(&sm.pv_done[buf]);
      mma_commit(&sm.empty[kk % kStages]);
      if (i + 2 < T && !issue_scores(sm, md, tmem, kk + 2, crank)) goto fail;
    }
    k += T;
  }
  mma_commit(&sm.mma_done);
  mbar_wait(&sm.mma_done, 0, 54);
  return;
fail:
  set_abort(sm);
  mma_commit(&sm.mma_done);
  mbar_wait(&sm.mma_done, 0, 55);
}

// ---------------------------------------------------------------- softmax
#define MLA_WARP_WAIT(expr) (__all_sync(0xffffffffu, (expr)))

// This thread's share of row r of the query: half (ch) of the CTA's q_lat
// columns -> TMEM (bf16 pairs); on CTA 1 also half of the rotary query ->
// shared memory, K-major with the 128-byte swizzle.
__device__ __forceinline__ void load_query(const Params& p, Smem& sm, int v, int r, int ch, uint32_t crank,
                                           uint32_t taddr) {
  const float* ql = p.q_lat + ((long long)v * kH + r) * kDc + crank * 256 + ch * 128;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {  // 32 values per chunk
    const float4* src = reinterpret_cast<const float4*>(ql + c * 32);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 f = __ldg(src + i);
      w[2 * i] = pack_bf16x2(f.x, f.y);
      w[2 * i + 1] = pack_bf16x2(f.z, f.w);
    }
    tmem_st16(taddr + ch * 64 + c * 16, w);
  }
  if (crank == 1) {
    const float4* src = reinterpret_cast<const float4*>(p.q_rope + ((long long)v * kH + r) * kDr + ch * 32);
    uint8_t* row = sm.qrope + r * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c) {  // 16-byte chunk 4 ch + c holds values 8 (4 ch + c) .. + 7
      const float4 f0 = __ldg(src + 2 * c), f1 = __ldg(src + 2 * c + 1);
      const int chunk = ch * 4 + c;
      *reinterpret_cast<uint4*>(row + ((chunk ^ (r & 7)) * 16)) =
          make_uint4(pack_bf16x2(f0.x, f0.y), pack_bf16x2(f0.z, f0.w), pack_bf16x2(f1.x, f1.y),
                     pack_bf16x2(f1.z, f1.w));
    }
    fence_proxy_async_smem();
  }
}

__device__ __forceinline__ void load_scores32(uint32_t taddr, float (&s)[32]) {
  uint32_t a[32];
  tmem_ld32(taddr, a);
  tmem_wait_ld();
#pragma unroll
  for (int t = 0; t < 32; ++t) s[t] = __uint_as_float(a[t]);
}

__device__ void softmax_role(Smem& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end,
                             uint32_t crank, int warp, int lane) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const int qw = warp & 3;                                 // TMEM lane quarter
  const int ch = (warp - 2) >> 2;                          // which 32 tokens of a page
  const int r = qw * 32 + lane;                            // head row == TMEM lane
  const int tid = (warp - 2) * 32 + lane;                  // 0..255
  uint64_t* rowsync = &sm.rowsync[qw];                     // the two warps of this lane quarter
  int rs_phase = 0;
  const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);  // this warp's lane quarter
  const uint32_t peer = crank ^ 1u;
  const int wi = warp - 2;                                 // softmax warp index 0..7
  const uint32_t xrow_peer = mapa(smem_u32(&sm.xrecv[0][wi][lane][0]), peer);
  const uint32_t xfull_peer[2] = {mapa(smem_u32(&sm.xfull[0]), peer), mapa(smem_u32(&sm.xfull[1]), peer)};
  const uint32_t xempty_peer[2] = {mapa(smem_u32(&sm.xempty[0]), peer), mapa(smem_u32(&sm.xempty[1]), peer)};
  const int xsw = lane & 7;
  float* part_o = ws_at<float>(p.ws, p.L.off_o);
  float* part_lse = ws_at<float>(p.ws, p.L.off_lse);

  // This thread's 32 partial scores of page kk: TMEM -> registers -> the
  // peer's buffer kk % 2, once the peer has read what it held (page kk - 2).
  auto fetch_and_send = [&](int kk, float (&s)[32]) -> bool {
    const int buf = kk & 1;
    if (!MLA_WARP_WAIT(mbar_wait(&sm.s_full[buf], (kk >> 1) & 1, 60))) return false;
    tc_fence_after();
    load_scores32(tl + kTmemSP + buf * 64 + ch * 32, s);
    if (kk >= 2 && !MLA_WARP_WAIT(mbar_wait(&sm.xempty[buf], ((kk >> 1) - 1) & 1, 64))) return false;
    const uint32_t dst = xrow_peer + buf * kXStageBytes;
#pragma unroll
    for (int c = 0; c < 8; ++c)
      st_async_v4(dst + ((c ^ xsw) * 16), s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3], xfull_peer[buf]);
    return true;
  };
  // Whether page kk's scores are already in TMEM (no waiting).
  auto scores_ready = [&](int kk) -> bool {
    return __all_sync(0xffffffffu, mbar_test(&sm.s_full[kk & 1], (kk >> 1) & 1));
  };

  int k = 0;
  for (int si = seg_begin; si < seg_end; ++si) {
    const int4 sg = segs[si];
    const int v = sg.x, b = v / p.n_q, jq = v % p.n_q;
    const int len_v = p.seq_lens[b] - p.n_q + jq + 1;
    const int T = sg.z - sg.y;

    load_query(p, sm, v, r, ch, crank, tl + kTmemQ);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&sm.q_ready);

    float m_used = -INFINITY, l = 0.f;
    float sa[32], sb[32];
    if (!fetch_and_send(k, sa)) goto fail;
    for (int i = 0; i < T; ++i) {
      const int kk = k + i, buf = kk & 1, blk = sg.y + i;
      bool sent_next = false;
      // the peer's half of page kk (32 KiB counted on this barrier)
      if (tid == 0) mbar_arrive_expect_tx(&sm.xfull[buf], kXStageBytes);
      if (!MLA_WARP_WAIT(mbar_wait(&sm.xfull[buf], (kk >> 1) & 1, 61))) goto fail;
      {
        const float4* peer_s = reinterpret_cast<const float4*>(&sm.xrecv[buf][wi][lane][0]);
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 t4 = peer_s[c4 ^ xsw];
          sa[4 * c4] += t4.x;
          sa[4 * c4 + 1] += t4.y;
          sa[4 * c4 + 2] += t4.z;
          sa[4 * c4 + 3] += t4.w;
        }
      }
      mbar_arrive_cluster_relaxed(xempty_peer[buf]);  // buffer read: the peer may refill it
      // Send the next page's scores now if the MMA warp already has them;
      // otherwise process this page first and send them afterwards.
      if (i + 1 < T && scores_ready(kk + 1)) {
        if (!fetch_and_send(kk + 1, sb)) goto fail;
        sent_next = true;
      }

      // scale, mask past the sequence end, and the row max over both halves
      const int valid = min(kBS, len_v - blk * kBS) - ch * 32;
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        sa[t] = t < valid ? sa[t] * p.scale_log2 : -INFINITY;
        m8[t & 7] = fmaxf(m8[t & 7], sa[t]);
      }
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      sm.rowx[buf][qw][ch][lane] = mx;
      mbar_arrive(rowsync);
      if (!MLA_WARP_WAIT(mbar_wait(rowsync, (rs_phase++) & 1, 65))) goto fail;
      mx = fmaxf(mx, sm.rowx[buf][qw][ch ^ 1][lane]);

      bool rescale = false;
      float alpha = 1.f;
      if (i == 0) {
        m_used = mx;
      } else if (mx > m_used + kRescaleLog2) {
        alpha = fast_exp2(m_used - mx);
        m_used = mx;
        rescale = true;
      }
      uint32_t pk[16];
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float p0 = fast_exp2(sa[2 * t] - m_used), p1 = fast_exp2(sa[2 * t + 1] - m_used);
        ps[t & 3] += p0 + p1;
        pk[t] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));

      // tcgen05.ld / st are warp-collective: the warp rescales when any row needs it.
      if (__any_sync(0xffffffffu, rescale)) {
        // O must hold every earlier page before it is scaled: wait for P V of page kk - 1.
        if (!MLA_WARP_WAIT(mbar_wait(&sm.pv_done[buf ^ 1], ((kk - 1) >> 1) & 1, 62))) goto fail;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          const uint32_t a = tl + kTmemO + ch * 128 + c * 32;
          tmem_ld32(a, o);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
          tmem_st32(a, o);
        }
      }
      if (min(kBS, len_v - blk * kBS) < kBS) {
        // Rows past the sequence end hold whatever the pool holds (maybe NaN);
        // P is 0 there, but 0 x NaN is NaN, so clear them in the V slabs.
        const int vrows = min(kBS, len_v - blk * kBS);
        uint8_t* stage = sm.kv[kk % kStages];
        const int nrow = kBS - vrows, per_slab = nrow * 8;
        for (int c = tid; c < 4 * per_slab; c += kSoftmaxThreads) {
          const int slab = c / per_slab, rem = c % per_slab;
          *reinterpret_cast<uint4*>(stage + slab * kSlabBytes + (vrows + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tmem_st16(tl + kTmemSP + buf * 64 + ch * 16, pk);  // P over the page's own scores
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_ready[buf]);
      if (i + 1 < T && !sent_next && !fetch_and_send(kk + 1, sb)) goto fail;
#pragma unroll
      for (int t = 0; t < 32; ++t) sa[t] = sb[t];
    }
    {
      // epilogue of the segment: O / l and the log2-sum-exp
      sm.rowl[qw][ch][lane] = l;
      mbar_arrive(rowsync);
      if (!MLA_WARP_WAIT(mbar_wait(rowsync, (rs_phase++) & 1, 66))) goto fail;
      const float lt = l + sm.rowl[qw][ch ^ 1][lane];
      const int kl = k + T - 1;
      if (!MLA_WARP_WAIT(mbar_wait(&sm.pv_done[kl & 1], (kl >> 1) & 1, 63))) goto fail;
      tc_fence_after();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      float4* out = reinterpret_cast<float4*>(part_o + ((long long)si * kH + r) * kDc + crank * 256 + ch * 128);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tl + kTmemO + ch * 128 + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 8; ++t)
          out[c * 8 + t] = make_float4(__uint_as_float(o[4 * t]) * inv, __uint_as_float(o[4 * t + 1]) * inv,
                                       __uint_as_float(o[4 * t + 2]) * inv, __uint_as_float(o[4 * t + 3]) * inv);
      }
      if (crank == 0 && ch == 0) part_lse[(long long)si * kH + r] = lt > 0.f ? m_used + log2f(lt) : -INFINITY;
      mbar_arrive(rowsync);  // rowl is reused by the next segment
      if (!MLA_WARP_WAIT(mbar_wait(rowsync, (rs_phase++) & 1, 67))) goto fail;
    }
    k += T;
  }
  return;
fail:
  set_abort(sm);
}

// ---------------------------------------------------------------- kernel
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_tc2_kernel(const __grid_constant__ CUtensorMap tmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const int worker = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_ready[b], kSoftmaxThreads);
      mbar_init(&sm.pv_done[b], 1);
      mbar_init(&sm.xfull[b], 1);
      mbar_init(&sm.xempty[b], kSoftmaxThreads);
    }
    mbar_init(&sm.q_ready, kSoftmaxThreads);
    for (int q = 0; q < 4; ++q) mbar_init(&sm.rowsync[q], 64);
    mbar_init(&sm.mma_done, 1);
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
  cluster_sync();  // the peer's barriers exist before anyone signals them
  const uint32_t tmem = sm.tmem_base;

  int seg_begin = 0, seg_end = 0;
  if (worker < p.L.workers) {
    const int* wfirst = ws_at<int>(p.ws, p.L.off_worker_first);
    seg_begin = wfirst[worker];
    seg_end = wfirst[worker + 1];
  }

  if (warp == 0) {
    if (lane == 0) producer(sm, &tmap, p, seg_begin, seg_end, crank, crank == 0 ? 4 : 5);
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(sm, tmem, p, seg_begin, seg_end, crank);
  } else {
    softmax_role(sm, tmem, p, seg_begin, seg_end, crank, warp, lane);
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

#undef MLA_WARP_WAIT

}  // namespace tcdec2
}  // namespace mla

// Forward and merge kernels for sm_100a.
//
// Forward (the PAT review, section 三, Forward 阶段 and Figure 3: decode attention
// is two GEMVs, q.K^T then p.V, fed by a tiling pipeline that streams KV tiles
// from global memory through on-chip memory; multi-tile kernels with a runtime
// tile selector; multi-stream execution; long KV is split).  Two tile classes,
// chosen by the planner from the rows of each work unit (requests x G query
// heads), run as two concurrent launches of one persistent CTA per SM:
//   - MMA class: work units with two or more requests, up to 128 rows.  A
//     producer warp streams 64-key stages with 2-D TMA copies (128-byte
//     swizzle); 8 consumer warps each run bf16 mma.sync with fp32 accumulation
//     on 16 rows.
//   - SIMT class: work units of one request (G <= 8 rows).  Each of 8 warps
//     streams its own run of (page, kv head) tiles with 1-D bulk copies into a
//     private shared-memory ring and computes on the CUDA cores with packed
//     fp32x2 FMAs.
// Both emit, per (request, kv head, key range), the normalised partial output
// o = sum_t e^{s_t - m} v_t / l and lse = m + ln l in fp32.
//
// Merge (Merge 阶段: an online-softmax combine of each query's partial results
// across CTAs): LSE = log sum_j e^{lse_j}, out = sum_j e^{lse_j - LSE} o_j.  In
// the fused path the warp that writes the last partial row of a (request, kv
// head) merges it (arrival counter per pair); the same warp-level routine also
// runs as a stand-alone merge launch.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "plan.h"
#include "ptx.cuh"

namespace pa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kSmemMax = 232448;  // opt-in shared memory per CTA on sm_100

struct FwdArgs {
  const uint16_t* q;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  const pa_item* items;
  const pa_seg* segs;
  const int32_t* pages;
  const int32_t* queries;
  const int32_t* seg_prows;
  const int32_t* warp_segs;
  const int32_t* warp_loads;
  const int32_t* tiles;
  const int32_t* mma_cta_segs;
  const int32_t* prow_off;
  int32_t* counters;
  float* partial_lse;
  float* partial_o;
  int32_t* status;
  __nv_bfloat16* out;  // non-null: fused merge
  float* lse;
  int Hq, Hkv, G, n_simt_warps, n_segs_simt, n_mma_ctas;
  float qscale;  // softmax scale * log2(e): scores are kept in base-2 units
  uint64_t timeout_ns;
  int fault_drop;
};

// ---------------------------------------------------------------- merge of one (request, kv head)

// One warp merges the partial rows of (b, g) into out[b][g*G .. g*G+G-1][:] and
// lse[b][...].  Partial rows are read through L2 (they may have been written by
// other SMs in the same launch).
template <int D>
__device__ __forceinline__ void merge_pair(const int32_t* prow_off, const float* partial_lse, const float* partial_o,
                                           __nv_bfloat16* out, float* lse, int Hq, int Hkv, int G, int b, int g,
                                           int lane) {
  constexpr int VD = D / 32;
  const int p0 = prow_off[b * Hkv + g], p1 = prow_off[b * Hkv + g + 1];
  for (int r = 0; r < G; ++r) {
    float mx = -INFINITY;
    for (int p = p0; p < p1; ++p) mx = fmaxf(mx, __ldcg(partial_lse + (size_t)p * G + r));
    float z = 0.f;
    for (int p = p0; p < p1; ++p) z += expf(__ldcg(partial_lse + (size_t)p * G + r) - mx);
    const float L = mx + logf(z);
    float acc[VD];
#pragma unroll
    for (int i = 0; i < VD; ++i) acc[i] = 0.f;
    for (int p = p0; p < p1; ++p) {
      const float wgt = expf(__ldcg(partial_lse + (size_t)p * G + r) - L);
      const float* src = partial_o + ((size_t)p * G + r) * D + lane * VD;
      if constexpr (VD == 4) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
        acc[0] += wgt * v.x;
        acc[1] += wgt * v.y;
        acc[2] += wgt * v.z;
        acc[3] += wgt * v.w;
      } else {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
        acc[0] += wgt * v.x;
        acc[1] += wgt * v.y;
      }
    }
    const int h = g * G + r;
    __nv_bfloat16* dst = out + ((size_t)b * Hq + h) * D + lane * VD;
#pragma unroll
    for (int i = 0; i < VD; i += 2)
      *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i], acc[i + 1]);
    if (lse && lane == 0) lse[(size_t)b * Hq + h] = L;
  }
}

// Called by a whole warp after it wrote partial rows of (b, g): counts the
// arrival and merges the pair if this was the last of its partial rows.
template <int D>
__device__ __forceinline__ void arrive_and_merge(const FwdArgs& a, int b, int g, int lane) {
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) {
    const int bg = b * a.Hkv + g;
    const int n = a.prow_off[bg + 1] - a.prow_off[bg];
    last = atomicAdd(&a.counters[bg], 1) == n - 1;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) {
    __threadfence();
    merge_pair<D>(a.prow_off, a.partial_lse, a.partial_o, a.out, a.lse, a.Hq, a.Hkv, a.G, b, g, lane);
    __syncwarp();
    if (lane == 0) a.counters[b * a.Hkv + g] = 0;  // ready for the next launch
  }
}

// ---------------------------------------------------------------- SIMT class

template <int D, int G>
struct SimtShape {
  static constexpr int DPL = (64 / G) < (D / 2) ? (64 / G) : (D / 2);  // head dims per lane
  static constexpr int LPG = D / DPL;                                  // lanes per key group
  static constexpr int NG = 32 / LPG;                                  // key groups per warp
  static constexpr int KPG = 16 / NG;                                  // keys per group per page
  static constexpr int CPL = DPL / 8;                                  // 16-byte chunks per lane per row
  static constexpr int TILE = 16 * D * 2;                              // one (page, kv head) tile
  static constexpr int QT = G * D * 2;                                 // the G query rows
  static constexpr int STAGE = 2 * TILE;
  static constexpr int W = kSimtWarpsPerCta;
  static constexpr int NST_FIT = (kSmemMax - W * (2 * QT + 8 * 8)) / (W * STAGE);
  static constexpr int NST = NST_FIT < (D == 128 ? 3 : 6) ? NST_FIT : (D == 128 ? 3 : 6);  // ring stages
  static constexpr int WARP_BYTES = NST * STAGE + 2 * QT;
  static constexpr int SMEM = W * WARP_BYTES + W * (NST + 2) * 8;
  static_assert(NG * LPG == 32 && KPG * NG == 16 && DPL % 8 == 0, "bad SIMT shape");
  static_assert(NST >= 2 && SMEM <= kSmemMax, "SIMT ring does not fit in shared memory");
};

struct SegInfo {
  int n_tokens, prow, query, kv_head;
};

__device__ __forceinline__ SegInfo load_seg(const pa_seg* segs, int i, int end) {
  SegInfo r{0, 0, 0, 0};
  if (i < end) {
    const int4 x = *reinterpret_cast<const int4*>(segs + i);        // item, kv_head, page_begin, n_tokens
    const int2 y = *reinterpret_cast<const int2*>(&segs[i].prow);  // prow, query
    r.n_tokens = x.w;
    r.kv_head = x.y;
    r.prow = y.x;
    r.query = y.y;
  }
  return r;
}

// One page of 16 keys for one warp: scores, online softmax, p.V.  PARTIAL: the
// page holds fewer than 16 valid keys (its tail may hold NaN).
template <int D, int G, bool PARTIAL>
__device__ __forceinline__ void simt_page(const uint8_t* kt, const uint8_t* vt, int nvalid, int grp, int li,
                                          const float2 (&qf)[G][SimtShape<D, G>::CPL][4],
                                          float2 (&o)[G][SimtShape<D, G>::CPL][4], float (&m)[G], float (&l)[G]) {
  using S = SimtShape<D, G>;
  constexpr int LPG = S::LPG, KPG = S::KPG, CPL = S::CPL;
  float s[KPG][G];
#pragma unroll
  for (int kk = 0; kk < KPG; ++kk) {
    const int key = grp * KPG + kk;
    const uint32_t msk = (!PARTIAL || key < nvalid) ? 0xffffffffu : 0u;
    float2 acc[G];
#pragma unroll
    for (int r = 0; r < G; ++r) acc[r] = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      uint4 w = *reinterpret_cast<const uint4*>(kt + key * D * 2 + (li + LPG * j) * 16);
      if (PARTIAL) {
        w.x &= msk;
        w.y &= msk;
        w.z &= msk;
        w.w &= msk;
      }
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 kf = bf16x2_to_f2(ws[e]);
#pragma unroll
        for (int r = 0; r < G; ++r) acc[r] = ffma2(qf[r][j][e], kf, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < G; ++r) s[kk][r] = acc[r].x + acc[r].y;
  }
#pragma unroll
  for (int off = 1; off < LPG; off <<= 1)
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk)
#pragma unroll
      for (int r = 0; r < G; ++r) s[kk][r] += __shfl_xor_sync(0xffffffffu, s[kk][r], off);
  if (PARTIAL) {
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk)
      if (grp * KPG + kk >= nvalid)
#pragma unroll
        for (int r = 0; r < G; ++r) s[kk][r] = -INFINITY;
  }
  // online softmax (per group; every lane of a group holds the same values)
  bool grow = false;
  float mnew[G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    float pm = s[0][r];
#pragma unroll
    for (int kk = 1; kk < KPG; ++kk) pm = fmaxf(pm, s[kk][r]);
    mnew[r] = fmaxf(m[r], pm);
    grow |= mnew[r] > m[r];
  }
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int r = 0; r < G; ++r) {
      if (mnew[r] > m[r]) {
        const float alpha = ex2(m[r] - mnew[r]);
        l[r] *= alpha;
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[r][j][e] = fmul2(o[r][j][e], a2);
        m[r] = mnew[r];
      }
    }
  }
  float2 p[KPG][G];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    const float mr = m[r] == -INFINITY ? 0.f : m[r];
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk) {
      const float pv = ex2(s[kk][r] - mr);
      p[kk][r] = make_float2(pv, pv);
      l[r] += pv;
    }
  }
#pragma unroll
  for (int kk = 0; kk < KPG; ++kk) {
    const int key = grp * KPG + kk;
    const uint32_t msk = (!PARTIAL || key < nvalid) ? 0xffffffffu : 0u;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      uint4 w = *reinterpret_cast<const uint4*>(vt + key * D * 2 + (li + LPG * j) * 16);
      if (PARTIAL) {
        w.x &= msk;
        w.y &= msk;
        w.z &= msk;
        w.w &= msk;
      }
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 vf = bf16x2_to_f2(ws[e]);
#pragma unroll
        for (int r = 0; r < G; ++r) o[r][j][e] = ffma2(p[kk][r], vf, o[r][j][e]);
      }
    }
  }
}

template <int D, int G>
__device__ __forceinline__ void simt_role(const FwdArgs& a, uint8_t* smem) {
  using S = SimtShape<D, G>;
  constexpr int NST = S::NST, LPG = S::LPG, CPL = S::CPL;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= kSimtWarpsPerCta) return;
  const int gw = blockIdx.x * kSimtWarpsPerCta + warp;
  if (gw >= a.n_simt_warps) return;  // no block-wide barrier in this role
  uint8_t* wbase = smem + warp * S::WARP_BYTES;
  uint8_t* qslot = wbase + NST * S::STAGE;  // two q-row slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSimtWarpsPerCta * S::WARP_BYTES) + warp * (NST + 2);
  uint64_t* qbars = bars + NST;
  if (lane == 0) {
    for (int s = 0; s < NST + 2; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int grp = lane / LPG, li = lane % LPG;
  const int seg_begin = a.warp_segs[gw], seg_end = a.warp_segs[gw + 1];
  const int ld_begin = a.warp_loads[gw], ld_end = a.warp_loads[gw + 1];
  const bool drop_first = a.fault_drop && gw == 0;

  // ---- load side: lane 0 issues; lanes hold a sliding window of 32 tile ids
  int ld = ld_begin;
  int win_base = ld_begin;
  int win_cur = ld_begin + lane < ld_end ? a.tiles[ld_begin + lane] : 0;
  int win_nxt = ld_begin + 32 + lane < ld_end ? a.tiles[ld_begin + 32 + lane] : 0;
  uint32_t inflight = 0;  // bit s: a copy into stage s (or q slot s - NST) is outstanding
  uint32_t parity = 0;    // bit s: parity of the next phase to wait for on barrier s

  auto issue = [&](int stage) {
    if (ld >= ld_end) return;
    if (ld - win_base >= 32) {  // slide the window (warp-uniform)
      win_base += 32;
      win_cur = win_nxt;
      win_nxt = win_base + 32 + lane < ld_end ? a.tiles[win_base + 32 + lane] : 0;
    }
    const int tile = __shfl_sync(0xffffffffu, win_cur, ld - win_base);
    const bool drop = drop_first && ld == ld_begin;
    if (lane == 0 && !drop) {
      uint8_t* st = wbase + stage * S::STAGE;
      const uint32_t bar = smem_u32(&bars[stage]);
      mbar_arrive_expect_tx(bar, 2 * S::TILE);
      const size_t off = (size_t)tile * (16 * D);
      bulk_g2s(smem_u32(st), a.k_pool + off, S::TILE, bar);
      bulk_g2s(smem_u32(st + S::TILE), a.v_pool + off, S::TILE, bar);
    }
    if (!drop) inflight |= 1u << stage;
    ++ld;
  };
  // q rows (b, g*G .. g*G+G-1) are contiguous: q + (b*Hq + g*G)*D
  auto issue_q = [&](int slot, const SegInfo& si) {
    if (lane == 0) {
      const uint32_t bar = smem_u32(&qbars[slot]);
      mbar_arrive_expect_tx(bar, S::QT);
      bulk_g2s(smem_u32(qslot + slot * S::QT), a.q + ((size_t)si.query * a.Hq + si.kv_head * G) * D, S::QT, bar);
    }
    inflight |= 1u << (NST + slot);
  };

  SegInfo cur = load_seg(a.segs, seg_begin, seg_end);
  SegInfo nx = load_seg(a.segs, seg_begin + 1, seg_end);
  SegInfo nxx = load_seg(a.segs, seg_begin + 2, seg_end);
  if (seg_begin < seg_end) issue_q(0, cur);
  for (int s = 0; s < NST; ++s) issue(s);

  int stage = 0;
  bool failed = false;
  for (int si = seg_begin; si < seg_end; ++si) {
    const int k = si - seg_begin;
    const int qs = k & 1;
    if (!mbar_wait_bounded(smem_u32(&qbars[qs]), (parity >> (NST + qs)) & 1u, a.timeout_ns)) {
      if (lane == 0) record_status(a.status, PA_ERR_TIMEOUT, gw, si);
      failed = true;
      break;
    }
    inflight &= ~(1u << (NST + qs));
    parity ^= 1u << (NST + qs);
    float2 qf[G][CPL][4];
#pragma unroll
    for (int r = 0; r < G; ++r)
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(qslot + qs * S::QT + r * D * 2 + (li + LPG * j) * 16);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = bf16x2_to_f2(ws[e]);
          qf[r][j][e] = make_float2(f.x * a.qscale, f.y * a.qscale);
        }
      }
    __syncwarp();
    if (si + 1 < seg_end) issue_q(qs ^ 1, nx);

    const int npages = (cur.n_tokens + 15) >> 4;
    float2 o[G][CPL][4];
    float m[G], l[G];
#pragma unroll
    for (int r = 0; r < G; ++r) {
      m[r] = -INFINITY;
      l[r] = 0.f;
#pragma unroll
      for (int j = 0; j < CPL; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[r][j][e] = make_float2(0.f, 0.f);
    }
    for (int pg = 0; pg < npages; ++pg) {
      if (!mbar_wait_bounded(smem_u32(&bars[stage]), (parity >> stage) & 1u, a.timeout_ns)) {
        if (lane == 0) record_status(a.status, PA_ERR_TIMEOUT, gw, si);
        failed = true;
        break;
      }
      inflight &= ~(1u << stage);
      parity ^= 1u << stage;
      const uint8_t* kt = wbase + stage * S::STAGE;
      const int nvalid = cur.n_tokens - pg * 16;
      if (nvalid >= 16) simt_page<D, G, false>(kt, kt + S::TILE, 16, grp, li, qf, o, m, l);
      else simt_page<D, G, true>(kt, kt + S::TILE, nvalid, grp, li, qf, o, m, l);
      __syncwarp();
      issue(stage);
      stage = stage + 1 == NST ? 0 : stage + 1;
    }
    if (failed) break;

    // combine the NG key groups (butterfly over the group bits of the lane id)
#pragma unroll
    for (int msk = LPG; msk < 32; msk <<= 1) {
#pragma unroll
      for (int r = 0; r < G; ++r) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[r], msk);
        const float lo = __shfl_xor_sync(0xffffffffu, l[r], msk);
        const float mn = fmaxf(m[r], mo);
        const float ca = m[r] == -INFINITY ? 0.f : ex2(m[r] - mn);
        const float cb = mo == -INFINITY ? 0.f : ex2(mo - mn);
        l[r] = l[r] * ca + lo * cb;
        m[r] = mn;
        const float2 ca2 = make_float2(ca, ca), cb2 = make_float2(cb, cb);
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float2 other;
            other.x = __shfl_xor_sync(0xffffffffu, o[r][j][e].x, msk);
            other.y = __shfl_xor_sync(0xffffffffu, o[r][j][e].y, msk);
            o[r][j][e] = ffma2(o[r][j][e], ca2, fmul2(other, cb2));
          }
      }
    }
    // write: group k writes rows r with r % NG == k
#pragma unroll
    for (int r = 0; r < G; ++r) {
      if (r % S::NG != grp) continue;
      const float inv = 1.f / l[r];
      float* dst = a.partial_o + ((size_t)cur.prow * G + r) * D;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        float4* d4 = reinterpret_cast<float4*>(dst + (li + LPG * j) * 8);
        d4[0] = make_float4(o[r][j][0].x * inv, o[r][j][0].y * inv, o[r][j][1].x * inv, o[r][j][1].y * inv);
        d4[1] = make_float4(o[r][j][2].x * inv, o[r][j][2].y * inv, o[r][j][3].x * inv, o[r][j][3].y * inv);
      }
      if (li == 0) a.partial_lse[(size_t)cur.prow * G + r] = (m[r] + lg2(l[r])) * kLn2;
    }
    if (a.out) arrive_and_merge<D>(a, cur.query, cur.kv_head, lane);
    cur = nx;
    nx = nxx;
    nxx = load_seg(a.segs, si + 3, seg_end);
  }
  if (failed) {
    // wait (bounded) for this warp's copies still in flight before leaving
    for (int s = 0; s < NST + 2; ++s)
      if (inflight & (1u << s)) mbar_wait_bounded(smem_u32(&bars[s]), (parity >> s) & 1u, a.timeout_ns);
  }
}

// ---------------------------------------------------------------- MMA class

constexpr int kMmaKT = 64;  // keys per stage (4 pages)
constexpr int kMmaNST = 4;  // stages
constexpr int kMmaConsumers = kMmaRowsPerCta / 16;
constexpr int kMmaThreads = (kMmaConsumers + 1) * 32;  // + producer warp

template <int D>
struct MmaShape {
  static constexpr int HALVES = D / 64;
  static constexpr int KBYTES = HALVES * kMmaKT * 128;  // one operand of one stage
  static constexpr int STAGE = 2 * KBYTES;
  static constexpr int SMEM = kMmaNST * STAGE + 2 * kMmaNST * 8 + 1024;  // + alignment slack
  static_assert(SMEM <= kSmemMax, "MMA ring does not fit");
};

// byte offset of (row, 16-byte chunk) in a 128-byte-swizzled [rows][64] bf16 block
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int D>
__device__ __forceinline__ void mma_role(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                                         uint8_t* smem_raw) {
  using S = MmaShape<D>;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kMmaNST * S::STAGE);
  uint64_t* empty = full + kMmaNST;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.G;
  const int s_begin = a.n_segs_simt + a.mma_cta_segs[blockIdx.x];
  const int s_end = a.n_segs_simt + a.mma_cta_segs[blockIdx.x + 1];

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMmaNST; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), kMmaConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kMmaConsumers) {
    // ---------------- producer: every stage of every segment of this CTA, in order
    if (lane == 0) {
      prefetch_tmap(tk);
      prefetch_tmap(tv);
      uint32_t lastpar = 0;  // bit s: parity of the last phase loaded on stage s
      uint32_t any = 0;      // bit s: stage s has been loaded at least once
      int i = 0;             // stages issued so far
      bool ok = true;
      for (int si = s_begin; si < s_end && ok; ++si) {
        const pa_seg seg = a.segs[si];
        const int page_base = a.items[seg.item].page_off + seg.page_begin;
        const int npages = (seg.n_tokens + 15) >> 4;
        for (int st = 0; st < npages; st += 4, ++i) {
          const int s = i % kMmaNST;
          if (i >= kMmaNST && !mbar_wait_bounded(smem_u32(&empty[s]), ((i / kMmaNST) - 1) & 1, a.timeout_ns)) {
            record_status(a.status, PA_ERR_TIMEOUT, blockIdx.x, -2);
            ok = false;
            break;
          }
          const int np = min(4, npages - st);
          const uint32_t fb = smem_u32(&full[s]);
          if (a.fault_drop && blockIdx.x == 0 && i == 0) continue;  // test: this stage never arrives
          mbar_arrive_expect_tx(fb, (uint32_t)np * 2 * 16 * D * 2);
          uint8_t* kst = smem + s * S::STAGE;
          uint8_t* vst = kst + S::KBYTES;
          for (int pp = 0; pp < np; ++pp) {
            const int row = (a.pages[page_base + st + pp] * a.Hkv + seg.kv_head) * 16;
#pragma unroll
            for (int h = 0; h < S::HALVES; ++h) {
              tma_load_2d(smem_u32(kst + h * kMmaKT * 128 + pp * 2048), tk, 64 * h, row, fb);
              tma_load_2d(smem_u32(vst + h * kMmaKT * 128 + pp * 2048), tv, 64 * h, row, fb);
            }
          }
          lastpar = (lastpar & ~(1u << s)) | ((uint32_t)((i / kMmaNST) & 1) << s);
          any |= 1u << s;
        }
      }
      // drain: the last load of every stage used must have landed before exit
      for (int s = 0; s < kMmaNST; ++s)
        if (any & (1u << s)) mbar_wait_bounded(smem_u32(&full[s]), (lastpar >> s) & 1u, a.timeout_ns);
    }
    return;
  }

  // ---------------- consumers: warp w owns rows 16w .. 16w+15 of each segment
  const int t4 = lane >> 2, c4 = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;
  constexpr int KS = D / 16;  // k-steps over the head dim
  int i = 0;                  // stages consumed so far
  for (int si = s_begin; si < s_end; ++si) {
    const pa_seg seg = a.segs[si];
    const pa_item item = a.items[seg.item];
    const int g = seg.kv_head;
    const int npages = (seg.n_tokens + 15) >> 4;
    const int R = item.n_queries * G;
    const bool active = warp * 16 < R;
    const int r0 = warp * 16 + t4, r1 = r0 + 8;
    uint32_t qa[KS][4];
    if (active) {
      auto qrow = [&](int r) -> const uint16_t* {
        if (r >= R) return nullptr;
        const int b = a.queries[item.query_off + r / G];
        return a.q + ((size_t)b * a.Hq + g * G + (r % G)) * D;
      };
      const uint16_t* q0 = qrow(r0);
      const uint16_t* q1 = qrow(r1);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        const int d0 = kk * 16 + 2 * c4;
        qa[kk][0] = q0 ? *reinterpret_cast<const uint32_t*>(q0 + d0) : 0u;
        qa[kk][1] = q1 ? *reinterpret_cast<const uint32_t*>(q1 + d0) : 0u;
        qa[kk][2] = q0 ? *reinterpret_cast<const uint32_t*>(q0 + d0 + 8) : 0u;
        qa[kk][3] = q1 ? *reinterpret_cast<const uint32_t*>(q1 + d0 + 8) : 0u;
      }
    }
    float oacc[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int st = 0; st < npages; st += 4, ++i) {
      const int s = i % kMmaNST;
      if (!mbar_wait_bounded(smem_u32(&full[s]), (i / kMmaNST) & 1, a.timeout_ns)) {
        if (lane == 0) record_status(a.status, PA_ERR_TIMEOUT, blockIdx.x, warp);
        return;
      }
      const int np = min(4, npages - st);
      const int kvalid = min(kMmaKT, seg.n_tokens - st * 16);
      const bool partial = kvalid < np * 16;
      if (active) {
        const uint32_t kb = smem_u32(smem + s * S::STAGE), vb = kb + S::KBYTES;
        float sacc[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
        for (int ntp = 0; ntp < 4; ++ntp) {
          if (ntp < np) {
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
              const int key = (2 * ntp + (mi >> 1)) * 8 + rr;
              const int dof = kk * 16 + 8 * (mi & 1);
              uint32_t b0, b1, b2, b3;
              ldsm_x4(kb + (dof >> 6) * (kMmaKT * 128) + swz(key, (dof & 63) >> 3), b0, b1, b2, b3);
              mma_bf16_16816(sacc[2 * ntp], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
              mma_bf16_16816(sacc[2 * ntp + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
            }
          }
        }
        // scale, mask, row max
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = n * 8 + 2 * c4 + (e & 1);
            sacc[n][e] = key < kvalid ? sacc[n][e] * a.qscale : -INFINITY;
          }
          mx0 = fmaxf(mx0, fmaxf(sacc[n][0], sacc[n][1]));
          mx1 = fmaxf(mx1, fmaxf(sacc[n][2], sacc[n][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = mn0 == -INFINITY ? 1.f : ex2(m0 - mn0);
        const float al1 = mn1 == -INFINITY ? 1.f : ex2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        const float ms0 = m0 == -INFINITY ? 0.f : m0, ms1 = m1 == -INFINITY ? 0.f : m1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          oacc[n][0] *= al0;
          oacc[n][1] *= al0;
          oacc[n][2] *= al1;
          oacc[n][3] *= al1;
        }
        uint32_t pf[8][2];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          const float p0 = ex2(sacc[n][0] - ms0), p1 = ex2(sacc[n][1] - ms0);
          const float p2 = ex2(sacc[n][2] - ms1), p3 = ex2(sacc[n][3] - ms1);
          l0 += p0 + p1;
          l1 += p2 + p3;
          pf[n][0] = pack_bf16x2(p0, p1);
          pf[n][1] = pack_bf16x2(p2, p3);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          if (kk < np) {
            const uint32_t a0 = pf[2 * kk][0], a1 = pf[2 * kk][1], a2 = pf[2 * kk + 1][0], a3 = pf[2 * kk + 1][1];
            uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
            if (partial) {
              // V rows past the last valid key may hold NaN; p = 0 there, but 0 * NaN
              // would still poison the product, so the fragments are zeroed instead
              const int k0 = kk * 16 + 2 * c4;
              mlo = (k0 < kvalid ? 0x0000FFFFu : 0u) | (k0 + 1 < kvalid ? 0xFFFF0000u : 0u);
              mhi = (k0 + 8 < kvalid ? 0x0000FFFFu : 0u) | (k0 + 9 < kvalid ? 0xFFFF0000u : 0u);
            }
#pragma unroll
            for (int ntp = 0; ntp < D / 16; ++ntp) {
              const int key = kk * 16 + 8 * (mi & 1) + rr;
              const int d = (2 * ntp + (mi >> 1)) * 8;
              uint32_t b0, b1, b2, b3;
              ldsm_x4_t(vb + (d >> 6) * (kMmaKT * 128) + swz(key, (d & 63) >> 3), b0, b1, b2, b3);
              mma_bf16_16816(oacc[2 * ntp], a0, a1, a2, a3, b0 & mlo, b1 & mhi);
              mma_bf16_16816(oacc[2 * ntp + 1], a0, a1, a2, a3, b2 & mlo, b3 & mhi);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
    if (!active) continue;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
    if (r0 < R) {
      const int prow = a.seg_prows[seg.prow + r0 / G];
      float* dst = a.partial_o + ((size_t)prow * G + (r0 % G)) * D;
#pragma unroll
      for (int n = 0; n < D / 8; ++n)
        *reinterpret_cast<float2*>(dst + n * 8 + 2 * c4) = make_float2(oacc[n][0] * inv0, oacc[n][1] * inv0);
      if (c4 == 0) a.partial_lse[(size_t)prow * G + (r0 % G)] = (m0 + lg2(l0)) * kLn2;
    }
    if (r1 < R) {
      const int prow = a.seg_prows[seg.prow + r1 / G];
      float* dst = a.partial_o + ((size_t)prow * G + (r1 % G)) * D;
#pragma unroll
      for (int n = 0; n < D / 8; ++n)
        *reinterpret_cast<float2*>(dst + n * 8 + 2 * c4) = make_float2(oacc[n][2] * inv1, oacc[n][3] * inv1);
      if (c4 == 0) a.partial_lse[(size_t)prow * G + (r1 % G)] = (m1 + lg2(l1)) * kLn2;
    }
    if (a.out) {
      // this warp's 16 rows hold whole (request, kv head) row groups (16 % G == 0)
      const int qpw = 16 / G;
      for (int j = warp * qpw; j < min((warp + 1) * qpw, item.n_queries); ++j)
        arrive_and_merge<D>(a, a.queries[item.query_off + j], g, lane);
    }
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kSimtWarpsPerCta * 32, 1) fwd_simt_kernel(const FwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  simt_role<D, G>(a, smem);
}

template <int D>
__global__ void __launch_bounds__(kMmaThreads, 1)
    fwd_mma_kernel(const FwdArgs a, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
  extern __shared__ __align__(1024) uint8_t smem[];
  mma_role<D>(a, &tk, &tv, smem);
}

struct MergeArgs {
  const int32_t* prow_off;
  const float* partial_lse;
  const float* partial_o;
  __nv_bfloat16* out;
  float* lse;
  int B, Hq, Hkv, G;
};

template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const MergeArgs a) {
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= a.B * a.Hkv) return;
  merge_pair<D>(a.prow_off, a.partial_lse, a.partial_o, a.out, a.lse, a.Hq, a.Hkv, a.G, w / a.Hkv, w % a.Hkv, lane);
}

FwdArgs make_fwd_args(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse) {
  FwdArgs a;
  a.q = d.q;
  a.k_pool = d.k_pool;
  a.v_pool = d.v_pool;
  a.items = d.items;
  a.segs = d.segs;
  a.pages = d.pages;
  a.queries = d.queries;
  a.seg_prows = d.seg_prows;
  a.warp_segs = d.warp_segs;
  a.warp_loads = d.warp_loads;
  a.tiles = d.tiles;
  a.mma_cta_segs = d.mma_cta_segs;
  a.prow_off = d.prow_off;
  a.counters = d.counters;
  a.partial_lse = d.partial_lse;
  a.partial_o = d.partial_o;
  a.status = d.status;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.G = p.G;
  a.n_simt_warps = p.hdr.simt_warps;
  a.n_segs_simt = p.hdr.num_segments_simt;
  a.n_mma_ctas = p.hdr.mma_ctas;
  a.qscale = p.scale * kLog2e;
  a.timeout_ns = (uint64_t)p.wait_timeout_us * 1000ull;
  a.fault_drop = (p.flags & PA_PLAN_FAULT_DROP_LOAD) ? 1 : 0;
  return a;
}

template <int D, int G>
int launch_simt_t(const FwdArgs& a, cudaStream_t st) {
  constexpr int smem = SimtShape<D, G>::SMEM;
  auto k = fwd_simt_kernel<D, G>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  const int grid = (a.n_simt_warps + kSimtWarpsPerCta - 1) / kSimtWarpsPerCta;
  if (grid <= 0) return 0;
  k<<<grid, kSimtWarpsPerCta * 32, smem, st>>>(a);
  return (int)cudaGetLastError();
}

template <int D>
int launch_mma_t(const pa_plan& p, const FwdArgs& a, cudaStream_t st) {
  constexpr int smem = MmaShape<D>::SMEM;
  auto k = fwd_mma_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  if (a.n_mma_ctas <= 0) return 0;
  const CUtensorMap* tk = reinterpret_cast<const CUtensorMap*>(p.tma_k);
  const CUtensorMap* tv = reinterpret_cast<const CUtensorMap*>(p.tma_v);
  k<<<a.n_mma_ctas, kMmaThreads, smem, st>>>(a, *tk, *tv);
  return (int)cudaGetLastError();
}

}  // namespace pa

using namespace pa;

int pa_launch_forward_simt(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream) {
  const FwdArgs a = make_fwd_args(p, d, out, lse);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
#define PA_FWD_CASE(DD, GG) \
  if (p.D == DD && p.G == GG) return launch_simt_t<DD, GG>(a, st);
  PA_FWD_CASE(128, 4)
  PA_FWD_CASE(128, 1)
  PA_FWD_CASE(128, 2)
  PA_FWD_CASE(128, 8)
  PA_FWD_CASE(64, 4)
  PA_FWD_CASE(64, 1)
  PA_FWD_CASE(64, 2)
  PA_FWD_CASE(64, 8)
#undef PA_FWD_CASE
  return (int)cudaErrorInvalidValue;
}

int pa_launch_forward_mma(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* side) {
  const FwdArgs a = make_fwd_args(p, d, out, lse);
  cudaStream_t st = static_cast<cudaStream_t>(side);
  return p.D == 128 ? launch_mma_t<128>(p, a, st) : launch_mma_t<64>(p, a, st);
}

int pa_launch_merge(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream) {
  MergeArgs a;
  a.prow_off = d.prow_off;
  a.partial_lse = d.partial_lse;
  a.partial_o = d.partial_o;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.G = p.G;
  const int warps = p.B * p.Hkv;
  const int grid = (warps + 7) / 8;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p.D == 128) merge_kernel<128><<<grid, 256, 0, st>>>(a);
  else merge_kernel<64><<<grid, 256, 0, st>>>(a);
  return (int)cudaGetLastError();
}

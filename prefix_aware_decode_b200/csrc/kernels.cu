// Forward and merge kernels for sm_100a.
//
// Forward (the PAT review, section 三, Forward 阶段 and Figure 3: decode attention
// is two GEMVs, q.K^T then p.V, fed by a tiling pipeline that streams KV tiles
// from global memory through on-chip memory; multi-tile kernels with a runtime
// tile selector; long KV is split).  The planner gives every work unit one of
// two tile classes, chosen by its rows (requests x G query heads), and splits
// the SMs between the classes so that both finish together; the two classes
// are two launches of one CTA per SM that run side by side (the pages'
// multi-stream execution, done here with programmatic dependent launch):
//   - MMA class: work units with two or more requests, up to 128 rows, on the
//     5th-generation tensor cores: two producer warps stream the K and the V
//     of 64-key stages with 2-D TMA copies (128-byte swizzle), one thread
//     issues the S products and another the p.V products (tcgen05.mma, S, P
//     and the accumulators in tensor memory), and 8 warps run the softmax.
//   - SIMT class: work units of one request (G <= 8 rows).  Each warp of a
//     CTA streams its own run of (page, kv head) tiles with 3-D TMA copies
//     into a private shared-memory ring and computes with warp-level
//     tensor-core products (mma.sync), the request's rows held in registers.
// Both emit, per (request, kv head, key range), the normalised partial output
// o = sum_t e^{s_t - m} v_t / l and lse = m + ln l in fp32.
//
// Merge (Merge 阶段: an online-softmax combine of each query's partial results
// across CTAs): LSE = log sum_j e^{lse_j}, out = sum_j e^{lse_j - LSE} o_j.  In
// the fused path the SIMT warp that writes the last SIMT partial row of a
// (request, kv head) merges it (arrival counter per pair), waiting for the
// tensor-core launch first when the pair also has tensor-core rows; pairs with
// tensor-core rows only are merged by a short merge launch.  The same
// warp-level routine also runs as the stand-alone merge launch.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "plan.h"
#include "ptx.cuh"

namespace pa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kSmemMax = 232448;  // opt-in shared memory per CTA on sm_100
constexpr float kRescaleLog2 = 8.f;  // a running maximum is raised only when it grows by more than this (log2 units)

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
  const int32_t* prow_off;
  int32_t* counters;
  float* partial_lse;
  float* partial_o;
  int32_t* status;
  __nv_bfloat16* out;  // non-null: fused merge
  float* lse;
  int Hq, Hkv, G, n_simt_warps, n_segs_simt, n_mma_ctas;
  int simt_wpc;  // SIMT warps per CTA of the small-row launch
  float qscale;  // softmax scale * log2(e): scores are kept in base-2 units
  uint64_t timeout_ns;
  int fault_drop;
  int debug_checks;  // PA_PLAN_DEBUG_CHECKS: page and request ids are range-checked before any load
  int tile_maps;     // the small-row class got whole-tile (3-D) maps: one copy per K or V tile
  int num_pages, B;
  int n_segs_mma;
  int32_t* mma_next;  // the counter of tensor-core work units taken (image header)
  const int32_t* mix_pairs;  // {pair, SIMT rows} of the pairs with both classes' rows
  int n_mix_pairs;
};

// ---------------------------------------------------------------- merge of one (request, kv head)

// One warp merges the partial rows [p0, p1) of (b, g) into
// out[b][g*G .. g*G+G-1][:] and lse[b][...]: lane l handles row l / (32/G) and
// a run of D*G/32 head dims.  The partial rows are taken in batches of NB
// whose loads are all issued before any is used, so a pair costs about one
// memory round trip per NB partial rows.  Partial rows are read through L2
// (they may have been written by other SMs in the same launch).
template <int D, int G, typename OutT = __nv_bfloat16>
__device__ __forceinline__ void merge_pair(const float* partial_lse, const float* partial_o, OutT* out,
                                           float* lse, int Hq, int b, int g, int p0, int p1, int lane) {
  constexpr int LPR = 32 / G;   // lanes per row
  constexpr int VPL = D / LPR;  // head dims per lane
  constexpr int NB = VPL >= 32 ? 2 : 4;
  const int r = lane / LPR, d0 = (lane % LPR) * VPL;
  float m = -INFINITY, z = 0.f, acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  for (int pb = p0; pb < p1; pb += NB) {
    float lp[NB], o[NB][VPL];
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      const int p = pb + k < p1 ? pb + k : p1 - 1;  // past the end: reload the last row, weight 0
      lp[k] = __ldcg(partial_lse + (size_t)p * G + r);
      const float* src = partial_o + ((size_t)p * G + r) * D + d0;
      if constexpr (VPL % 4 == 0) {
#pragma unroll
        for (int i = 0; i < VPL / 4; ++i) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(src) + i);
          o[k][4 * i] = v.x;
          o[k][4 * i + 1] = v.y;
          o[k][4 * i + 2] = v.z;
          o[k][4 * i + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < VPL / 2; ++i) {
          const float2 v = __ldcg(reinterpret_cast<const float2*>(src) + i);
          o[k][2 * i] = v.x;
          o[k][2 * i + 1] = v.y;
        }
      }
    }
    float mn = m;
#pragma unroll
    for (int k = 0; k < NB; ++k)
      if (pb + k < p1) mn = fmaxf(mn, lp[k]);
    const float sa = m == -INFINITY ? 0.f : expf(m - mn);
    z *= sa;
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] *= sa;
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      const float w = pb + k < p1 ? expf(lp[k] - mn) : 0.f;
      z += w;
#pragma unroll
      for (int i = 0; i < VPL; ++i) acc[i] = fmaf(o[k][i], w, acc[i]);
    }
    m = mn;
  }
  const float inv = 1.f / z;
  OutT* dst = out + ((size_t)b * Hq + g * G + r) * D + d0;
  if constexpr (std::is_same<OutT, float>::value) {
#pragma unroll
    for (int i = 0; i < VPL; i += 2) *reinterpret_cast<float2*>(dst + i) = make_float2(acc[i] * inv, acc[i + 1] * inv);
  } else {
#pragma unroll
    for (int i = 0; i < VPL; i += 2)
      *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
  }
  if (lse && lane % LPR == 0) lse[(size_t)b * Hq + g * G + r] = m + logf(z);
}

// Called by a whole SIMT warp after it wrote a partial row of pair bg = b*Hkv+g
// (or, for a pair that also has tensor-core rows, once that launch has
// finished): counts the arrival; true if this was the last of the pair's n.
__device__ __forceinline__ bool simt_arrive(const FwdArgs& a, int bg, int n_simt, int lane) {
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atomicAdd(&a.counters[bg], 1) == n_simt - 1;
  if (!__shfl_sync(0xffffffffu, last, 0)) return false;
  __threadfence();
  return true;
}

template <int D, int G>
__device__ __forceinline__ void merge_and_reset(const FwdArgs& a, int bg, int lane) {
  merge_pair<D, G>(a.partial_lse, a.partial_o, a.out, a.lse, a.Hq, bg / a.Hkv, bg % a.Hkv, a.prow_off[bg],
                   a.prow_off[bg + 1], lane);
  if (lane == 0) a.counters[bg] = 0;  // ready for the next launch
}

// ---------------------------------------------------------------- small-row class (one request, G rows)
//
// Each of the CTA's warps (8, or 6 for long runs: the plan's choice) streams
// its own run of (page, kv head) tiles through a private ring in shared
// memory: per tile, K and V arrive as D/64 boxes of 16
// keys x 64 dims each (2-D TMA, 128-byte swizzle, completed on the stage's
// mbarrier).  The G query rows of the request stay in registers as the B
// operand of warp-level tensor-core products (mma.sync m16n8k16, bf16 in,
// fp32 accumulate), with the keys as the M dimension so one request's rows
// never leave the warp:
//   S^T (16 keys x 8 rows) = K (16 x D) . Q^T            D/16 products
//   online softmax per row over the keys (3 shuffles per row pair)
//   P^T = P_hi + P_lo, each a bf16 B operand (transposed in registers)
//   O^T (D x 8 rows) += V^T (D x 16 keys) . P^T          2 D/16 products
// Rows past G are zero q rows whose results are dropped.  Per tile a warp
// issues about a hundred instructions (against about 800 for the same work on
// the CUDA cores with packed fp32 FMAs), so the class is bound by the bytes in
// flight, not by issue.

template <int D, int G>
struct SimtShape {
  static constexpr int TILE = 16 * D * 2;   // K (or V) of one (page, kv head) tile: D/64 swizzled 2 KB boxes
  static constexpr int QT = G * D * 2;      // the G query rows
  static constexpr int STAGE = 2 * TILE;
  static constexpr int W = kSimtWarpsPerCta;
  static constexpr int KT = D / 16;         // k steps of K.Q^T, d tiles of V^T.P^T
  static constexpr int FIXED = W * 2 * QT + 1024 + W * 8 * 8;  // q slots, alignment slack, barriers
  static constexpr int NST_FIT = (kSmemMax - FIXED) / (W * STAGE);
  // ring stages: two D = 128 tiles or three D = 64 tiles per warp (16 and 12 KB
  // in flight); deeper rings (3 and 6) were measured slower: config 3 232 ->
  // 211 us, config 4 275 -> 272 us, config 2 47.4 -> 45.6 us at 8 warps
  static constexpr int NST = NST_FIT < (D == 128 ? 2 : 3) ? NST_FIT : (D == 128 ? 2 : 3);
  static constexpr int RING = NST * STAGE;  // one warp's ring (a multiple of 1 KB: swizzle atoms stay aligned)
  static constexpr int OFF_Q = W * RING;
  static constexpr int OFF_BAR = OFF_Q + W * 2 * QT;
  static constexpr int SMEM = OFF_BAR + W * (NST + 2) * 8 + 1024;
  static_assert(NST >= 2 && SMEM <= kSmemMax, "ring does not fit in shared memory");
  static_assert(RING % 1024 == 0 && TILE % 2048 == 0, "swizzle atoms must stay 1 KB aligned");
  static_assert(G <= 8, "at most 8 rows per request");
};

struct SegInfo {
  int n_tokens, prow, query, kv_head;
  int mode, n_simt;  // how the fused path combines the partial row (pa_seg.sole)
};

__device__ __forceinline__ SegInfo load_seg(const pa_seg* segs, int i, int end) {
  SegInfo r{0, 0, 0, 0, 0, 0};
  if (i < end) {
    const int4 x = *reinterpret_cast<const int4*>(segs + i);        // item, kv_head, page_begin, n_tokens
    const int4 y = *reinterpret_cast<const int4*>(&segs[i].prow);  // prow, query, sole, pad
    r.n_tokens = x.w;
    r.kv_head = x.y;
    r.prow = y.x;
    r.query = y.y;
    r.mode = y.z & 3;
    r.n_simt = y.z >> 2;
  }
  return r;
}

// Shared-memory address of 16-byte chunk `ch` (8 dims) of key row `r` of a
// tile stored as D/64 boxes of 16 rows x 128 bytes with the 128-byte swizzle
// (chunk c of row r sits at chunk c ^ (r % 8) of the row).
__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int ch) {
  return base + (ch >> 3) * 2048 + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
}

// One tile of 16 keys for one warp: scores, online softmax (base-2 units,
// maximum raised lazily), p.V.  Thread (g, t) = (lane / 4, lane % 4) holds the
// scores of keys g and g + 8 for rows 2t and 2t + 1, and the accumulator
// O^T[d][2t..2t+1] for d = 16 i + g and 16 i + g + 8.  PARTIAL: the tile holds
// fewer than 16 valid keys (the rest may hold NaN).
template <int D, int G, bool PARTIAL>
__device__ __forceinline__ void tile_step(uint32_t kt, uint32_t vt, int nvalid, int lane, float c,
                                          const uint32_t (&qb)[D / 16][2], float (&o)[D / 16][4], float (&ms)[2],
                                          float (&l)[2]) {
  constexpr int KT = D / 16;
  const int g = lane >> 2, t = lane & 3;
  // S^T = K . Q^T, two accumulation chains; every K fragment is loaded before
  // the first product, and every V fragment (matrices (keys 0-7 | 8-15) x
  // (dims 16i..16i+7 | 16i+8..16i+15)) right after the last one, so the V loads
  // overlap the softmax
  uint32_t kf[KT][4], vf[KT][4];
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) ldsm_x4(swz(kt, lane & 15, 2 * kk + (lane >> 4)), kf[kk]);
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) {
    if (kk & 1) mma_bf16_16816(sb, kf[kk], qb[kk][0], qb[kk][1]);
    else mma_bf16_16816(sa, kf[kk], qb[kk][0], qb[kk][1]);
  }
  {
    const int vrow = (lane & 7) + ((lane >> 4) << 3), vch = (lane >> 3) & 1;
#pragma unroll
    for (int i = 0; i < KT; ++i) ldsm_x4_trans(swz(vt, vrow, 2 * i + vch), vf[i]);
  }
  float s[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) s[i] = sa[i] + sb[i];
  // s[0]: key g row 2t, s[1]: key g row 2t+1, s[2]: key g+8 row 2t, s[3]: key g+8 row 2t+1
  if (PARTIAL) {
    if (g >= nvalid) s[0] = s[1] = -INFINITY;
    if (g + 8 >= nvalid) s[2] = s[3] = -INFINITY;
  }
  if (2 * t >= G) s[0] = s[2] = -INFINITY;
  if (2 * t + 1 >= G) s[1] = s[3] = -INFINITY;
  float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  const float mn0 = mx0 * c, mn1 = mx1 * c;
  const bool up0 = mn0 > ms[0] + kRescaleLog2, up1 = mn1 > ms[1] + kRescaleLog2;
  if (up0 || up1) {
    // the running maximum moves up only when it grows by more than 2^8: p stays
    // below 256, and the accumulator is rescaled rarely
    const float a0 = up0 ? ex2(ms[0] - mn0) : 1.f, a1 = up1 ? ex2(ms[1] - mn1) : 1.f;
#pragma unroll
    for (int i = 0; i < KT; ++i) {
      o[i][0] *= a0;
      o[i][1] *= a1;
      o[i][2] *= a0;
      o[i][3] *= a1;
    }
    l[0] *= a0;
    l[1] *= a1;
    if (up0) ms[0] = mn0;
    if (up1) ms[1] = mn1;
  }
  const float m0 = ms[0] == -INFINITY ? 0.f : ms[0], m1 = ms[1] == -INFINITY ? 0.f : ms[1];
  const float p0 = ex2(fmaf(s[0], c, -m0)), p1 = ex2(fmaf(s[1], c, -m1));
  const float p2 = ex2(fmaf(s[2], c, -m0)), p3 = ex2(fmaf(s[3], c, -m1));
  l[0] += p0 + p2;
  l[1] += p1 + p3;
  // P = P_hi + P_lo: P_hi the truncated bf16 of p (so p - P_hi is exact),
  // P_lo that remainder rounded to the nearest bf16; then each 8x8 block
  // (keys x rows) is transposed into the B-operand layout (keys 2t, 2t+1 of row g)
  const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
  const uint32_t u2 = __float_as_uint(p2), u3 = __float_as_uint(p3);
  const uint32_t h01 = __byte_perm(u0, u1, 0x7632), h23 = __byte_perm(u2, u3, 0x7632);
  const uint32_t l01 = pack_bf16x2(p0 - __uint_as_float(u0 & 0xFFFF0000u), p1 - __uint_as_float(u1 & 0xFFFF0000u));
  const uint32_t l23 = pack_bf16x2(p2 - __uint_as_float(u2 & 0xFFFF0000u), p3 - __uint_as_float(u3 & 0xFFFF0000u));
  const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
  const uint32_t bl0 = movmatrix_trans(l01), bl1 = movmatrix_trans(l23);
  // V rows past the last valid key may hold NaN: p = 0 there, but 0 * NaN would
  // still poison the product, so those keys' V values are zeroed
  uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
  if (PARTIAL) {
    mlo = (2 * t < nvalid ? 0x0000ffffu : 0u) | (2 * t + 1 < nvalid ? 0xffff0000u : 0u);
    mhi = (2 * t + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * t + 9 < nvalid ? 0xffff0000u : 0u);
  }
  // O^T += V^T . P^T
#pragma unroll
  for (int i = 0; i < KT; ++i) {
    uint32_t (&af)[4] = vf[i];
    if (PARTIAL) {
      af[0] &= mlo;
      af[1] &= mlo;
      af[2] &= mhi;
      af[3] &= mhi;
    }
    mma_bf16_16816(o[i], af, bh0, bh1);
    mma_bf16_16816(o[i], af, bl0, bl1);
  }
}

template <int D, int G>
__device__ __forceinline__ void simt_role(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                                          uint8_t* smem_raw) {
  using S = SimtShape<D, G>;
  constexpr int NST = S::NST, KT = S::KT;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= kSimtWarpsPerCta) return;
  const int gw = blockIdx.x * a.simt_wpc + warp;
  if (gw >= a.n_simt_warps) return;  // no block-wide barrier in this role
  const uint32_t ring = smem_u32(smem + warp * S::RING);
  uint8_t* qslot = smem + S::OFF_Q + warp * 2 * S::QT;  // two q-row slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR) + warp * (NST + 2);
  uint64_t* qbars = bars + NST;
  if (lane == 0) {
    for (int s = 0; s < NST + 2; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
    prefetch_tmap(tk);
    prefetch_tmap(tv);
  }
  __syncwarp();

  const int g8 = lane >> 2, t4 = lane & 3;
  const int seg_begin = a.warp_segs[gw], seg_end = a.warp_segs[gw + 1];
  const bool drop_first = a.fault_drop && gw == 0;

  // ---- load side (lane 0 issues).  The warp's loads are the pages of its
  // segments, in order.  Lanes hold the descriptors of a group of up to 32
  // segments (first page index, page count, kv head) and their exclusive
  // prefix sums; a window of 32 tile ids (page * Hkv + kv head) is filled by a
  // per-lane binary search over the group plus one page-id load, and the next
  // window is fetched one window ahead.
  int sg_base = seg_begin;  // first segment of the current group
  int sg_pstart = 0, sg_npg = 0, sg_g = 0, sg_off = 0, sg_tot = 0, sg_n = 0;
  auto load_group = [&]() {
    sg_n = min(32, seg_end - sg_base);
    sg_pstart = 0;
    sg_npg = 0;
    sg_g = 0;
    if (lane < sg_n) {
      const pa_seg& sd = a.segs[sg_base + lane];
      sg_pstart = sd.page_start;
      sg_npg = (sd.n_tokens + 15) >> 4;
      sg_g = sd.kv_head;
    }
    int incl = sg_npg;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    sg_off = incl - sg_npg;
    sg_tot = __shfl_sync(0xffffffffu, incl, 31);
  };
  auto tile_for = [&](int x) -> int {  // x: page index within the group
    int lo = 0;
#pragma unroll
    for (int step = 16; step > 0; step >>= 1) {
      const int cand = lo + step;
      const int oc = __shfl_sync(0xffffffffu, sg_off, cand & 31);
      if (cand < sg_n && oc <= x) lo = cand;
    }
    const int ps = __shfl_sync(0xffffffffu, sg_pstart, lo);
    const int o0 = __shfl_sync(0xffffffffu, sg_off, lo);
    const int g = __shfl_sync(0xffffffffu, sg_g, lo);
    if (x >= sg_tot) return 0;
    int page = a.pages[ps + (x - o0)];
    if (a.debug_checks && (uint32_t)page >= (uint32_t)a.num_pages) {
      record_status(a.status, PA_ERR_DEVICE, gw, page);
      page = 0;
    }
    return page * a.Hkv + g;
  };
  int ld_x = 0, wbase = 0;  // next load (within the group), current window base
  bool ld_more = seg_begin < seg_end;
  int win_cur = 0, win_nxt = 0;
  if (ld_more) {
    load_group();
    win_cur = tile_for(lane);
    win_nxt = tile_for(32 + lane);
  }
  uint32_t inflight = 0;  // bit s: a copy into stage s (or q slot s - NST) is outstanding
  uint32_t parity = 0;    // bit s: parity of the next phase to wait for on barrier s
  bool first_load = true;

  auto issue = [&](int stage) {
    if (!ld_more) return;
    if (ld_x >= sg_tot) {  // next group of segments (warp-uniform; only warps with > 32 segments)
      sg_base += 32;
      if (sg_base >= seg_end) {
        ld_more = false;
        return;
      }
      load_group();
      ld_x = 0;
      wbase = 0;
      win_cur = tile_for(lane);
      win_nxt = tile_for(32 + lane);
    }
    if (ld_x - wbase >= 32) {  // slide the window (warp-uniform)
      wbase += 32;
      win_cur = win_nxt;
      win_nxt = tile_for(wbase + 32 + lane);
    }
    const int tile = __shfl_sync(0xffffffffu, win_cur, ld_x - wbase);
    const bool drop = drop_first && first_load;
    first_load = false;
    if (lane == 0 && !drop) {
      const uint32_t st = ring + stage * S::STAGE;
      const uint32_t bar = smem_u32(&bars[stage]);
      mbar_arrive_expect_tx(bar, 2 * S::TILE);
      if (D == 128 && a.tile_maps) {
        tma_load_3d(st, tk, 0, tile * 16, 0, bar);
        tma_load_3d(st + S::TILE, tv, 0, tile * 16, 0, bar);
      } else {
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_2d(st + h * 2048, tk, 64 * h, tile * 16, bar);
          tma_load_2d(st + S::TILE + h * 2048, tv, 64 * h, tile * 16, bar);
        }
      }
    }
    if (!drop) inflight |= 1u << stage;
    ++ld_x;
    if (ld_x >= sg_tot && sg_base + 32 >= seg_end) ld_more = false;
  };
  // q rows (b, g*G .. g*G+G-1) are contiguous: q + (b*Hq + g*G)*D
  auto issue_q = [&](int slot, const SegInfo& si) {
    if (lane == 0) {
      int b = si.query;
      if (a.debug_checks && (uint32_t)b >= (uint32_t)a.B) {
        record_status(a.status, PA_ERR_DEVICE, gw, -1 - b);
        b = 0;
      }
      const uint32_t bar = smem_u32(&qbars[slot]);
      mbar_arrive_expect_tx(bar, S::QT);
      bulk_g2s(smem_u32(qslot + slot * S::QT), a.q + ((size_t)b * a.Hq + si.kv_head * G) * D, S::QT, bar);
    }
    inflight |= 1u << (NST + slot);
  };

  SegInfo cur = load_seg(a.segs, seg_begin, seg_end);
  SegInfo nx = load_seg(a.segs, seg_begin + 1, seg_end);
  SegInfo nxx = load_seg(a.segs, seg_begin + 2, seg_end);
  if (seg_begin < seg_end) issue_q(0, cur);
  for (int s = 0; s < NST; ++s) issue(s);

  const float c = a.qscale;  // scale * log2(e), applied to the fp32 scores
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
    // B operand of K.Q^T: b0 = q[row g][16 kk + 2t, +1], b1 = q[row g][16 kk + 2t + 8, +9]
    uint32_t qb[KT][2];
    {
      const uint8_t* qrow = qslot + qs * S::QT + (g8 < G ? g8 : 0) * D * 2;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(qrow + (16 * kk + 2 * t4) * 2);
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(qrow + (16 * kk + 2 * t4 + 8) * 2);
        qb[kk][0] = g8 < G ? w0 : 0u;
        qb[kk][1] = g8 < G ? w1 : 0u;
      }
    }
    __syncwarp();
    if (si + 1 < seg_end) issue_q(qs ^ 1, nx);

    const int npages = (cur.n_tokens + 15) >> 4;
    float o[KT][4];
#pragma unroll
    for (int i = 0; i < KT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float ms[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    for (int pg = 0; pg < npages; ++pg) {
      if (!mbar_wait_bounded(smem_u32(&bars[stage]), (parity >> stage) & 1u, a.timeout_ns)) {
        if (lane == 0) record_status(a.status, PA_ERR_TIMEOUT, gw, si);
        failed = true;
        break;
      }
      inflight &= ~(1u << stage);
      parity ^= 1u << stage;
      const uint32_t kt = ring + stage * S::STAGE;
      const int nvalid = cur.n_tokens - pg * 16;
      if (nvalid >= 16) tile_step<D, G, false>(kt, kt + S::TILE, 16, lane, c, qb, o, ms, l);
      else tile_step<D, G, true>(kt, kt + S::TILE, nvalid, lane, c, qb, o, ms, l);
      __syncwarp();
      issue(stage);
      stage = stage + 1 == NST ? 0 : stage + 1;
    }
    if (failed) break;

    // the sum over the keys of each row: the 8 lanes that share t
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l[0] += __shfl_xor_sync(0xffffffffu, l[0], off);
      l[1] += __shfl_xor_sync(0xffffffffu, l[1], off);
    }
    // write: thread (g, t) holds dims 16 i + g and 16 i + g + 8 of rows 2t, 2t+1;
    // a (request, kv head) with a single partial row goes straight to the
    // output when the merge is fused
    const bool direct = a.out && cur.mode == 1;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int r = 2 * t4 + j;
      if (r >= G) continue;
      const float inv = 1.f / l[j];
      const float lse_r = (ms[j] + lg2(l[j])) * kLn2;
      if (direct) {
        __nv_bfloat16* dst = a.out + ((size_t)cur.query * a.Hq + cur.kv_head * G + r) * D + g8;
#pragma unroll
        for (int i = 0; i < KT; ++i) {
          dst[16 * i] = __float2bfloat16_rn(o[i][j] * inv);
          dst[16 * i + 8] = __float2bfloat16_rn(o[i][2 + j] * inv);
        }
        if (g8 == 0 && a.lse) a.lse[(size_t)cur.query * a.Hq + cur.kv_head * G + r] = lse_r;
      } else {
        float* dst = a.partial_o + ((size_t)cur.prow * G + r) * D + g8;
#pragma unroll
        for (int i = 0; i < KT; ++i) {
          dst[16 * i] = o[i][j] * inv;
          dst[16 * i + 8] = o[i][2 + j] * inv;
        }
        if (g8 == 0) a.partial_lse[(size_t)cur.prow * G + r] = lse_r;
      }
    }
    if (a.out && (cur.mode == 0 || cur.mode == 2)) {
      // a mixed pair (mode 2) counts one more arrival, made once the
      // tensor-core launch has finished (below): if that one came first, this
      // warp's is the last and the tensor-core rows are there
      const int bg = cur.query * a.Hkv + cur.kv_head;
      if (simt_arrive(a, bg, cur.n_simt + (cur.mode == 2 ? 1 : 0), lane)) merge_and_reset<D, G>(a, bg, lane);
    }
    cur = nx;
    nx = nxx;
    nxx = load_seg(a.segs, si + 3, seg_end);
  }
  // after its own work, warp gw makes the tensor-core-side arrival of the
  // mixed pairs in entries gw, gw + W, ... (W SIMT warps; at most a few per
  // warp); whichever arrival is a pair's last merges it
  if (a.out && a.n_mix_pairs > 0 && !failed) {
    griddep_wait();
    for (int k = gw; k < a.n_mix_pairs; k += a.n_simt_warps) {
      const int bg = a.mix_pairs[2 * k], n_simt = a.mix_pairs[2 * k + 1];
      if (bg < 0) continue;  // an entry no pair takes
      if (simt_arrive(a, bg, n_simt + 1, lane)) merge_and_reset<D, G>(a, bg, lane);
    }
  }
  if (failed) {
    // wait (bounded) for this warp's copies still in flight before leaving
    for (int s = 0; s < NST + 2; ++s)
      if (inflight & (1u << s)) mbar_wait_bounded(smem_u32(&bars[s]), (parity >> s) & 1u, a.timeout_ns);
  }
}

// ---------------------------------------------------------------- MMA class (tcgen05 + TMEM)
//
// Its own launch of one CTA per SM, each running a list of segments (item of
// <= 128 rows, kv head g, key range).  Warp 0: TMA producer of 64-key K/V
// stages.  Warp 1: TMEM owner and single-thread tcgen05.mma issuer.  Warps
// 2-9: softmax: warps 2-5 take keys 0-31 of every stage, warps 6-9 keys 32-63,
// each half with its own running maximum, sum and accumulator, so the halves
// never wait on each other inside a segment; the two partial results are
// combined once per segment.  Tiles of more than 64 rows are M = 128 products
// (two threads per row); tiles of at most 64 rows are M = 64 products, whose
// rows the TMEM layout spreads over all four lane quarters (four threads per
// row, 16 keys each).  Per 64-key stage i (S/P buffer i % 3 in TMEM):
//   S(i) = Q K^T                  -> TMEM, 64 columns
//   p = exp2(s - m)               -> P = P_hi + P_lo, two bf16 matrices written
//                                    over S(i) in TMEM (P_hi truncated, P_lo =
//                                    p - P_hi rounded to nearest: P keeps about
//                                    16 bits of p)
//   O_h += P_hi,h V_h + P_lo,h V_h  (A operand read from TMEM)
// S(i+1) is issued before p.V(i), so the tensor core overlaps the softmax; a
// buffer is reused for S(i+3) only after p.V(i) has completed.  A half's
// running maximum is only raised (and O_h rescaled in TMEM) when it grows by
// more than 2^8; numerator and denominator use the same maximum, so the result
// is unchanged.

constexpr int kMmaKT = 64;           // keys per stage (4 pages)
constexpr int kMmaWarps = 12;        // K producer, S issuer, 8 softmax warps, p.V issuer, V producer
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kSmaxThreads = 256;    // softmax threads (two per tile row)
constexpr int kSBufs = 3;            // S/P buffers in TMEM
constexpr int kSegQ = 8;             // entries of a CTA's queue of work units taken from the shared counter
constexpr int kSegQConsumers = 11;   // V producer, S issuer, p.V issuer, 8 softmax warps
constexpr uint32_t kTmemCols = 512;  // the whole tensor memory of the SM (one CTA per SM)
constexpr float kRescaleThreshold = kRescaleLog2;

// QR: rows of a Q buffer, 128, or 64 when no tile of the launch has more
// (the smaller Q buffers leave room for a deeper K/V ring at D = 128)
template <int D, int QR>
struct MmaShape {
  static constexpr int HALVES = D / 64;
  static constexpr int KBLK = kMmaKT * 128;        // one 64-key x 64-dim swizzled block (8 KB)
  static constexpr int KSTAGE = HALVES * KBLK;     // K (or V) of one stage
  static constexpr int STAGE = 2 * KSTAGE;         // K and V of one stage
  static constexpr int QBLK = QR * 128;            // QR rows x 64 dims
  static constexpr int QBUF = HALVES * QBLK;       // the Q rows of one segment
  static constexpr int FIXED = 2 * QBUF + 1024 + 1024;  // two Q buffers, barriers and queue, alignment slack
  static constexpr int NST_FIT = (kSmemMax - FIXED) / STAGE;
  static constexpr int NST = NST_FIT < 8 ? NST_FIT : 8;  // slots of the K ring and of the V ring
  static constexpr int OFF_K = 0, OFF_V = NST * KSTAGE;
  static constexpr int OFF_Q = NST * STAGE;
  static constexpr int OFF_BAR = OFF_Q + 2 * QBUF;
  static constexpr int SMEM = OFF_BAR + 1024 + 1024;
  // barriers: K full / empty and V full / empty per ring slot; S full, P full,
  // p.V done per buffer; Q loaded per Q buffer; O read out; all MMAs retired;
  // the two halves of each lane quarter have exchanged (m, l)
  static constexpr int B_FULL = 0, B_EMPTY = NST, B_VFULL = 2 * NST, B_VEMPTY = 3 * NST,
                       B_SFULL = 4 * NST, B_PFULL = B_SFULL + kSBufs,
                       B_PV = B_PFULL + kSBufs, B_QFULL = B_PV + kSBufs, B_OFREE = B_QFULL + 2, B_DONE = B_OFREE + 1,
                       B_XCH = B_DONE + 1, B_QF = B_XCH + 4, B_QE = B_QF + kSegQ, NBARS = B_QE + kSegQ;
  // tensor memory columns: S/P buffers, the two half accumulators, (m, l) exchange
  static constexpr uint32_t T_S = 0, T_O = kSBufs * kMmaKT, T_X = T_O + 2 * D;
  static_assert(NST >= 3 && SMEM <= kSmemMax, "MMA ring does not fit");
  static_assert(NBARS * 8 + 8 + kSegQ * 4 <= 1024, "barrier area");
  static_assert(T_X + 4 <= kTmemCols, "tensor memory plan does not fit");
};

// All lanes wait; the warp fails together if any lane timed out.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

template <int D, int G, int QR>
__device__ __forceinline__ void mma_role(const FwdArgs& a, const CUtensorMap* tk, const CUtensorMap* tv,
                                         uint8_t* smem_raw) {
  using S = MmaShape<D, QR>;
  constexpr int NST = S::NST;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::NBARS);
  volatile int32_t* segq = reinterpret_cast<int32_t*>(bars + S::NBARS + 1);  // work units taken, in order
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t q_base = smem_u32(smem + S::OFF_Q);
  // The work units (segments) are taken one at a time from the counter in the
  // image: the K producer takes the next one as soon as it has issued the
  // loads of the current one and puts it into this CTA's queue (kSegQ
  // entries, full / empty barriers); the other roles read the queue in order.
  // -1 ends the CTA's work.  Queue entry n is slot n % kSegQ, phase n / kSegQ.
  // Returns the global segment index, -1 at the end, -2 if a wait gave up.
  auto seg_take = [&](int& n, bool arrive) -> int {
    const int j = n % kSegQ;
    if (!mbar_wait_bounded(bar(S::B_QF + j), (n / kSegQ) & 1, a.timeout_ns)) return -2;
    const int v = segq[j];
    if (arrive) mbar_arrive(bar(S::B_QE + j));
    ++n;
    return v < 0 ? -1 : a.n_segs_simt + v;
  };
  // The entry after n, if the K producer has already put it there (no wait).
  auto seg_peek = [&](int n, int& si) -> bool {
    const int j = n % kSegQ;
    if (!mbar_test_wait(bar(S::B_QF + j), (n / kSegQ) & 1)) return false;
    const int v = segq[j];
    si = v < 0 ? -1 : a.n_segs_simt + v;
    return true;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar(S::B_FULL + s), 1);
      mbar_init(bar(S::B_EMPTY + s), 1);
      mbar_init(bar(S::B_VFULL + s), 1);
      mbar_init(bar(S::B_VEMPTY + s), 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(bar(S::B_SFULL + b), 1);
      mbar_init(bar(S::B_PFULL + b), kSmaxThreads);
      mbar_init(bar(S::B_PV + b), 1);
    }
    mbar_init(bar(S::B_QFULL), kSmaxThreads);
    mbar_init(bar(S::B_QFULL + 1), kSmaxThreads);
    mbar_init(bar(S::B_OFREE), kSmaxThreads);
    mbar_init(bar(S::B_DONE), 2);
    for (int q = 0; q < 4; ++q) mbar_init(bar(S::B_XCH + q), 64);
    for (int q = 0; q < kSegQ; ++q) {
      mbar_init(bar(S::B_QF + q), 1);
      mbar_init(bar(S::B_QE + q), kSegQConsumers);
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp == kMmaWarps - 1) {
    // ---------------- TMA producers: warp 0 streams the K stages, the last warp
    // the V stages, of every segment of this CTA in order, each into its own
    // ring.  A K slot is free again once S of its stage is done, a V slot once
    // p.V is; so K runs ahead of V and neither ring holds a tile longer than
    // it is needed.  The warp holds the segment's page ids in a sliding window
    // of 32 lanes (plus the next window, prefetched), so no issue waits on a load.
    const bool is_v = warp != 0;
    const CUtensorMap* tm = is_v ? tv : tk;
    const int b_full = is_v ? S::B_VFULL : S::B_FULL, b_empty = is_v ? S::B_VEMPTY : S::B_EMPTY;
    uint8_t* ring = smem + (is_v ? S::OFF_V : S::OFF_K);
    if (lane == 0) prefetch_tmap(tm);
    uint32_t lastpar = 0, any = 0;
    int i = 0, qn = 0;
    bool ok = true;
    for (;;) {
      int si;
      if (!is_v) {
        // take the next work unit from the shared counter and queue it
        const int j = qn % kSegQ;
        if (qn >= kSegQ && !warp_wait(bar(S::B_QE + j), ((qn / kSegQ) - 1) & 1, a.timeout_ns)) {
          if (lane == 0) record_status(a.status, PA_ERR_TIMEOUT, blockIdx.x, -6);
          ok = false;
          break;
        }
        // CTA c's first unit is unit c (no atomic on the way to its first
        // load); the later ones come from the counter, after the first
        // min(grid, units) units.  Every CTA that had a first unit makes one
        // take that finds the list empty, so the takes return 0 .. units - 1
        // and the last of them puts the counter back to zero.
        int v = -1;
        if (lane == 0) {
          const int n_first = min((int)gridDim.x, a.n_segs_mma);
          if (qn == 0) {
            v = (int)blockIdx.x < n_first ? (int)blockIdx.x : -1;
          } else {
            const int t = atomicAdd(a.mma_next, 1);
            if (n_first + t < a.n_segs_mma) v = n_first + t;
            if (t == a.n_segs_mma - 1) *a.mma_next = 0;  // the launch's last take
          }
          segq[j] = v;
          mbar_arrive(bar(S::B_QF + j));
        }
        v = __shfl_sync(0xffffffffu, v, 0);
        ++qn;
        if (v < 0) break;
        si = a.n_segs_simt + v;
      } else {
        int v = 0;
        if (lane == 0) v = seg_take(qn, true);
        v = __shfl_sync(0xffffffffu, v, 0);
        if (lane != 0) ++qn;
        if (v == -2) {
          if (lane == 0) record_status(a.status, PA_ERR_TIMEOUT, blockIdx.x, -7);
          ok = false;
          break;
        }
        if (v < 0) break;
        si = v;
      }
      const pa_seg seg = a.segs[si];
      const int32_t* pg = a.pages + seg.page_start;
      const int npages = (seg.n_tokens + 15) >> 4;
      auto page_at = [&](int x) -> int {
        if (x >= npages) return 0;
        int pid = pg[x];
        if (a.debug_checks && (uint32_t)pid >= (uint32_t)a.num_pages) {
          record_status(a.status, PA_ERR_DEVICE, blockIdx.x, pid);
          pid = 0;
        }
        return pid;
      };
      int wbase = 0;
      int wcur = page_at(lane);
      int wnxt = page_at(32 + lane);
      for (int st = 0; st < npages; st += 4, ++i) {
        if (st - wbase >= 32) {
          wbase += 32;
          wcur = wnxt;
          wnxt = page_at(wbase + 32 + lane);
        }
        const int s = i % NST;
        if (i >= NST && !warp_wait(bar(b_empty + s), ((i / NST) - 1) & 1, a.timeout_ns)) {
          if (lane == 0) record_status(a.status, PA_ERR_TIMEOUT, blockIdx.x, is_v ? -4 : -2);
          ok = false;
          break;
        }
        const int np = min(4, npages - st);
        int rows[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp)
          rows[pp] = (__shfl_sync(0xffffffffu, wcur, (st - wbase + pp) & 31) * a.Hkv + seg.kv_head) * 16;
        if (!is_v && a.fault_drop && blockIdx.x == 0 && i == 0) continue;  // test: this K stage never arrives
        if (lane == 0) {
          const uint32_t fb = bar(b_full + s);
          mbar_arrive_expect_tx(fb, (uint32_t)np * 16 * D * 2);
          uint8_t* dst = ring + s * S::KSTAGE;
          for (int pp = 0; pp < np; ++pp) {
#pragma unroll
            for (int h = 0; h < S::HALVES; ++h)
              tma_load_2d(smem_u32(dst + h * S::KBLK + pp * 2048), tm, 64 * h, rows[pp], fb);
          }
        }
        lastpar = (lastpar & ~(1u << s)) | ((uint32_t)((i / NST) & 1) << s);
        any |= 1u << s;
      }
      if (!ok) break;
    }
    if (lane == 0)
      for (int s = 0; s < NST; ++s)
        if (any & (1u << s)) mbar_wait_bounded(bar(b_full + s), (lastpar >> s) & 1u, a.timeout_ns);
  } else if (warp == 1 || warp == kMmaWarps - 2) {
    // ---------------- tcgen05.mma issuers: lane 0 of warp 1 issues the S
    // products, lane 0 of the second-to-last warp the p.V products, each on its
    // own waits, so neither issue path waits behind the other; a commit tracks
    // the MMAs of the thread that issues it.
    if (lane == 0) {
      const bool is_s = warp == 1;
      // tiles of at most 64 rows: M = 64 products (rows in the first 16 lanes of
      // each lane quarter, the layout the softmax reads them in)
      constexpr uint32_t idesc_s128 = umma_idesc_bf16(128, kMmaKT, false, false);
      constexpr uint32_t idesc_o128 = umma_idesc_bf16(128, D, false, true);
      constexpr uint32_t idesc_s64 = umma_idesc_bf16(64, kMmaKT, false, false);
      constexpr uint32_t idesc_o64 = umma_idesc_bf16(64, D, false, true);
      bool ok = true;
      int i = 0, segord = 0, qn = 0;
      for (;;) {
        const int si = seg_take(qn, true);
        if (si == -2) ok = false;
        if (si < 0) break;
        const pa_seg seg = a.segs[si];
        const bool m64 = seg.sole * G <= 64;  // a tensor-core unit's sole: its requests
        if (a.debug_checks && QR == 64 && !m64) record_status(a.status, PA_ERR_DEVICE, blockIdx.x, -8);
        const uint32_t idesc_s = m64 ? idesc_s64 : idesc_s128, idesc_o = m64 ? idesc_o64 : idesc_o128;
        const int npages = (seg.n_tokens + 15) >> 4;
        for (int st = 0; st < npages; st += 4, ++i) {
          const int s = i % NST, b = i % kSBufs;
          const bool first = st == 0;
          if (is_s) {
            // K landed; Q of the segment loaded; the buffer's last p.V (stage i - 3) done
            if (!mbar_wait_bounded(bar(S::B_FULL + s), (i / NST) & 1, a.timeout_ns) ||
                (first && !mbar_wait_bounded(bar(S::B_QFULL + (segord & 1)), (segord >> 1) & 1, a.timeout_ns)) ||
                (i >= kSBufs && !mbar_wait_bounded(bar(S::B_PV + b), ((i / kSBufs) - 1) & 1, a.timeout_ns))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t k_base = smem_u32(smem + S::OFF_K + s * S::KSTAGE);
            const uint32_t qb = q_base + (segord & 1) * S::QBUF;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // Q and K: K-major 128-byte swizzle, 64-dim blocks, 8-row groups at +1 KB
              const uint64_t ad = umma_sdesc_sw128(qb + (kk >> 2) * S::QBLK + (kk & 3) * 32, 1, 64);
              const uint64_t bd = umma_sdesc_sw128(k_base + (kk >> 2) * S::KBLK + (kk & 3) * 32, 1, 64);
              umma_bf16(tmem + S::T_S + b * kMmaKT, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar(S::B_SFULL + b));
            umma_commit(bar(S::B_EMPTY + s));  // the K slot is free once S is done
          } else {
            // P written; V landed; the first p.V of a segment overwrites O, so the
            // previous epilogue must have read it
            if (!mbar_wait_bounded(bar(S::B_PFULL + b), (i / kSBufs) & 1, a.timeout_ns) ||
                !mbar_wait_bounded(bar(S::B_VFULL + s), (i / NST) & 1, a.timeout_ns) ||
                (first && segord >= 1 && !mbar_wait_bounded(bar(S::B_OFREE), (segord - 1) & 1, a.timeout_ns))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t v_base = smem_u32(smem + S::OFF_V + s * S::KSTAGE);
            const int np = min(4, npages - st);
            // 64-row launches: the whole stage goes to the accumulator of the
            // group that owns it (stage j of the unit: group j % 2), whose first
            // stage in the unit (j < 2) overwrites it
            const int jst = st >> 2;
            for (int c = 0; c < np; ++c) {
              // 16-key chunk c (page c of the stage) belongs to key half c / 2.  P
              // chunk c: P_hi in columns [16c, 16c + 8), P_lo in [16c + 8, 16c + 16)
              // of the buffer; V: MN-major (64-dim atoms at +KBLK, 8-key groups at +1 KB)
              const uint32_t d_o = tmem + S::T_O + (QR == 64 ? (jst & 1) : (c >> 1)) * D;
              const bool init = QR == 64 ? (jst < 2 && c == 0) : (first && (c & 1) == 0);
              const uint32_t a_p = tmem + S::T_S + b * kMmaKT + 16 * c;
              const uint64_t bd = umma_sdesc_sw128(v_base + c * 2048, S::KBLK >> 4, 64);
              umma_bf16_ts(d_o, a_p, bd, idesc_o, init ? 0u : 1u);
              umma_bf16_ts(d_o, a_p + 8, bd, idesc_o, 1u);
            }
            umma_commit(bar(S::B_PV + b));
            umma_commit(bar(S::B_VEMPTY + s));
          }
        }
        if (!ok) break;
        ++segord;
      }
      if (!ok) record_status(a.status, PA_ERR_TIMEOUT, blockIdx.x, is_s ? -3 : -5);
      // every MMA issued by either thread has completed before TMEM is released
      umma_commit(bar(S::B_DONE));
      mbar_wait_bounded(bar(S::B_DONE), 0, a.timeout_ns);
    }
  } else {
    // ---------------- softmax: warps 2-5 take key half 0 of every stage, warps
    // 6-9 key half 1; the rows a thread holds depend on the tile's shape
    // (run_segment below)
    const int h = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int hw = lane >> 4;
    const int rq = quad * 32 + lane;  // the Q row this thread copies
    const int tid = (warp - 2) * 32 + lane;  // 0 .. 255
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    constexpr int QCH = D / 16;  // 16-byte q chunks per row loaded by each half
    bool ok = true;
    int i = 0, segord = 0;
    // The q row this thread copies for segment si (nullptr: a row past the tile's)
    auto q_src = [&](int si) -> const uint16_t* {
      const pa_seg seg = a.segs[si];  // query: the unit's first index into queries; sole: its requests
      if (rq >= seg.sole * G || rq >= QR) return nullptr;
      int b = a.queries[seg.query + rq / G];
      if (a.debug_checks && (uint32_t)b >= (uint32_t)a.B) {
        record_status(a.status, PA_ERR_DEVICE, blockIdx.x, -1 - b);
        b = 0;
      }
      return a.q + ((size_t)b * a.Hq + seg.kv_head * G + (rq % G)) * D;
    };
    // This thread's half of Q row rq into Q buffer qbuf (K-major, 128-byte swizzle).
    auto q_dst = [&](int qbuf, int c) -> uint8_t* {
      return smem + S::OFF_Q + qbuf * S::QBUF + (c >> 3) * S::QBLK + rq * 128 + (((c & 7) ^ (rq & 7)) << 4);
    };
    // the first segment: plain loads
    auto load_q = [&](int si) {
      const uint16_t* src = q_src(si);
#pragma unroll
      for (int cc = 0; cc < QCH; ++cc) {
        const int c = h * QCH + cc;
        const uint4 v = src ? *reinterpret_cast<const uint4*>(src + 8 * c) : make_uint4(0, 0, 0, 0);
        if (rq < QR) *reinterpret_cast<uint4*>(q_dst(0, c)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(S::B_QFULL));
    };
    // later segments: copied asynchronously while the previous segment runs
    // (16-byte cp.async, zero-filled past the tile's rows), published on the
    // buffer's barrier a stage later
    auto prefetch_q = [&](int si, int qbuf) {
      const uint16_t* src = q_src(si);
      if (rq < QR) {
#pragma unroll
        for (int cc = 0; cc < QCH; ++cc) {
          const int c = h * QCH + cc;
          cp_async16(smem_u32(q_dst(qbuf, c)), src ? src + 8 * c : a.q, src ? 16u : 0u);
        }
      }
      cp_async_commit();
    };
    bool q_pending = false;
    // S(i) is read from tensor memory into sv; inside a segment the load of
    // S(i + 1) is issued while P(i) is being stored, when S(i + 1) is already
    // there (else at the top of the next stage)
    float sv[32];
    bool have_s = false;
    int qn = 0;
    // the next queue entry, by the whole warp (lane 0 frees the entry)
    auto take = [&]() -> int {
      const int j = qn % kSegQ;
      const bool got = warp_wait(bar(S::B_QF + j), (qn / kSegQ) & 1, a.timeout_ns);
      const int v = segq[j];
      __syncwarp();
      if (lane == 0 && got) mbar_arrive(bar(S::B_QE + j));
      ++qn;
      return !got ? -2 : v < 0 ? -1 : a.n_segs_simt + v;
    };
    int si = take();
    if (si == -2) ok = false;
    if (si >= 0) load_q(si);
    // One work unit, in the TMEM layout of its tile shape.  Tiles of more than
    // 64 rows use M = 128 products: row r in lane r, thread (r, h) holds keys
    // [32h, 32h + 32) of every stage.  Tiles of at most 64 rows use M = 64
    // products, whose rows sit in the first 16 lanes of each lane quarter (row
    // 16q + j in lane 32q + j): thread (row, h, hw = lane / 16) holds keys
    // [32h + 16hw, 32h + 16hw + 16), so all four quarters, and with them all four
    // SM sub-partitions, share the exponentials of a 64-row tile; the two
    // half-warps of a row combine their maxima with one shuffle per stage and
    // their sums in the epilogue.  Returns false if a wait gave up.
    auto run_segment = [&](auto m64_tag, const pa_seg& seg, const int R) -> bool {
      constexpr bool M64 = decltype(m64_tag)::value;
      constexpr int KT = M64 ? 16 : 32;  // keys of a stage held by this thread
      const int r = M64 ? quad * 16 + (lane & 15) : rq;
      const int kt0 = M64 ? 32 * h + 16 * hw : 32 * h;  // its first key in the stage
      // a warp whose rows all lie past the tile's keeps every barrier of the
      // protocol but skips the arithmetic (its P and O rows are never read out)
      const bool act = (M64 ? quad * 16 : quad * 32) < R;
      auto load_s_tile = [&](int i_) {
        tc_fence_after();
        const uint32_t ta = tmem + S::T_S + (i_ % kSBufs) * kMmaKT + 32 * h + lane_off;
        if constexpr (M64) tmem_ld16x2_x16<16>(ta, sv);
        else tmem_ld32(ta, sv);
      };
      const int npages = (seg.n_tokens + 15) >> 4;
      float m_used = -INFINITY, l = 0.f;
      bool q_known = false;  // the next work unit has been seen in the queue
      int q_at = 0;          // the stage at which its Q rows were requested
      for (int st = 0; st < npages; st += 4, ++i) {
        const int s = i % NST, b = i % kSBufs;
        const int np = min(4, npages - st);
        const int kvalid = min(kMmaKT, seg.n_tokens - st * 16);
        const int kv_t = max(0, min(KT, kvalid - kt0));  // valid keys of this thread
        const bool last = st + 4 >= npages;
        if (!have_s) {
          if (!warp_wait(bar(S::B_SFULL + b), (i / kSBufs) & 1, a.timeout_ns)) return false;
          if (act) load_s_tile(i);
        }
        have_s = false;
        if (act) tmem_wait_ld_into(sv);
        const uint32_t t_s = tmem + S::T_S + b * kMmaKT + 32 * h + lane_off;
        // the Q buffer of the previous segment is free (all its S products have
        // been read): the next work unit's rows are copied into it as soon as
        // the unit is in the queue, and published a stage later (or at this
        // segment's last stage).  At the last stage the wait for the queue entry
        // is a real one: the K producer has issued this segment's loads by then
        // and takes the next unit at once.
        if (!q_known) {
          int nsi = -1;
          bool seen = seg_peek(qn, nsi);
          if (!seen && last) {
            if (!mbar_wait_bounded(bar(S::B_QF + qn % kSegQ), (qn / kSegQ) & 1, a.timeout_ns)) return false;
            seen = seg_peek(qn, nsi);
          }
          if (seen) {
            q_known = true;
            q_at = st;
            if (nsi >= 0) {
              prefetch_q(nsi, (segord + 1) & 1);
              q_pending = true;
            }
          }
        }
        if (q_pending && (st > q_at || last)) {
          cp_async_wait_all();
          fence_proxy_async_smem();
          mbar_arrive(bar(S::B_QFULL + ((segord + 1) & 1)));
          q_pending = false;
        }
        if (act) {
          // the unmasked path only when every lane of the warp has all its keys
          // (with M = 64 the two half-warps can differ): the tensor-memory
          // stores below are .sync.aligned, so the branch must not diverge
          const bool full = __all_sync(0xffffffffu, kv_t == KT);
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if (full) {
#pragma unroll
            for (int j = 0; j < KT; ++j) mx4[j & 3] = fmaxf(mx4[j & 3], sv[j]);
          } else {
#pragma unroll
            for (int j = 0; j < KT; ++j)
              if (j < kv_t) mx4[j & 3] = fmaxf(mx4[j & 3], sv[j]);
          }
          float mraw = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          if constexpr (M64) mraw = fmaxf(mraw, __shfl_xor_sync(0xffffffffu, mraw, 16));
          const float mnew = fmaxf(m_used, mraw == -INFINITY ? -INFINITY : mraw * a.qscale);
          if (st == 0) {
            m_used = mnew;
          } else {
            const bool need = mnew > m_used + kRescaleThreshold;
            if (__any_sync(0xffffffffu, need)) {
              // O_h must hold every earlier p.V product before it is rescaled
              const int j = i - 1;
              if (!warp_wait(bar(S::B_PV + j % kSBufs), (j / kSBufs) & 1, a.timeout_ns)) return false;
              tc_fence_after();
              const float alpha = need ? ex2(m_used - mnew) : 1.f;
              if constexpr (M64) {
                // half-warp hw rescales columns [hw D/2, (hw + 1) D/2) of the row
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                  float ov[32];
                  tmem_ld16x2_x32<D / 2>(tmem + S::T_O + h * D + lane_off + 32 * c, ov);
                  tmem_wait_ld();
#pragma unroll
                  for (int jj = 0; jj < 32; ++jj) ov[jj] *= alpha;
                  tmem_st16x2_x32<D / 2>(tmem + S::T_O + h * D + lane_off + 32 * c, ov);
                }
              } else {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                  float ov[32];
                  tmem_ld32(tmem + S::T_O + h * D + lane_off + 32 * c, ov);
                  tmem_wait_ld();
#pragma unroll
                  for (int jj = 0; jj < 32; ++jj) ov[jj] *= alpha;
                  tmem_st32(tmem + S::T_O + h * D + lane_off + 32 * c, ov);
                }
              }
              tmem_wait_st();
              if (need) {
                l *= alpha;
                m_used = mnew;
              }
            }
          }
          const float ms = m_used == -INFINITY ? 0.f : m_used;
          // p, and its split P_hi + P_lo: P_hi keeps the top 16 bits of p (a
          // truncated bf16, so the remainder p - P_hi is exact in fp32), P_lo is
          // that remainder rounded to the nearest bf16 (P_hi + P_lo is within
          // 2^-16 p of p, with no one-sided bias).  A page of 16 keys is 8 P_hi
          // words then 8 P_lo words; each is stored as soon as it is done, so
          // its store overlaps the next page's exponentials.
          float pw[32];
          float l4[4] = {0.f, 0.f, 0.f, 0.f};
          auto page = [&](auto pg_tag, auto full_tag) {
            constexpr int PG = decltype(pg_tag)::value;
            constexpr bool FULL = decltype(full_tag)::value;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int j = PG * 8 + jj;
              float p0 = ex2(fmaf(sv[2 * j], a.qscale, -ms));
              float p1 = ex2(fmaf(sv[2 * j + 1], a.qscale, -ms));
              if (!FULL) {
                p0 = 2 * j < kv_t ? p0 : 0.f;
                p1 = 2 * j + 1 < kv_t ? p1 : 0.f;
              }
              l4[jj & 3] += p0 + p1;
              const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
              const float r0 = p0 - __uint_as_float(u0 & 0xFFFF0000u), r1 = p1 - __uint_as_float(u1 & 0xFFFF0000u);
              pw[PG * 16 + jj] = __uint_as_float(__byte_perm(u0, u1, 0x7632));
              pw[PG * 16 + jj + 8] = __uint_as_float(pack_bf16x2(r0, r1));
            }
            // M = 64: the two half-warps' pages go to columns [0, 16) and
            // [16, 32) of the key half in one store
            if constexpr (M64) tmem_st16x2_x16<16>(t_s, pw);
            else tmem_st16<PG * 16>(t_s + PG * 16, pw);
          };
          using I0 = std::integral_constant<int, 0>;
          using I1 = std::integral_constant<int, 1>;
          if (full) {
            page(I0{}, std::true_type{});
            if constexpr (!M64) page(I1{}, std::true_type{});
          } else {
            page(I0{}, std::false_type{});
            if constexpr (!M64) page(I1{}, std::false_type{});
          }
          l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
          if (!last &&
              __all_sync(0xffffffffu, mbar_test_wait(bar(S::B_SFULL + (i + 1) % kSBufs), ((i + 1) / kSBufs) & 1))) {
            load_s_tile(i + 1);
            have_s = true;
          }
        }  // act
        if (kvalid < np * 16) {
          // V rows past the last valid key may hold NaN; p = 0 there but 0 * NaN
          // would still poison the product, so those rows are zeroed (once the
          // V tile has landed)
          if (!warp_wait(bar(S::B_VFULL + s), (i / NST) & 1, a.timeout_ns)) return false;
          uint8_t* vst = smem + S::OFF_V + s * S::KSTAGE;
          const int nz = np * 16 - kvalid;
          for (int idx = tid; idx < nz * S::HALVES * 8; idx += kSmaxThreads) {
            const int row = kvalid + idx / (S::HALVES * 8);
            const int hh = (idx >> 3) % S::HALVES, c = idx & 7;
            *reinterpret_cast<uint4*>(vst + hh * S::KBLK + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(S::B_PFULL + b));
      }
      // ---- epilogue: combine the two key halves of each row; this thread
      // writes head dims [h D/2, (h + 1) D/2) of the row's partial result
      // (M = 64: [h D/2 + hw D/4, h D/2 + (hw + 1) D/4))
      {
        const int j = i - 1;
        if (!warp_wait(bar(S::B_PV + j % kSBufs), (j / kSBufs) & 1, a.timeout_ns)) return false;
      }
      if constexpr (M64) l += __shfl_xor_sync(0xffffffffu, l, 16);
      tc_fence_after();
      if (act) {
        const uint32_t mine[2] = {__float_as_uint(m_used), __float_as_uint(l)};
        tmem_st2(tmem + S::T_X + 2 * h + lane_off, mine);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(S::B_XCH + quad));
      if (!warp_wait(bar(S::B_XCH + quad), segord & 1, a.timeout_ns)) return false;
      tc_fence_after();
      if (act) {
        uint32_t other[2];
        tmem_ld2(tmem + S::T_X + 2 * (1 - h) + lane_off, other);
        tmem_wait_ld();
        const float m0 = h == 0 ? m_used : __uint_as_float(other[0]), l0 = h == 0 ? l : __uint_as_float(other[1]);
        const float m1 = h == 0 ? __uint_as_float(other[0]) : m_used, l1 = h == 0 ? __uint_as_float(other[1]) : l;
        const float mm = fmaxf(m0, m1);
        const float w0 = l0 > 0.f ? ex2(m0 - mm) : 0.f, w1 = l1 > 0.f ? ex2(m1 - mm) : 0.f;
        const float L = w0 * l0 + w1 * l1;
        const float c0 = w0 / L, c1 = w1 / L;
        constexpr int NCOL = M64 ? D / 4 : D / 2;  // dims written by this thread
        float* dst = nullptr;
        if (r < R) {
          const int prow = a.seg_prows[seg.prow + r / G];
          dst = a.partial_o + ((size_t)prow * G + (r % G)) * D + h * (D / 2) + (M64 ? hw * NCOL : 0);
          if (h == 0 && (!M64 || hw == 0)) a.partial_lse[(size_t)prow * G + (r % G)] = (mm + lg2(L)) * kLn2;
        }
        // n dims from column 0 of o0 / o1 to d (32-byte aligned), 8 per store
        auto emit = [&](const float (&o0)[32], const float (&o1)[32], int n, float* d) {
          auto cmb = [&](int j) { return c0 * o0[j] + (w1 > 0.f ? c1 * o1[j] : 0.f); };
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            if (8 * q8 >= n) break;
            const int j = 8 * q8;
            st_global_v8(d + j, cmb(j), cmb(j + 1), cmb(j + 2), cmb(j + 3), cmb(j + 4), cmb(j + 5), cmb(j + 6),
                         cmb(j + 7));
          }
        };
        if constexpr (M64) {
          float o0[32], o1[32];
          const uint32_t col = h * (D / 2);
          if constexpr (NCOL == 32) {
            tmem_ld16x2_x32<NCOL>(tmem + S::T_O + col + lane_off, o0);
            tmem_ld16x2_x32<NCOL>(tmem + S::T_O + D + col + lane_off, o1);
          } else {
            tmem_ld16x2_x16<NCOL>(tmem + S::T_O + col + lane_off, o0);
            tmem_ld16x2_x16<NCOL>(tmem + S::T_O + D + col + lane_off, o1);
          }
          tmem_wait_ld();
          if (dst) emit(o0, o1, NCOL, dst);
        } else {
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc) {
            const uint32_t col = h * (D / 2) + 32 * cc;
            float o0[32], o1[32];
            tmem_ld32(tmem + S::T_O + col + lane_off, o0);
            tmem_ld32(tmem + S::T_O + D + col + lane_off, o1);
            tmem_wait_ld();
            if (dst) emit(o0, o1, 32, dst + 32 * cc);
          }
        }
      }  // act
      return true;
    };
    // 64-row launches (QR = 64): the two warp groups take alternate stages of a
    // work unit instead of alternate key halves of every stage.  Group g (warps
    // 2-5: g = 0, 6-9: g = 1) owns stages j = g, g + 2, ... of the unit, with
    // its own running maximum, sum and accumulator O_g; thread (row, hw = lane /
    // 16) holds keys [32 hw, 32 hw + 32) of an owned stage, the two half-warps
    // of a row combining their maxima with one shuffle.  Each group then has
    // two stage periods for the chain S load -> exponentials -> P store of
    // one stage, so the chains of two stages overlap.  A group arrives on the
    // P barrier of a stage it does not own once S of that stage is there (so
    // the barrier's previous phase is complete).  Returns false if a wait
    // gave up.
    auto run_segment_il = [&](auto, const pa_seg& seg, const int R) -> bool {
      constexpr int KT = 32;
      const int r = quad * 16 + (lane & 15);
      const int kt0 = 32 * hw;
      const bool act = quad * 16 < R;
      const int npages = (seg.n_tokens + 15) >> 4;
      float m_used = -INFINITY, l = 0.f;
      bool mine_seen = false;  // this group has run a stage of the unit
      bool q_known = false;
      int q_at = 0;
      for (int st = 0, j = 0; st < npages; st += 4, ++i, ++j) {
        const int s = i % NST, b = i % kSBufs;
        const int np = min(4, npages - st);
        const int kvalid = min(kMmaKT, seg.n_tokens - st * 16);
        const bool last = st + 4 >= npages;
        const bool mine = (j & 1) == h;
        // next work unit's Q rows (as in run_segment)
        if (!q_known) {
          int nsi = -1;
          bool seen = seg_peek(qn, nsi);
          if (!seen && last) {
            if (!mbar_wait_bounded(bar(S::B_QF + qn % kSegQ), (qn / kSegQ) & 1, a.timeout_ns)) return false;
            seen = seg_peek(qn, nsi);
          }
          if (seen) {
            q_known = true;
            q_at = st;
            if (nsi >= 0) {
              prefetch_q(nsi, (segord + 1) & 1);
              q_pending = true;
            }
          }
        }
        if (q_pending && (st > q_at || last)) {
          cp_async_wait_all();
          fence_proxy_async_smem();
          mbar_arrive(bar(S::B_QFULL + ((segord + 1) & 1)));
          q_pending = false;
        }
        if (!mine) {
          // S(i) issued means p.V(i - 3), and with it the previous phase of
          // this P barrier, is complete; only then is the arrival counted for
          // stage i
          if (!warp_wait(bar(S::B_SFULL + b), (i / kSBufs) & 1, a.timeout_ns)) return false;
          mbar_arrive(bar(S::B_PFULL + b));
          continue;
        }
        if (!warp_wait(bar(S::B_SFULL + b), (i / kSBufs) & 1, a.timeout_ns)) return false;
        const uint32_t t_s = tmem + S::T_S + b * kMmaKT + lane_off;
        if (act) {
          tc_fence_after();
          tmem_ld16x2_x32<32>(t_s, sv);
          tmem_wait_ld_into(sv);
          const int kv_t = max(0, min(KT, kvalid - kt0));
          const bool full = __all_sync(0xffffffffu, kv_t == KT);
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if (full) {
#pragma unroll
            for (int jj = 0; jj < KT; ++jj) mx4[jj & 3] = fmaxf(mx4[jj & 3], sv[jj]);
          } else {
#pragma unroll
            for (int jj = 0; jj < KT; ++jj)
              if (jj < kv_t) mx4[jj & 3] = fmaxf(mx4[jj & 3], sv[jj]);
          }
          float mraw = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          mraw = fmaxf(mraw, __shfl_xor_sync(0xffffffffu, mraw, 16));
          const float mnew = fmaxf(m_used, mraw == -INFINITY ? -INFINITY : mraw * a.qscale);
          if (!mine_seen) {
            m_used = mnew;
          } else {
            const bool need = mnew > m_used + kRescaleThreshold;
            if (__any_sync(0xffffffffu, need)) {
              // O_g must hold every earlier p.V product of the group (stage i - 2)
              const int jp = i - 2;
              if (!warp_wait(bar(S::B_PV + jp % kSBufs), (jp / kSBufs) & 1, a.timeout_ns)) return false;
              tc_fence_after();
              const float alpha = need ? ex2(m_used - mnew) : 1.f;
#pragma unroll
              for (int c = 0; c < D / 64; ++c) {
                float ov[32];
                tmem_ld16x2_x32<D / 2>(tmem + S::T_O + h * D + lane_off + 32 * c, ov);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) ov[jj] *= alpha;
                tmem_st16x2_x32<D / 2>(tmem + S::T_O + h * D + lane_off + 32 * c, ov);
              }
              tmem_wait_st();
              if (need) {
                l *= alpha;
                m_used = mnew;
              }
            }
          }
          const float ms = m_used == -INFINITY ? 0.f : m_used;
          // P_hi / P_lo of the thread's two 16-key chunks (2 hw and 2 hw + 1):
          // pw[16 c' + 0..7] = P_hi words, pw[16 c' + 8..15] = P_lo words
          float pw[32];
          float l4[4] = {0.f, 0.f, 0.f, 0.f};
          auto chunk = [&](auto pg_tag, auto full_tag) {
            constexpr int PG = decltype(pg_tag)::value;
            constexpr bool FULL = decltype(full_tag)::value;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int k2 = PG * 8 + jj;
              float p0 = ex2(fmaf(sv[2 * k2], a.qscale, -ms));
              float p1 = ex2(fmaf(sv[2 * k2 + 1], a.qscale, -ms));
              if (!FULL) {
                p0 = 2 * k2 < kv_t ? p0 : 0.f;
                p1 = 2 * k2 + 1 < kv_t ? p1 : 0.f;
              }
              l4[jj & 3] += p0 + p1;
              const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
              const float r0 = p0 - __uint_as_float(u0 & 0xFFFF0000u), r1 = p1 - __uint_as_float(u1 & 0xFFFF0000u);
              pw[PG * 16 + jj] = __uint_as_float(__byte_perm(u0, u1, 0x7632));
              pw[PG * 16 + jj + 8] = __uint_as_float(pack_bf16x2(r0, r1));
            }
          };
          using I0 = std::integral_constant<int, 0>;
          using I1 = std::integral_constant<int, 1>;
          if (full) {
            chunk(I0{}, std::true_type{});
            chunk(I1{}, std::true_type{});
          } else {
            chunk(I0{}, std::false_type{});
            chunk(I1{}, std::false_type{});
          }
          // lanes 0-15: columns [0, 32) of the stage, lanes 16-31: [32, 64)
          tmem_st16x2_x32<32>(t_s, pw);
          l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
        }  // act
        mine_seen = true;
        if (kvalid < np * 16) {
          // V rows past the last valid key may hold NaN (see run_segment);
          // zeroed by the owning group once the V tile has landed
          if (!warp_wait(bar(S::B_VFULL + s), (i / NST) & 1, a.timeout_ns)) return false;
          uint8_t* vst = smem + S::OFF_V + s * S::KSTAGE;
          const int nz = np * 16 - kvalid;
          const int gt = tid & 127;  // thread within the group
          for (int idx = gt; idx < nz * S::HALVES * 8; idx += 128) {
            const int row = kvalid + idx / (S::HALVES * 8);
            const int hh = (idx >> 3) % S::HALVES, c = idx & 7;
            *reinterpret_cast<uint4*>(vst + hh * S::KBLK + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(S::B_PFULL + b));
      }
      // ---- epilogue: combine the two groups' partial results of each row;
      // thread (row, g, hw) writes head dims [g D/2 + hw D/4, g D/2 + (hw + 1) D/4)
      {
        const int jl = i - 1;
        if (!warp_wait(bar(S::B_PV + jl % kSBufs), (jl / kSBufs) & 1, a.timeout_ns)) return false;
      }
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      tc_fence_after();
      if (act) {
        const uint32_t mine2[2] = {__float_as_uint(m_used), __float_as_uint(l)};
        tmem_st2(tmem + S::T_X + 2 * h + lane_off, mine2);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(S::B_XCH + quad));
      if (!warp_wait(bar(S::B_XCH + quad), segord & 1, a.timeout_ns)) return false;
      tc_fence_after();
      if (act) {
        uint32_t other[2];
        tmem_ld2(tmem + S::T_X + 2 * (1 - h) + lane_off, other);
        tmem_wait_ld();
        const float m0 = h == 0 ? m_used : __uint_as_float(other[0]), l0 = h == 0 ? l : __uint_as_float(other[1]);
        const float m1 = h == 0 ? __uint_as_float(other[0]) : m_used, l1 = h == 0 ? __uint_as_float(other[1]) : l;
        const float mm = fmaxf(m0, m1);
        const float w0 = l0 > 0.f ? ex2(m0 - mm) : 0.f, w1 = l1 > 0.f ? ex2(m1 - mm) : 0.f;
        const float L = w0 * l0 + w1 * l1;
        const float c0 = w0 / L, c1 = w1 / L;
        constexpr int NCOL = D / 4;
        float* dst = nullptr;
        if (r < R) {
          const int prow = a.seg_prows[seg.prow + r / G];
          dst = a.partial_o + ((size_t)prow * G + (r % G)) * D + h * (D / 2) + hw * NCOL;
          if (h == 0 && hw == 0) a.partial_lse[(size_t)prow * G + (r % G)] = (mm + lg2(L)) * kLn2;
        }
        float o0[32], o1[32];
        const uint32_t col = h * (D / 2);
        if constexpr (NCOL == 32) {
          tmem_ld16x2_x32<NCOL>(tmem + S::T_O + col + lane_off, o0);
          tmem_ld16x2_x32<NCOL>(tmem + S::T_O + D + col + lane_off, o1);
        } else {
          tmem_ld16x2_x16<NCOL>(tmem + S::T_O + col + lane_off, o0);
          tmem_ld16x2_x16<NCOL>(tmem + S::T_O + D + col + lane_off, o1);
        }
        tmem_wait_ld();
        if (dst) {
          // a group that ran no stage of the unit (a one-stage unit) left its
          // accumulator unwritten: its weight is 0 and its values are not read
          auto cmb = [&](int j) { return (w0 > 0.f ? c0 * o0[j] : 0.f) + (w1 > 0.f ? c1 * o1[j] : 0.f); };
#pragma unroll
          for (int q8 = 0; q8 < NCOL / 8; ++q8) {
            const int j = 8 * q8;
            st_global_v8(dst + j, cmb(j), cmb(j + 1), cmb(j + 2), cmb(j + 3), cmb(j + 4), cmb(j + 5), cmb(j + 6),
                         cmb(j + 7));
          }
        }
      }  // act
      return true;
    };
    while (si >= 0 && ok) {
      const pa_seg seg = a.segs[si];
      const int R = seg.sole * G;
      if constexpr (QR == 64) ok = run_segment_il(0, seg, R);
      else ok = R <= 64 ? run_segment(std::true_type{}, seg, R) : run_segment(std::false_type{}, seg, R);
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(bar(S::B_OFREE));
      // these rows' pairs are merged by their last arrival (fused merge) or the tail merge launch
      ++segord;
      si = take();
      if (si == -2) ok = false;
    }
    tmem_wait_ld();  // a load of S issued ahead before a failed wait
    cp_async_wait_all();  // a Q prefetch still in flight after a failed wait
    if (!ok && lane == 0) record_status(a.status, PA_ERR_TIMEOUT, blockIdx.x, warp);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, kTmemCols);
}

// Tensor-core class: CTA c runs MMA CTA list c.  It lets the CUDA-core launch
// that follows it in the stream start at once (programmatic dependent launch).
template <int D, int G, int QR>
__global__ void __launch_bounds__(kMmaThreads, 1)
    mma_fwd_kernel(const FwdArgs a, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
  griddep_launch_dependents();
  extern __shared__ __align__(1024) uint8_t smem[];
  mma_role<D, G, QR>(a, &tk, &tv, smem);
}

// CUDA-core class: block c runs SIMT warps [8c, 8c + 8).  When it runs beside
// a tensor-core launch it does not end before that launch has, so work later
// in the stream sees both.
template <int D, int G>
__global__ void __launch_bounds__(kSimtWarpsPerCta * 32, 1)
    simt_fwd_kernel(const FwdArgs a, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
  extern __shared__ __align__(1024) uint8_t smem[];
  simt_role<D, G>(a, &tk, &tv, smem);
  griddep_wait();
}

struct MergeArgs {
  const int32_t* prow_off;
  const float* partial_lse;
  const float* partial_o;
  void* out;  // bf16 [B][Hq][D], or fp32 when out_f32
  float* lse;
  int B, Hq, Hkv, G;
  int out_f32;
};

// One warp per (request, kv head) pair: every pair (list == nullptr), or the
// n pairs b*Hkv+g listed.
template <int D, int G>
__global__ void __launch_bounds__(256) merge_kernel(const MergeArgs a, const int32_t* list, int n) {
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= n) return;
  const int bg = list ? list[w] : w;
  if (a.out_f32)
    merge_pair<D, G, float>(a.partial_lse, a.partial_o, static_cast<float*>(a.out), a.lse, a.Hq, bg / a.Hkv,
                            bg % a.Hkv, a.prow_off[bg], a.prow_off[bg + 1], lane);
  else
    merge_pair<D, G>(a.partial_lse, a.partial_o, static_cast<__nv_bfloat16*>(a.out), a.lse, a.Hq, bg / a.Hkv,
                     bg % a.Hkv, a.prow_off[bg], a.prow_off[bg + 1], lane);
}

// Merge of rows gathered from several parts (context parallelism: each part
// is one rank's attention over its slice of the requests' KV, normalised, in
// fp32, with its log-sum-exp).  Part p holds rows_per_part rows; row j of part
// p is request req[p][j] (ascending within a part; -1 marks padding).  One
// warp per (request, query head): for each part, a binary search finds the
// request's row, and the rows found are combined with the merge stage's
// log-sum-exp rule in part order.
template <int D>
__global__ void __launch_bounds__(256)
    merge_rows_kernel(int n_parts, int rows_per_part, int B, int Hq, const int32_t* __restrict__ req,
                      const float* __restrict__ part_o, const float* __restrict__ part_lse, __nv_bfloat16* out,
                      float* lse) {
  constexpr int VPL = D / 32;
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= B * Hq) return;
  const int b = w / Hq, h = w % Hq;
  float m = -INFINITY, z = 0.f, acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  for (int p = 0; p < n_parts; ++p) {
    const int32_t* rq = req + (size_t)p * rows_per_part;
    int lo = 0, hi = rows_per_part;  // first row whose request is >= b (padding counts as past the end)
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      const int v = rq[mid];
      if (v >= 0 && v < b) lo = mid + 1;
      else hi = mid;
    }
    if (lo >= rows_per_part || rq[lo] != b) continue;
    const size_t row = (size_t)p * rows_per_part + lo;
    const float lp = part_lse[row * Hq + h];
    if (lp == -INFINITY) continue;
    const float* src = part_o + (row * Hq + h) * D + lane * VPL;
    float o[VPL];
#pragma unroll
    for (int i = 0; i < VPL; i += 2) {
      const float2 v = *reinterpret_cast<const float2*>(src + i);
      o[i] = v.x;
      o[i + 1] = v.y;
    }
    const float mn = fmaxf(m, lp);
    const float sa = m == -INFINITY ? 0.f : expf(m - mn);
    const float wgt = expf(lp - mn);
    z = z * sa + wgt;
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] = fmaf(o[i], wgt, acc[i] * sa);
    m = mn;
  }
  __nv_bfloat16* dst = out + ((size_t)b * Hq + h) * D + lane * VPL;
  const float inv = z > 0.f ? 1.f / z : 0.f;
#pragma unroll
  for (int i = 0; i < VPL; i += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
  if (lse && lane == 0) lse[(size_t)b * Hq + h] = z > 0.f ? m + logf(z) : -INFINITY;
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
  a.simt_wpc = p.hdr.simt_warps_per_cta >= 1 && p.hdr.simt_warps_per_cta <= kSimtWarpsPerCta
                   ? p.hdr.simt_warps_per_cta : kSimtWarpsPerCta;
  a.n_segs_simt = p.hdr.num_segments_simt;
  a.n_mma_ctas = p.hdr.mma_ctas;
  a.qscale = p.scale * kLog2e;
  a.timeout_ns = (uint64_t)p.wait_timeout_us * 1000ull;
  a.fault_drop = (p.flags & PA_PLAN_FAULT_DROP_LOAD) ? 1 : 0;
  a.debug_checks = (p.flags & PA_PLAN_DEBUG_CHECKS) ? 1 : 0;
  a.tile_maps = p.tma_tiles ? 1 : 0;
  a.n_segs_mma = p.hdr.num_segments_mma;
  a.mma_next = d.mma_next;
  a.mix_pairs = d.mix_pairs;
  a.n_mix_pairs = p.hdr.num_mix_pairs;
  a.num_pages = p.num_pages_in_pool;
  a.B = p.B;
  return a;
}

// Max dynamic shared memory is set once per kernel and device.
template <typename K>
int set_smem_attr(K kernel, bool (&done)[64]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (e != cudaSuccess) return (int)e;
    done[dev] = true;
  }
  return 0;
}

// The tensor-core launch (if any) first, then the CUDA-core launch, which may
// start while the first still runs (programmatic stream serialization); the
// two occupy disjoint SMs (one CTA per SM each, n_mma + n_simt <= SMs).
template <int D, int G>
int launch_fwd_t(const pa_plan& p, const FwdArgs& a, cudaStream_t st) {
  static bool attr_mma[64] = {}, attr_mma64[64] = {}, attr_simt[64] = {};
  const int n_simt_ctas = (a.n_simt_warps + a.simt_wpc - 1) / a.simt_wpc;
  const CUtensorMap* tk = reinterpret_cast<const CUtensorMap*>(p.tma_k);
  const CUtensorMap* tv = reinterpret_cast<const CUtensorMap*>(p.tma_v);
  if (a.n_mma_ctas > 0) {
    // launches whose tiles all have at most 64 rows: 64-row Q buffers (a
    // deeper K/V ring at D = 128) and the stage-interleaved softmax
    if (p.mma_max_rows <= 64) {
      auto k = mma_fwd_kernel<D, G, 64>;
      if (int e = set_smem_attr(k, attr_mma64)) return e;
      k<<<a.n_mma_ctas, kMmaThreads, MmaShape<D, 64>::SMEM, st>>>(a, *tk, *tv);
    } else {
      auto k = mma_fwd_kernel<D, G, 128>;
      if (int e = set_smem_attr(k, attr_mma)) return e;
      k<<<a.n_mma_ctas, kMmaThreads, MmaShape<D, 128>::SMEM, st>>>(a, *tk, *tv);
    }
    if (cudaError_t e = cudaGetLastError()) return (int)e;
  }
  if (n_simt_ctas > 0) {
    const CUtensorMap* sk = p.tma_tiles ? reinterpret_cast<const CUtensorMap*>(p.tma_k3) : tk;
    const CUtensorMap* sv = p.tma_tiles ? reinterpret_cast<const CUtensorMap*>(p.tma_v3) : tv;
    auto k = simt_fwd_kernel<D, G>;
    if (int e = set_smem_attr(k, attr_simt)) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_simt_ctas);
    cfg.blockDim = dim3(a.simt_wpc * 32);
    cfg.dynamicSmemBytes = SimtShape<D, G>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.n_mma_ctas > 0 ? 1 : 0;
    if (cudaError_t e = cudaLaunchKernelEx(&cfg, k, a, *sk, *sv)) return (int)e;
  }
  return 0;
}

template <int D, int G>
int launch_merge_t(const MergeArgs& a, const int32_t* list, int n, cudaStream_t st) {
  merge_kernel<D, G><<<(n + 7) / 8, 256, 0, st>>>(a, list, n);
  return (int)cudaGetLastError();
}

}  // namespace pa

using namespace pa;

int pa_launch_forward(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream) {
  const FwdArgs a = make_fwd_args(p, d, out, lse);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
#define PA_FWD_CASE(DD, GG) \
  if (p.D == DD && p.G == GG) return launch_fwd_t<DD, GG>(p, a, st);
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

namespace {

int launch_merge_list(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, const int32_t* list, int n,
                      void* stream, bool out_f32 = false) {
  if (n <= 0) return 0;
  MergeArgs a;
  a.prow_off = d.prow_off;
  a.partial_lse = d.partial_lse;
  a.partial_o = d.partial_o;
  a.out = out;
  a.out_f32 = out_f32 ? 1 : 0;
  a.lse = lse;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.G = p.G;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
#define PA_MERGE_CASE(DD, GG) \
  if (p.D == DD && p.G == GG) return launch_merge_t<DD, GG>(a, list, n, st);
  PA_MERGE_CASE(128, 4)
  PA_MERGE_CASE(128, 1)
  PA_MERGE_CASE(128, 2)
  PA_MERGE_CASE(128, 8)
  PA_MERGE_CASE(64, 4)
  PA_MERGE_CASE(64, 1)
  PA_MERGE_CASE(64, 2)
  PA_MERGE_CASE(64, 8)
#undef PA_MERGE_CASE
  return (int)cudaErrorInvalidValue;
}

}  // namespace

int pa_launch_merge(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream, bool out_f32) {
  return launch_merge_list(p, d, out, lse, nullptr, p.B * p.Hkv, stream, out_f32);
}

int pa_launch_merge_rows(int n_parts, int rows_per_part, int B, int Hq, int D, const int32_t* req,
                         const float* part_o, const float* part_lse, void* out, float* lse, void* stream) {
  const int n = B * Hq;
  if (n <= 0) return 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  if (D == 128) merge_rows_kernel<128><<<(n + 7) / 8, 256, 0, st>>>(n_parts, rows_per_part, B, Hq, req, part_o,
                                                                    part_lse, o, lse);
  else if (D == 64) merge_rows_kernel<64><<<(n + 7) / 8, 256, 0, st>>>(n_parts, rows_per_part, B, Hq, req, part_o,
                                                                       part_lse, o, lse);
  else return (int)cudaErrorInvalidValue;
  return (int)cudaGetLastError();
}

int pa_launch_tail_merge(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream) {
  return launch_merge_list(p, d, out, lse, d.tail_pairs, p.hdr.num_tail_pairs, stream);
}

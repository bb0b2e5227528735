// Pack stage (host): tree-structured block table, profit model, split of long
// nodes, tile-class selection, work ordering and partial-row assignment.
//
// Source: the PAT review, section 三 (Pack Scheduler 工作流, Figure 7: a decode
// batch, its tree-structured block table, packing scheme 1 that keeps a parent
// node separate from its leaves and packing scheme 2 that folds a leaf together
// with its parent; Pack 阶段: group queries by shared prefix into CTA work with a
// profit-model heuristic that weighs prefix length and query count; Forward 阶段:
// a runtime tile selector, multi-stream execution and long-KV splitting).  The
// page gives no formula for the profit model or the split; the rules used here
// are stated at each step.
//
// Cost: every (request, page) entry of the block table is compared at most
// once while the tree is built, and the work lists are written with one pass
// over the items, so planning is linear in the number of pages.
#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstring>
#include <cstdlib>
#include <mutex>
#include <new>
#include <numeric>
#include <stdexcept>
#include <thread>
#include <vector>

#include "plan.h"

namespace {

std::mutex g_buf_mu;
std::vector<HostBuf> g_buf_free;  // at most kMaxFreeBufs kept

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

// First index in [from, to) where rows a and b differ (to if none): 64-byte
// chunks compared with memcmp, then the differing chunk element by element.
inline int first_diff(const int32_t* a, const int32_t* b, int from, int to) {
  int i = from;
  while (i + 16 <= to && std::memcmp(a + i, b + i, 64) == 0) i += 16;
  for (; i < to; ++i)
    if (a[i] != b[i]) return i;
  return to;
}

struct ItemRec {
  int page_off, n_tokens, n_queries, query_off;
  bool simt;
};

struct SegRec {
  int item, kv_head, page_begin, n_tokens, prow, query;
  // a resized list is overwritten before it is read: no zero fill
  SegRec() {}
  SegRec(int it, int g, int pb, int nt, int pr, int q)
      : item(it), kv_head(g), page_begin(pb), n_tokens(nt), prow(pr), query(q) {}
};

struct Planner {
  const int32_t* kv_lens;
  const int32_t* bt;
  int max_pages, P, G, Hq, Hkv, D;
  uint32_t flags;
  int num_pages_in_pool;
  std::vector<int>& order;
  std::vector<int>& npg;
  // outputs of the tree walk
  std::vector<ItemRec>& items;
  std::vector<int32_t>& pages;
  std::vector<int32_t>& queries;
  std::vector<int>& qbuf;
  int64_t unique_tokens = 0, read_tokens = 0;
  int num_nodes = 0, num_shared = 0, num_kept = 0;
  bool invalid = false;
  // set for the first call of the walk: its subtrees may be walked on several
  // threads (walk_kids)
  bool split_top = false;

  const int32_t* row(int b) const { return bt + (size_t)b * max_pages; }

  void add_item(int rep, int page_lo, int page_hi, int64_t tokens, const int* qs, int nq, bool simt) {
    const int off = (int)pages.size();
    const int32_t* r = row(rep);
    pages.insert(pages.end(), r + page_lo, r + page_hi);
    // page ids are validated here: every (request, page) entry of the batch is
    // copied into exactly one item (entries of a shared run are equal across
    // its requests), so this checks each id once per item instead of once per
    // request
    uint32_t bad = 0;
    for (int j = off; j < (int)pages.size(); ++j) bad |= (uint32_t)pages[j] >= (uint32_t)num_pages_in_pool ? 1u : 0u;
    if (bad) invalid = true;
    if (simt) {
      items.push_back({off, (int)tokens, 1, (int)queries.size(), true});
      queries.push_back(qs[0]);
      read_tokens += tokens;
      return;
    }
    // tensor-core class: query tiles of at most kMmaRowsPerCta rows
    const int qpt = std::max(1, kMmaRowsPerCta / G);
    for (int t = 0; t < nq; t += qpt) {
      const int n = std::min(qpt, nq - t);
      items.push_back({off, (int)tokens, n, (int)queries.size(), false});
      queries.insert(queries.end(), qs + t, qs + t + n);
      read_tokens += tokens;
    }
  }

  // Profit model (packing scheme 1 vs 2).  A node with n >= 2 requests whose
  // item would cover L tokens stays shared iff
  //     (n - 1) * L * Bt  >  n * Hq * (4D + 4) * 2 + C_item,
  // Bt = K+V bytes per token over all kv heads: what sharing saves is the
  // (n - 1) extra reads of the node; what it costs is one more fp32 partial row
  // per request and head (written by forward, read by merge) and a fixed
  // per-item overhead C_item.  Otherwise the node is folded into its children.
  // C_item is a tensor-core work unit's fixed cost (an epilogue of ≈3.7 us,
  // the Q rows, the pipeline ramp) in bytes of re-reading instead: a 16-page
  // prefix shared by 4 requests (config 1, 393 KB saved) ran slower shared
  // than inlined (1024 such problems: 129 us against 107 us on one B200).
  bool keep_shared(int n, int64_t L) const {
    if (flags & PA_PLAN_NO_SHARING) return false;
    if (flags & PA_PLAN_ALWAYS_SHARE) return true;
    const double Bt = 2.0 * Hkv * D * 2, C_item = 512.0 * 1024;
    return (n - 1) * (double)L * Bt > n * (double)Hq * (4.0 * D + 4.0) * 2.0 + C_item;
  }

  // Requests order[lo, hi) share logical pages [0, depth).  eff_lo is the first
  // page not yet covered by an emitted ancestor (pages of folded ancestors are
  // read again by this subtree's items).
  void walk(int lo, int hi, int depth, int eff_lo) {
    if (invalid) return;
    const bool top = split_top;
    split_top = false;
    if (hi - lo == 1) {
      const int b = order[lo];
      if (npg[b] > depth) {
        ++num_nodes;
        unique_tokens += kv_lens[b] - (int64_t)depth * P;
      }
      add_item(b, eff_lo, npg[b], kv_lens[b] - (int64_t)eff_lo * P, &b, 1, true);
      return;
    }
    // extend the common prefix: the shortest agreement of any row with the first
    const int32_t* r0 = row(order[lo]);
    int l = npg[order[lo]];
    for (int i = lo + 1; i < hi; ++i) l = std::min(l, npg[order[i]]);
    for (int i = lo + 1; i < hi && l > depth; ++i) l = first_diff(r0, row(order[i]), depth, l);
    bool keep = false;
    int next_eff = eff_lo;
    if (l > depth) {
      // a page is packed as shared only where it is full for every request
      // that holds it: the shared node stops before the first page that is
      // partial for one of them
      int lf = l;
      for (int i = lo; i < hi; ++i) lf = std::min(lf, kv_lens[order[i]] / P);
      if (lf <= depth) {
        // page `depth` is the last, partial page of some requests (the same
        // page id for all of them): those read their own tail; the requests
        // for which it is full are walked again without them
        auto mid = std::partition(order.begin() + lo, order.begin() + hi,
                                  [&](int b) { return kv_lens[b] / P <= depth; });
        const int e = (int)(mid - order.begin());
        int64_t tail = 0;
        for (int i = lo; i < e; ++i) {
          const int b = order[i];
          tail = std::max<int64_t>(tail, kv_lens[b] - (int64_t)depth * P);
          add_item(b, eff_lo, npg[b], kv_lens[b] - (int64_t)eff_lo * P, &b, 1, true);
        }
        if (e < hi) {
          walk(e, hi, depth, eff_lo);  // they hold page `depth` whole: it counts there
        } else {
          ++num_nodes;
          unique_tokens += tail;
        }
        return;
      }
      l = lf;
    }
    const int nq = hi - lo;
    if (l > depth) {
      ++num_nodes;
      ++num_shared;
      unique_tokens += (int64_t)(l - depth) * P;
      keep = keep_shared(nq, (int64_t)(l - eff_lo) * P);
      if (keep) {
        ++num_kept;
        qbuf.assign(order.begin() + lo, order.begin() + hi);
        std::sort(qbuf.begin(), qbuf.end());
        add_item(qbuf[0], eff_lo, l, (int64_t)(l - eff_lo) * P, qbuf.data(), nq, false);
        next_eff = l;
      }
    }
    // requests ending at page l come first; the rest are grouped by their page at l
    auto mid = std::partition(order.begin() + lo, order.begin() + hi, [&](int b) { return npg[b] == l; });
    const int e = (int)(mid - order.begin());
    for (int i = lo; i < e; ++i)
      if (!keep && l > eff_lo) {
        const int b = order[i];
        add_item(b, eff_lo, l, kv_lens[b] - (int64_t)eff_lo * P, &b, 1, true);
      }
    std::sort(order.begin() + e, order.begin() + hi, [&](int a, int b) {
      const int32_t pa = row(a)[l], pb = row(b)[l];
      return pa != pb ? pa < pb : a < b;
    });
    int start = e;
    std::vector<std::pair<int, int>> kids;  // the first call's subtrees
    for (int i = e + 1; i <= hi; ++i) {
      if (i == hi || row(order[i])[l] != row(order[start])[l]) {
        if (top) kids.emplace_back(start, i);
        else walk(start, i, l, next_eff);
        start = i;
      }
    }
    if (top) walk_kids(kids, l, next_eff);
  }

  // The subtrees of the first call, in order.  The walk reads the block table
  // once (each row is compared with its group's first row), ≈10 MB for a
  // batch like config 5's, so large batches walk contiguous runs of subtrees
  // of about equal work on up to kWalkThreads threads: each thread writes its
  // own items, pages and queries (the subtrees own disjoint ranges of `order`
  // and read the inputs only), and the outputs are appended in subtree order,
  // so the plan is the one the serial walk gives.
  void walk_kids(const std::vector<std::pair<int, int>>& kids, int depth, int eff) {
    constexpr int kWalkThreads = 8;
    constexpr int64_t kMinWalkPagesPerThread = 32768;
    std::vector<int64_t> work(kids.size(), 0);
    int64_t total = 0;
    for (size_t k = 0; k < kids.size(); ++k) {
      for (int i = kids[k].first; i < kids[k].second; ++i) work[k] += std::max(0, npg[order[i]] - depth);
      total += work[k];
    }
    int T = (int)std::min<int64_t>({(int64_t)kWalkThreads, (int64_t)kids.size(), total / kMinWalkPagesPerThread});
    if (T >= 2) {
      // the host's thread count, asked once (a system call of a few us)
      static const unsigned hw = std::max(1u, std::thread::hardware_concurrency());
      T = std::min<int>(T, (int)hw);
    }
    if (T < 2) {
      for (const auto& k : kids) walk(k.first, k.second, depth, eff);
      return;
    }
    // contiguous runs of subtrees, about total / T pages each
    std::vector<size_t> cut(1, 0);
    int64_t acc = 0;
    for (size_t k = 0; k < kids.size(); ++k) {
      acc += work[k];
      if ((int)cut.size() < T && acc * T >= total * (int64_t)cut.size() && k + 1 < kids.size()) cut.push_back(k + 1);
    }
    cut.push_back(kids.size());
    const int n = (int)cut.size() - 1;
    struct Part {
      std::vector<ItemRec> items;
      std::vector<int32_t> pages, queries;
      std::vector<int> qbuf;
    };
    std::vector<Part> parts(n);
    std::vector<Planner> subs;
    subs.reserve(n);
    for (int t = 0; t < n; ++t)
      subs.push_back(Planner{kv_lens, bt, max_pages, P, G, Hq, Hkv, D, flags, num_pages_in_pool, order, npg,
                             parts[t].items, parts[t].pages, parts[t].queries, parts[t].qbuf});
    auto run = [&](int t) {
      try {
        for (size_t k = cut[t]; k < cut[t + 1]; ++k) subs[t].walk(kids[k].first, kids[k].second, depth, eff);
      } catch (...) {
        subs[t].invalid = true;
      }
    };
    std::vector<std::thread> th;
    th.reserve(n);
    int started = 0;
    try {
      for (int t = 1; t < n; ++t, ++started) th.emplace_back(run, t);
    } catch (...) {
      // a thread could not start: the rest of the runs are walked here
    }
    run(0);
    for (int t = 1 + started; t < n; ++t) run(t);
    for (auto& x : th) x.join();
    for (int t = 0; t < n; ++t) {
      const Planner& sp = subs[t];
      const int base_p = (int)pages.size(), base_q = (int)queries.size();
      for (ItemRec it : parts[t].items) {
        it.page_off += base_p;
        it.query_off += base_q;
        items.push_back(it);
      }
      pages.insert(pages.end(), parts[t].pages.begin(), parts[t].pages.end());
      queries.insert(queries.end(), parts[t].queries.begin(), parts[t].queries.end());
      unique_tokens += sp.unique_tokens;
      read_tokens += sp.read_tokens;
      num_nodes += sp.num_nodes;
      num_shared += sp.num_shared;
      num_kept += sp.num_kept;
      invalid = invalid || sp.invalid;
    }
  }
};

// Reusable scratch of the planner (one per host thread), so a plan costs no
// allocation once the sizes have been seen.
struct Scratch {
  std::vector<int> order, npg, qbuf;
  std::vector<ItemRec> items;
  std::vector<int32_t> pages, queries, warp_segs, mma_cta_segs, prow_off, cursor, seg_prows, tail_pairs, mix_pairs,
      warp_order;
  std::vector<SegRec> simt_segs, mma_segs;
  std::vector<int32_t> n_mma_rows;
};

Scratch& scratch() {
  static thread_local Scratch sc;
  return sc;
}

}  // namespace

HostBuf hostbuf_acquire(size_t n) {
  {
    std::lock_guard<std::mutex> lock(g_buf_mu);
    size_t best = g_buf_free.size();
    for (size_t i = 0; i < g_buf_free.size(); ++i)
      if (g_buf_free[i].cap >= n && (best == g_buf_free.size() || g_buf_free[i].cap < g_buf_free[best].cap)) best = i;
    if (best < g_buf_free.size()) {
      HostBuf b = g_buf_free[best];
      g_buf_free.erase(g_buf_free.begin() + best);
      b.size = n;
      return b;
    }
  }
  HostBuf b;
  size_t cap = 4096;
  while (cap < n) cap <<= 1;
  b.ptr = static_cast<uint8_t*>(std::malloc(cap));
  if (!b.ptr) throw std::bad_alloc();
  b.cap = cap;
  b.size = n;
  return b;
}

namespace {
thread_local ImageSink t_sink = nullptr;
thread_local void* t_sink_ctx = nullptr;
}  // namespace

void pa_set_image_sink(ImageSink sink, void* ctx) {
  t_sink = sink;
  t_sink_ctx = ctx;
}

void hostbuf_release(HostBuf& b) {
  if (!b.ptr) return;
  if (!b.owned) {
    b = HostBuf{};
    return;
  }
  constexpr size_t kMaxFreeBufs = 16;
  std::lock_guard<std::mutex> lock(g_buf_mu);
  if (g_buf_free.size() < kMaxFreeBufs) g_buf_free.push_back(b);
  else std::free(b.ptr);
  b = HostBuf{};
}

// What the split and the image need from the pack stage.
struct PackCounts {
  int64_t unique_tokens = 0, read_tokens = 0;
  int num_nodes = 0, num_shared = 0, num_kept = 0;
};

// Split, partial rows and image of a plan whose pack result (items, their
// pages and requests) is given; fills plan->hdr, plan->image and plan->stats.
static void finish_plan(pa_plan* plan, Scratch& sc, const std::vector<ItemRec>& items, const std::vector<int32_t>& pages,
                 const std::vector<int32_t>& queries, const PackCounts& pc, const int32_t* kv_lens,
                 std::chrono::steady_clock::time_point t0) {
  const int batch = plan->B, Hq = plan->Hq, Hkv = plan->Hkv, G = plan->G, D = plan->D, P = plan->P;
  const pa_config* cfg = &plan->cfg;

  // ---- split and tile selection
  // Tile class by rows (requests x G): one request -> SIMT class (CUDA
  // cores); two or more -> MMA class (tensor cores, query tiles of <= 128 rows).
  // The two classes run as two concurrent launches of one CTA per SM each; k
  // SMs take the MMA class, the rest the SIMT class.  k balances the two
  // classes' estimated times:
  //   T_simt(k) = SIMT tile bytes / ((num_sms - k) * kSimtBytesPerSmUs)
  //   T_mma(k)  = sum over MMA tiles of max(bytes / kMmaBytesPerSmUs,
  //               flops / kMmaFlopsPerSmUs) / k
  // Both classes split their work stream-K: the (item, kv head) page runs are
  // concatenated and cut into equal spans, one span per SIMT warp or per MMA
  // CTA; a span may end inside an item, so partial rows appear only at span
  // boundaries (long-KV splitting without a fixed chunk size).
  const double kSimtBytesPerSmUs = 56.0e3;   // bytes per us per SM, small-row class
  const int kSimtSegPages = 2;               // fixed cost of a SIMT work unit, in pages
  const double kMmaBytesPerSmUs = 40.0e3;    // bytes per us per SM, tensor-core class
  const double kMmaFlopsPerSmUs = 5.0e6;     // flop per us per SM, tcgen05 class, running beside the SIMT class
  const int kMmaSegPages = 24;               // fixed cost of a 128-row tensor-core segment (epilogue), in pages
  // the epilogue's stores scale with the tile's rows: a tile of r rows pays
  // kMmaSegPages * max(32, r) / 128
  auto mma_seg_pages = [&](const ItemRec& it) -> int64_t {
    const int rows = std::min(kMmaRowsPerCta, it.n_queries * G);
    return (int64_t)kMmaSegPages * std::max(32, rows) / kMmaRowsPerCta;
  };
  const int64_t max_chunk_pages = cfg->max_chunk_tokens > 0 ? std::max(1, cfg->max_chunk_tokens / P) : 0;
  const double tile_bytes = 2.0 * 16 * D * 2;
  int64_t simt_pages = 0, mma_pages = 0;
  double mma_cost = 0;  // SM-us
  for (const auto& it : items) {
    const int64_t np = ceil_div(it.n_tokens, P) * Hkv;
    if (it.simt) {
      // a SIMT work unit also pays a fixed latency (q rows, partial row,
      // arrival): counted as kSimtSegPages more pages
      simt_pages += np + kSimtSegPages * Hkv;
    } else {
      mma_pages += np;
      // a tcgen05.mma costs the same for any rows up to 128, so a tile costs 128 rows
      const double rows = kMmaRowsPerCta;
      const double flops = 16.0 * rows * D * 6;  // per page: S (2rD per key) + split-p P.V (2 x 2rD per key)
      mma_cost += (np + mma_seg_pages(it) * Hkv) * std::max(tile_bytes / kMmaBytesPerSmUs, flops / kMmaFlopsPerSmUs);
    }
  }
  const int S = plan->num_sms;
  int n_mma = 0;  // SMs given to the MMA class
  if (mma_pages > 0 && simt_pages == 0) {
    n_mma = S;
  } else if (mma_pages > 0) {
    // T_simt = A / (S - k) and T_mma = C / k are equal at k = S C / (A + C);
    // take the better of the two integers around it; no more CTAs than
    // 16-page spans of tensor-core work
    const double A = simt_pages * tile_bytes / kSimtBytesPerSmUs, C = mma_cost;
    const int k_cap = (int)std::min<int64_t>(S - 1, std::max<int64_t>(1, ceil_div(mma_pages, 16)));
    const int k0 = std::max(1, std::min(k_cap, (int)(S * C / (A + C))));
    double best = 1e300;
    for (int kk = k0; kk <= std::min(k_cap, k0 + 1); ++kk) {
      const double t = std::max(A / (S - kk), C / kk);
      if (t < best) { best = t; n_mma = kk; }
    }
    // one SM: each class still gets one CTA (the two launches then run one
    // after the other instead of side by side)
    if (n_mma < 1) n_mma = 1;
  }
  std::vector<SegRec>& simt_segs = sc.simt_segs;
  std::vector<SegRec>& mma_segs = sc.mma_segs;
  std::vector<int32_t>& warp_segs = sc.warp_segs;
  std::vector<int32_t>& mma_cta_segs = sc.mma_cta_segs;
  simt_segs.clear();
  mma_segs.clear();
  warp_segs.assign(1, 0);
  mma_cta_segs.assign(1, 0);
  if (mma_pages > 0) {
    // Tensor-core work units, cut for guided self-scheduling: the CTAs take
    // the units one after another from a counter in the image (the K producer
    // of each CTA fetches the next one), longest first, so an SM that runs
    // faster takes more of them (the same stage of the same work was measured
    // to take from 0.79 to 1.17 us on different SMs of one launch).  Each cut
    // takes about R / (kGuide * CTAs) pages, R being the tensor-core work not
    // yet cut, from the run with the most pages left: the units shrink as the
    // queue drains, so the last ones, whose end on a slow SM decides when the
    // launch ends, are short, while most of the work still runs in long units.
    // A unit is at least kMmaMinChunkPages long: each one pays an epilogue
    // (about 3 us, during which its CTA's tensor pipe waits) and one more
    // partial row per request and head.  When that leaves about one unit per
    // CTA, each unit gets a CTA of its own.
    const int kMmaMinChunkPages = 64;
    const double kGuide = 2.0;
    struct Run {
      int64_t rem;  // pages not yet cut
      int item, g, pb;
    };
    const auto fewer = [](const Run& x, const Run& y) { return x.rem < y.rem; };  // max-heap on rem
    std::vector<Run> runs;
    int64_t R = 0;
    for (size_t i = 0; i < items.size(); ++i) {
      const ItemRec& it = items[i];
      if (it.simt) continue;
      const int64_t npages = ceil_div(it.n_tokens, P);
      for (int g = 0; g < Hkv; ++g) runs.push_back({npages, (int)i, g, 0});
      R += npages * Hkv;
    }
    std::make_heap(runs.begin(), runs.end(), fewer);
    while (!runs.empty()) {
      std::pop_heap(runs.begin(), runs.end(), fewer);
      Run& r = runs.back();
      int64_t t = std::max<int64_t>(kMmaMinChunkPages, (int64_t)std::ceil((double)R / (kGuide * n_mma)));
      if (max_chunk_pages) t = std::min(t, max_chunk_pages);
      int64_t cut = std::min(t, r.rem);
      // no sliver of less than half a minimum unit is left behind
      if (!max_chunk_pages && r.rem - cut < kMmaMinChunkPages / 2) cut = r.rem;
      const ItemRec& it = items[r.item];
      const int tok = (int)(std::min<int64_t>(it.n_tokens, (r.pb + cut) * P) - (int64_t)r.pb * P);
      mma_segs.push_back({r.item, r.g, r.pb, tok, -1, queries[it.query_off]});
      r.pb += (int)cut;
      r.rem -= cut;
      R -= cut;
      if (r.rem > 0) std::push_heap(runs.begin(), runs.end(), fewer);
      else runs.pop_back();
    }
    std::stable_sort(mma_segs.begin(), mma_segs.end(),
                     [](const SegRec& x, const SegRec& y) { return x.n_tokens > y.n_tokens; });
    const int64_t n_chunks = (int64_t)mma_segs.size();
    if (2 * n_chunks <= 3 * (int64_t)n_mma) n_mma = (int)std::min<int64_t>(n_chunks, std::max(1, S - 1));
    n_mma = (int)std::min<int64_t>(n_mma, n_chunks);
    mma_cta_segs.push_back((int32_t)mma_segs.size());
  }

  // SIMT warps per CTA.  Each warp keeps two D = 128 tiles (16 KB) or three
  // D = 64 tiles (12 KB) in flight; when every warp streams a long run of
  // D = 128 tiles (kSimtLongSpan or more at 8 warps), 6 warps per SM (96 KB in
  // flight) moved the bytes faster than 8 (128 KB) or 10: config 4 262.5
  // against 271.8 and 274.8 us, config 3 208.4 against 211.5 us; with short
  // runs the warps' fixed costs dominate and 8 are faster (config 2 45.6
  // against 47.6 us, 1024 config-1 problems at D = 64 105 against 129 us).
  // The rule is about the HBM traffic of many SMs: a class of a few CTAs
  // beside a long tensor-core launch (config 5) keeps its 8 warps.
  int simt_wpc = kSimtWarpsPerCta;
  if (simt_pages > 0 && D == 128 && 2 * (S - n_mma) >= S &&
      ceil_div(simt_pages, (int64_t)std::max(1, S - n_mma) * kSimtWarpsPerCta) >= kSimtLongSpan)
    simt_wpc = kSimtWarpsPerCtaLong;
  if (simt_pages > 0) {
    const int64_t W = (int64_t)std::max(1, S - n_mma) * simt_wpc;
    int64_t span = ceil_div(simt_pages, W);
    if (span < 4) span = 4;
    if (max_chunk_pages) span = std::min(span, max_chunk_pages);
    // one segment per (item, kv head) run plus one per warp boundary; more
    // when max_chunk_tokens caps the spans below the work per warp (the last
    // warp then cuts its runs into one-page segments), so the writer grows the
    // buffer if needed
    size_t n_units = 0;
    for (const auto& it : items) n_units += it.simt;
    simt_segs.resize(n_units * Hkv + (size_t)W + 8);
    warp_segs.resize((size_t)W + 2);
    SegRec* sp = simt_segs.data();
    int32_t* wp = warp_segs.data() + 1;
    int32_t n_seg = 0, cap = (int32_t)simt_segs.size();
    const int span_i = (int)std::min<int64_t>(span, INT32_MAX / 4), W_i = (int)W;
    int n_warp = 1;
    int used = 0;  // pages in the current warp's span
    for (size_t i = 0; i < items.size(); ++i) {
      const ItemRec& it = items[i];
      if (!it.simt) continue;
      const int npages = (int)ceil_div(it.n_tokens, P);
      const int b = queries[it.query_off];
      for (int g = 0; g < Hkv; ++g) {
        int pb = 0;
        used += kSimtSegPages;  // the unit's fixed cost
        while (pb < npages) {
          const int take = std::max(1, std::min(npages - pb, span_i - used));
          const int tok = std::min(it.n_tokens, (pb + take) * P) - pb * P;
          if (n_seg == cap) {
            simt_segs.resize(2 * (size_t)cap);
            sp = simt_segs.data();
            cap = (int32_t)simt_segs.size();
          }
          sp[n_seg++] = SegRec{(int)i, g, pb, tok, -1, b};
          pb += take;
          used += take;
          if (used >= span_i && n_warp < W_i) {  // never more than W warps
            *wp++ = n_seg;
            ++n_warp;
            used = 0;
          }
        }
      }
    }
    if (used > 0) {
      *wp++ = n_seg;
      ++n_warp;
    }
    simt_segs.resize(n_seg);
    warp_segs.resize(n_warp);
  }
  // ---- partial rows: contiguous per (request, kv head), in a fixed order
  std::vector<int32_t>& prow_off = sc.prow_off;
  prow_off.assign((size_t)batch * Hkv + 1, 0);
  for (const auto& s : mma_segs) {
    const ItemRec& it = items[s.item];
    for (int j = 0; j < it.n_queries; ++j) prow_off[(size_t)queries[it.query_off + j] * Hkv + s.kv_head + 1]++;
  }
  // fused merge: the last SIMT partial row of a pair to be written merges the
  // pair; pairs with tensor-core rows only are merged by the tail merge
  // launch.  A pair with both (mixed) also counts one arrival from a SIMT warp
  // that makes it after its own work, once the tensor-core launch has
  // finished: whichever arrival is the last merges the pair, so it is merged
  // as soon as both classes' rows are there.  Entry k of mix_pairs takes that
  // arrival from warp k mod W (W SIMT warps); the t-th mixed pair goes to the
  // t-th warp of an order that visits every CTA before the second warp of
  // any, so the merges after the tensor-core launch spread over all the
  // class's SMs (entries no pair takes hold -1).  A warp merges its pairs one
  // after another, ≈2.5 us each once the tensor-core launch has finished, so
  // plans with more than kMixPerWarp mixed pairs per warp send them to the
  // tail merge launch instead (config 5: 4096 pairs, 8 warps).
  constexpr int kMixPerWarp = 3;
  std::vector<int32_t>& n_mma_rows = sc.n_mma_rows;
  n_mma_rows.assign(prow_off.begin() + 1, prow_off.end());
  for (const auto& s : simt_segs) prow_off[(size_t)s.query * Hkv + s.kv_head + 1]++;
  const int W = (int)warp_segs.size() - 1;
  int64_t n_mixed = 0;
  for (size_t bg = 0; bg + 1 < prow_off.size(); ++bg)
    n_mixed += n_mma_rows[bg] > 0 && prow_off[bg + 1] > n_mma_rows[bg];
  const bool mixed_to_tail = n_mixed > (int64_t)kMixPerWarp * W;
  std::vector<int32_t>& tail_pairs = sc.tail_pairs;
  std::vector<int32_t>& mix_pairs = sc.mix_pairs;
  tail_pairs.clear();
  mix_pairs.clear();
  std::vector<int32_t>& warp_order = sc.warp_order;
  warp_order.clear();
  if (n_mixed > 0 && !mixed_to_tail) {
    const int n_ctas = (W + simt_wpc - 1) / simt_wpc;
    for (int slot = 0; slot < simt_wpc; ++slot)
      for (int c = 0; c < n_ctas; ++c)
        if (c * simt_wpc + slot < W) warp_order.push_back(c * simt_wpc + slot);
    // the t-th mixed pair takes entry (t / W) W + warp_order[t % W]; the list
    // ends after the last entry taken
    const int64_t last = n_mixed - 1, base = last / W * W;
    int32_t top = 0;
    for (int64_t r = 0; r <= last % W; ++r) top = std::max(top, warp_order[(size_t)r]);
    mix_pairs.assign((size_t)(2 * (base + top + 1)), -1);
  }
  int64_t round = 0;  // (t / W) W for the t-th mixed pair
  int pos = 0;        // t % W
  for (size_t bg = 0; bg + 1 < prow_off.size(); ++bg) {
    if (n_mma_rows[bg] == 0) continue;
    const int n_simt = prow_off[bg + 1] - n_mma_rows[bg];
    if (n_simt == 0 || mixed_to_tail) {
      tail_pairs.push_back((int32_t)bg);
      continue;
    }
    const size_t k = (size_t)(round + warp_order[(size_t)pos]);
    if (++pos == W) {
      pos = 0;
      round += W;
    }
    mix_pairs[2 * k] = (int32_t)bg;
    mix_pairs[2 * k + 1] = n_simt;
  }
  for (size_t i = 1; i < prow_off.size(); ++i) prow_off[i] += prow_off[i - 1];
  std::vector<int32_t>& cursor = sc.cursor;
  cursor.assign(prow_off.begin(), prow_off.end() - 1);
  std::vector<int32_t>& seg_prows = sc.seg_prows;
  seg_prows.clear();
  for (auto& s : mma_segs) {
    const ItemRec& it = items[s.item];
    s.prow = (int)seg_prows.size();
    for (int j = 0; j < it.n_queries; ++j)
      seg_prows.push_back(cursor[(size_t)queries[it.query_off + j] * Hkv + s.kv_head]++);
  }
  for (auto& s : simt_segs) s.prow = cursor[(size_t)s.query * Hkv + s.kv_head]++;
  const int num_prows = prow_off.back();

  // ---- image
  pa_image_header& h = plan->hdr;
  std::memset(&h, 0, sizeof(h));
  h.magic = 0x50414231u;
  h.batch = batch;
  h.num_q_heads = Hq;
  h.num_kv_heads = Hkv;
  h.head_dim = D;
  h.page_size = P;
  h.num_items = (int32_t)items.size();
  h.num_segments_simt = (int32_t)simt_segs.size();
  h.num_segments_mma = (int32_t)mma_segs.size();
  h.num_segments = h.num_segments_simt + h.num_segments_mma;
  h.simt_warps = (int32_t)warp_segs.size() - 1;
  h.simt_warps_per_cta = simt_wpc;
  h.mma_ctas = mma_segs.empty() ? 0 : n_mma;
  plan->mma_max_rows = 0;
  for (const auto& s : mma_segs)
    plan->mma_max_rows = std::max(plan->mma_max_rows, std::min(kMmaRowsPerCta, items[s.item].n_queries * G));
  h.num_partial_rows = num_prows;
  h.num_tail_pairs = (int32_t)tail_pairs.size();
  h.num_mix_pairs = (int32_t)(mix_pairs.size() / 2);
  uint64_t off = align256(sizeof(pa_image_header));
  h.off_nodes = off; off = align256(off + items.size() * sizeof(pa_item));
  h.off_segs = off; off = align256(off + (size_t)h.num_segments * sizeof(pa_seg));
  h.off_pages = off; off = align256(off + pages.size() * 4);
  h.off_queries = off; off = align256(off + queries.size() * 4);
  h.off_seg_prows = off; off = align256(off + seg_prows.size() * 4);
  h.off_mma_segs = off; off = align256(off + mma_cta_segs.size() * 4);
  h.off_counters = off; off = align256(off + (size_t)batch * Hkv * 4);
  h.off_warp_segs = off; off = align256(off + warp_segs.size() * 4);
  h.off_prow_off = off; off = align256(off + prow_off.size() * 4);
  h.off_tail_pairs = off; off = align256(off + tail_pairs.size() * 4);
  h.off_mix_pairs = off; off = align256(off + mix_pairs.size() * 4);
  h.image_bytes = off;
  h.off_partial_lse = off; off = align256(off + (uint64_t)num_prows * G * 4);
  h.off_partial_o = off; off = align256(off + (uint64_t)num_prows * G * D * 4);
  h.workspace_bytes = off;

  uint8_t* lent = t_sink ? t_sink(h.image_bytes, t_sink_ctx) : nullptr;
  if (lent) {
    plan->image.ptr = lent;
    plan->image.size = plan->image.cap = h.image_bytes;
    plan->image.owned = false;
  } else {
    plan->image = hostbuf_acquire(h.image_bytes);
  }
  uint8_t* img = plan->image.data();
  std::memcpy(img, &h, sizeof(h));
  std::memset(img + h.off_counters, 0, (size_t)batch * Hkv * 4);
  pa_item* di = reinterpret_cast<pa_item*>(img + h.off_nodes);
  for (size_t i = 0; i < items.size(); ++i)
    di[i] = {items[i].page_off, items[i].n_tokens, items[i].n_queries, items[i].query_off};
  pa_seg* ds = reinterpret_cast<pa_seg*>(img + h.off_segs);
  size_t k = 0;
  {
    size_t pbg = SIZE_MAX;
    int sole = 0;
    for (const auto& s : simt_segs) {
      const size_t bg = (size_t)s.query * Hkv + s.kv_head;
      if (bg != pbg) {  // a pair's segments are consecutive
        pbg = bg;
        const int n_rows = prow_off[bg + 1] - prow_off[bg], n_simt = n_rows - n_mma_rows[bg];
        const int mode = n_mma_rows[bg] > 0 ? (mixed_to_tail ? 3 : 2) : n_rows == 1 ? 1 : 0;
        sole = mode | (n_simt << 2);
      }
      ds[k++] = {s.item, s.kv_head, s.page_begin, s.n_tokens, s.prow, s.query, sole,
                 items[s.item].page_off + s.page_begin};
    }
  }
  // a tensor-core unit carries its item's request list (query_off, n_queries)
  // itself, so the kernel reaches its pages and Q rows without the item
  for (const auto& s : mma_segs) {
    const ItemRec& it = items[s.item];
    ds[k++] = {s.item, s.kv_head, s.page_begin, s.n_tokens, s.prow, it.query_off, it.n_queries,
               it.page_off + s.page_begin};
  }
  auto put = [&](uint64_t o, const std::vector<int32_t>& v) {
    if (!v.empty()) std::memcpy(img + o, v.data(), v.size() * 4);
  };
  put(h.off_pages, pages);
  put(h.off_queries, queries);
  put(h.off_seg_prows, seg_prows);
  put(h.off_mma_segs, mma_cta_segs);
  put(h.off_warp_segs, warp_segs);
  put(h.off_prow_off, prow_off);
  put(h.off_tail_pairs, tail_pairs);
  put(h.off_mix_pairs, mix_pairs);
  // the alignment gaps after the regions are zeroed: the image depends on the inputs only
  const uint64_t region_end[] = {sizeof(h),
                                 h.off_nodes + items.size() * sizeof(pa_item),
                                 h.off_segs + (uint64_t)h.num_segments * sizeof(pa_seg),
                                 h.off_pages + pages.size() * 4,
                                 h.off_queries + queries.size() * 4,
                                 h.off_seg_prows + seg_prows.size() * 4,
                                 h.off_mma_segs + mma_cta_segs.size() * 4,
                                 h.off_counters + (uint64_t)batch * Hkv * 4,
                                 h.off_warp_segs + warp_segs.size() * 4,
                                 h.off_prow_off + prow_off.size() * 4,
                                 h.off_tail_pairs + tail_pairs.size() * 4,
                                 h.off_mix_pairs + mix_pairs.size() * 4};
  for (const uint64_t e : region_end) std::memset(img + e, 0, align256(e) - e);

  pa_plan_stats& st = plan->stats;
  st.batch = batch;
  st.num_nodes = pc.num_nodes;
  st.num_shared_nodes = pc.num_shared;
  st.num_kept_shared = pc.num_kept;
  st.num_items = (int32_t)items.size();
  st.num_segments = h.num_segments;
  st.num_segments_simt = h.num_segments_simt;
  st.num_segments_mma = h.num_segments_mma;
  st.num_partial_rows = num_prows;
  st.simt_warps = h.simt_warps;
  st.mma_ctas = h.mma_ctas;
  st.num_tail_pairs = h.num_tail_pairs;
  st.unique_tokens = pc.unique_tokens;
  int64_t naive = 0;
  for (int b = 0; b < batch; ++b) naive += kv_lens[b];
  st.naive_tokens = naive;
  st.read_tokens = pc.read_tokens;
  st.unique_kv_bytes = pc.unique_tokens * (int64_t)(2 * Hkv * D * 2);
  st.read_kv_bytes = pc.read_tokens * (int64_t)(2 * Hkv * D * 2);
  st.workspace_bytes = h.workspace_bytes;
  st.image_bytes = h.image_bytes;
  st.plan_us = std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - t0).count();
}

// Stores the pack result in the plan (PA_PLAN_KEEP_PACK) for pa_plan_advance.
static void keep_pack(pa_plan* plan, const std::vector<ItemRec>& items, const std::vector<int32_t>& pages,
                      const std::vector<int32_t>& queries, const PackCounts& pc, const int32_t* kv_lens) {
  plan->pk_items.resize(items.size() * 5);
  for (size_t i = 0; i < items.size(); ++i) {
    int32_t* r = &plan->pk_items[i * 5];
    r[0] = items[i].page_off;
    r[1] = items[i].n_tokens;
    r[2] = items[i].n_queries;
    r[3] = items[i].query_off;
    r[4] = items[i].simt ? 1 : 0;
  }
  plan->pk_pages = pages;
  plan->pk_queries = queries;
  plan->pk_kv_lens.assign(kv_lens, kv_lens + plan->B);
  // a request's one-request item (there is at most one: it ends at the
  // request's last page)
  plan->pk_suffix.assign(plan->B, -1);
  for (size_t i = 0; i < items.size(); ++i)
    if (items[i].simt) plan->pk_suffix[queries[items[i].query_off]] = (int32_t)i;
  plan->pk_unique_tokens = pc.unique_tokens;
  plan->pk_read_tokens = pc.read_tokens;
  plan->pk_num_nodes = pc.num_nodes;
  plan->pk_num_shared = pc.num_shared;
  plan->pk_num_kept = pc.num_kept;
  plan->has_pack = true;
}

extern "C" pa_status pa_plan_create(const pa_config* cfg, int32_t batch, const int32_t* kv_lens,
                                    const int32_t* block_table, int32_t max_pages, int32_t num_pages_in_pool,
                                    pa_plan** out) {
  if (out) *out = nullptr;
  if (!cfg || !kv_lens || !block_table || !out) return PA_ERR_INVALID;
  auto t0 = std::chrono::steady_clock::now();
  const int Hq = cfg->num_q_heads, Hkv = cfg->num_kv_heads, D = cfg->head_dim, P = cfg->page_size;
  if (batch < 1 || max_pages < 1 || num_pages_in_pool < 1 || Hq < 1 || Hkv < 1 || D < 1 || P < 1)
    return PA_ERR_INVALID;
  if (Hq % Hkv != 0) return PA_ERR_INVALID;
  const int G = Hq / Hkv;
  if (!(G == 1 || G == 2 || G == 4 || G == 8)) return PA_ERR_UNSUPPORTED;
  if (!(D == 64 || D == 128)) return PA_ERR_UNSUPPORTED;
  if (P != 16) return PA_ERR_UNSUPPORTED;
  if (cfg->softmax_scale < 0.f || !std::isfinite(cfg->softmax_scale)) return PA_ERR_INVALID;
  if (cfg->max_chunk_tokens < 0 || cfg->wait_timeout_us < 0 || cfg->num_sms < 0) return PA_ERR_INVALID;
  const uint32_t flags = cfg->flags;
  if ((flags & PA_PLAN_NO_SHARING) && (flags & PA_PLAN_ALWAYS_SHARE)) return PA_ERR_INVALID;
  // the kernels address a pool as rows of D values (page, kv head, slot): a TMA coordinate is int32
  if ((int64_t)num_pages_in_pool * Hkv * P > INT32_MAX) return PA_ERR_UNSUPPORTED;

  pa_plan* plan = new (std::nothrow) pa_plan();
  if (!plan) return PA_ERR_NOMEM;
  try {
    plan->cfg = *cfg;
    plan->B = batch;
    plan->Hq = Hq;
    plan->Hkv = Hkv;
    plan->G = G;
    plan->D = D;
    plan->P = P;
    plan->num_pages_in_pool = num_pages_in_pool;
    plan->scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / std::sqrt((float)D);
    plan->num_sms = cfg->num_sms > 0 ? cfg->num_sms : 148;
    plan->flags = flags;
    plan->wait_timeout_us = cfg->wait_timeout_us > 0 ? cfg->wait_timeout_us : 2000000;

    // ---- validation
    Scratch& sc = scratch();
    sc.items.clear();
    sc.pages.clear();
    sc.queries.clear();
    Planner pl{kv_lens, block_table, max_pages, P, G, Hq, Hkv, D, flags, num_pages_in_pool, sc.order, sc.npg,
               sc.items, sc.pages, sc.queries, sc.qbuf};
    pl.kv_lens = kv_lens;
    pl.bt = block_table;
    pl.max_pages = max_pages;
    pl.P = P;
    pl.G = G;
    pl.Hq = Hq;
    pl.Hkv = Hkv;
    pl.D = D;
    pl.flags = flags;
    pl.num_pages_in_pool = num_pages_in_pool;
    pl.npg.resize(batch);
    int64_t total_pages = 0;
    for (int b = 0; b < batch; ++b) {
      const int64_t n = kv_lens[b];
      if (n < 1 || n > (int64_t)max_pages * P) { delete plan; return PA_ERR_INVALID; }
      pl.npg[b] = (int)ceil_div(n, P);
      total_pages += pl.npg[b];
    }

    // ---- tree-structured block table + profit model + emission
    pl.order.resize(batch);
    std::iota(pl.order.begin(), pl.order.end(), 0);
    pl.items.reserve(batch + 64);
    pl.pages.reserve(total_pages);
    pl.queries.reserve(2 * batch);
    pl.split_top = true;
    pl.walk(0, batch, 0, 0);
    if (pl.invalid) { delete plan; return PA_ERR_INVALID; }
    const std::vector<ItemRec>& items = pl.items;
    const std::vector<int32_t>& pages = pl.pages;
    const std::vector<int32_t>& queries = pl.queries;
    PackCounts pc;
    pc.unique_tokens = pl.unique_tokens;
    pc.read_tokens = pl.read_tokens;
    pc.num_nodes = pl.num_nodes;
    pc.num_shared = pl.num_shared;
    pc.num_kept = pl.num_kept;
    finish_plan(plan, sc, items, pages, queries, pc, kv_lens, t0);
    if (flags & PA_PLAN_KEEP_PACK) keep_pack(plan, items, pages, queries, pc, kv_lens);
    *out = plan;
    return PA_OK;
  } catch (const std::bad_alloc&) {
    delete plan;
    return PA_ERR_NOMEM;
  } catch (...) {
    delete plan;
    return PA_ERR_INVALID;
  }
}

extern "C" pa_status pa_plan_advance(const pa_plan* prev, const int32_t* kv_lens, const int32_t* block_table,
                                     int32_t max_pages, int32_t num_pages_in_pool, pa_plan** out) {
  if (out) *out = nullptr;
  if (!prev || !prev->has_pack || !kv_lens || !block_table || !out) return PA_ERR_INVALID;
  auto t0 = std::chrono::steady_clock::now();
  const int batch = prev->B, P = prev->P, Hkv = prev->Hkv;
  if (max_pages < 1 || num_pages_in_pool < 1) return PA_ERR_INVALID;
  if ((int64_t)num_pages_in_pool * Hkv * P > INT32_MAX) return PA_ERR_UNSUPPORTED;
  bool rebuild = num_pages_in_pool < prev->num_pages_in_pool;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = kv_lens[b];
    if (n < 1 || n > (int64_t)max_pages * P) return PA_ERR_INVALID;
    if (n < prev->pk_kv_lens[b]) rebuild = true;
  }
  if (rebuild) {
    const pa_status st = pa_plan_create(&prev->cfg, batch, kv_lens, block_table, max_pages, num_pages_in_pool, out);
    if (st == PA_OK) (*out)->stats.plan_us = std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - t0).count();
    return st;
  }

  pa_plan* plan = new (std::nothrow) pa_plan();
  if (!plan) return PA_ERR_NOMEM;
  try {
    plan->cfg = prev->cfg;
    plan->B = batch;
    plan->Hq = prev->Hq;
    plan->Hkv = Hkv;
    plan->G = prev->G;
    plan->D = prev->D;
    plan->P = P;
    plan->num_pages_in_pool = num_pages_in_pool;
    plan->scale = prev->scale;
    plan->num_sms = prev->num_sms;
    plan->flags = prev->flags;
    plan->wait_timeout_us = prev->wait_timeout_us;

    Scratch& sc = scratch();
    std::vector<ItemRec>& items = sc.items;
    std::vector<int32_t>& pages = sc.pages;
    std::vector<int32_t>& queries = sc.queries;
    const size_t n_items_prev = prev->pk_items.size() / 5;
    items.clear();
    pages.clear();
    queries.assign(prev->pk_queries.begin(), prev->pk_queries.end());
    pages.reserve(prev->pk_pages.size() + 2 * (size_t)batch);
    items.reserve(n_items_prev + batch);
    PackCounts pc;
    pc.unique_tokens = prev->pk_unique_tokens;
    pc.read_tokens = prev->pk_read_tokens;
    pc.num_nodes = prev->pk_num_nodes;
    pc.num_shared = prev->pk_num_shared;
    pc.num_kept = prev->pk_num_kept;
    uint32_t bad = 0;
    auto row = [&](int b) { return block_table + (size_t)b * max_pages; };
    auto append_pages = [&](int b, int from, int to) {
      const int32_t* r = row(b);
      for (int j = from; j < to; ++j) {
        bad |= (uint32_t)r[j] >= (uint32_t)num_pages_in_pool ? 1u : 0u;
        pages.push_back(r[j]);
      }
    };
    // the items in their old order; tiles of one node keep sharing their pages
    int last_old_off = -1, last_new_off = -1;
    for (size_t i = 0; i < n_items_prev; ++i) {
      const int32_t* r = &prev->pk_items[i * 5];
      ItemRec it{r[0], r[1], r[2], r[3], r[4] != 0};
      const int np_old = (int)ceil_div(it.n_tokens, P);
      if (!it.simt && it.page_off == last_old_off) {
        it.page_off = last_new_off;  // another query tile of the same node
      } else {
        const int new_off = (int)pages.size();
        pages.insert(pages.end(), prev->pk_pages.begin() + it.page_off, prev->pk_pages.begin() + it.page_off + np_old);
        last_old_off = it.page_off;
        last_new_off = new_off;
        it.page_off = new_off;
        if (it.simt) {
          // the request's own tail: it takes the new tokens and pages
          const int b = queries[it.query_off];
          const int64_t grow = (int64_t)kv_lens[b] - prev->pk_kv_lens[b];
          if (grow > 0) {
            const int npg_old = (int)ceil_div(prev->pk_kv_lens[b], P), npg_new = (int)ceil_div(kv_lens[b], P);
            append_pages(b, npg_old, npg_new);
            it.n_tokens += (int)grow;
            pc.unique_tokens += grow;
            pc.read_tokens += grow;
          }
        }
      }
      items.push_back(it);
    }
    // requests that ended at the end of a shared node: a new tail item
    for (int b = 0; b < batch; ++b) {
      const int64_t grow = (int64_t)kv_lens[b] - prev->pk_kv_lens[b];
      if (prev->pk_suffix[b] >= 0 || grow <= 0) continue;
      const int npg_old = (int)ceil_div(prev->pk_kv_lens[b], P), npg_new = (int)ceil_div(kv_lens[b], P);
      if ((int64_t)npg_old * P != prev->pk_kv_lens[b]) throw std::logic_error("request ends inside a shared page");
      const int off = (int)pages.size();
      append_pages(b, npg_old, npg_new);
      items.push_back({off, (int)grow, 1, (int)queries.size(), true});
      queries.push_back(b);
      ++pc.num_nodes;
      pc.unique_tokens += grow;
      pc.read_tokens += grow;
    }
    if (bad) {
      delete plan;
      return PA_ERR_INVALID;
    }
    finish_plan(plan, sc, items, pages, queries, pc, kv_lens, t0);
    keep_pack(plan, items, pages, queries, pc, kv_lens);
    plan->stats.plan_us = std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - t0).count();
    *out = plan;
    return PA_OK;
  } catch (const std::bad_alloc&) {
    delete plan;
    return PA_ERR_NOMEM;
  } catch (...) {
    delete plan;
    return PA_ERR_INVALID;
  }
}

extern "C" pa_status pa_plan_create_append(const pa_config* cfg, int32_t n_sessions, const int32_t* ctx_lens,
                                           const int32_t* chunk_lens, const int32_t* block_table, int32_t max_pages,
                                           int32_t num_pages_in_pool, pa_plan** out) {
  if (out) *out = nullptr;
  if (!cfg || !ctx_lens || !chunk_lens || !block_table || !out || n_sessions < 1 || max_pages < 1)
    return PA_ERR_INVALID;
  // one row per new token: row i of session s is a request over the session's
  // block-table row whose length stops at its own token (ctx_lens[s] + i + 1),
  // so it sees the whole context and the chunk tokens up to itself (causal
  // inside the chunk); the rows of a session share the context's full pages,
  // which the pack stage then reads once for all of them
  int64_t rows = 0;
  for (int s = 0; s < n_sessions; ++s) {
    if (ctx_lens[s] < 0 || chunk_lens[s] < 1) return PA_ERR_INVALID;
    if ((int64_t)ctx_lens[s] + chunk_lens[s] > (int64_t)max_pages * cfg->page_size) return PA_ERR_INVALID;
    rows += chunk_lens[s];
  }
  if (rows > INT32_MAX / 2) return PA_ERR_UNSUPPORTED;
  try {
    std::vector<int32_t> kv((size_t)rows), bt((size_t)rows * max_pages);
    size_t r = 0;
    for (int s = 0; s < n_sessions; ++s) {
      const int32_t* src = block_table + (size_t)s * max_pages;
      for (int i = 0; i < chunk_lens[s]; ++i, ++r) {
        kv[r] = ctx_lens[s] + i + 1;
        std::memcpy(&bt[r * max_pages], src, sizeof(int32_t) * max_pages);
      }
    }
    return pa_plan_create(cfg, (int32_t)rows, kv.data(), bt.data(), max_pages, num_pages_in_pool, out);
  } catch (const std::bad_alloc&) {
    return PA_ERR_NOMEM;
  }
}

extern "C" pa_status pa_plan_workspace_size(const pa_plan* plan, size_t* bytes) {
  if (!plan || !bytes) return PA_ERR_INVALID;
  *bytes = plan->hdr.workspace_bytes;
  return PA_OK;
}

extern "C" pa_status pa_plan_get_stats(const pa_plan* plan, pa_plan_stats* out) {
  if (!plan || !out) return PA_ERR_INVALID;
  *out = plan->stats;
  return PA_OK;
}

extern "C" pa_status pa_plan_host_image(const pa_plan* plan, void* dst, size_t bytes) {
  if (!plan || !dst) return PA_ERR_INVALID;
  if (bytes < plan->image.size) return PA_ERR_NOMEM;
  std::memcpy(dst, plan->image.data(), plan->image.size);
  return PA_OK;
}

extern "C" void pa_plan_destroy(pa_plan* plan) { delete plan; }

extern "C" const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PA_ERR_NOMEM: return "out of memory or workspace too small";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_TIMEOUT: return "device wait timed out";
    case PA_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

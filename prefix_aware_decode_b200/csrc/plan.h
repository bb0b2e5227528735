// Internal definition of the host plan object and the kernel launch entry points.
#pragma once

#include <cstdint>
#include <vector>

#include "pa.h"

static_assert(sizeof(pa_seg) == 32, "pa_seg must be 32 bytes (vector loads)");
static_assert(sizeof(pa_item) == 16, "pa_item must be 16 bytes");

// Forward launch shape: one CTA per SM.  A CUDA-core (SIMT) CTA runs up to 8
// independent warps (6 when every warp streams long runs of D = 128 tiles:
// kSimtLongSpan tiles or more; fewer bytes in flight per SM measured faster
// there, see the planner); a tensor-core (MMA) CTA works on tiles of up to
// 128 rows with 12 warps (two TMA producers, two tcgen05 issuers, 8 softmax
// warps).
constexpr int kSimtWarpsPerCta = 8;
constexpr int kSimtWarpsPerCtaLong = 6;
constexpr int kSimtLongSpan = 64;
constexpr int kMmaRowsPerCta = 128;

// Host buffer for plan images, taken from and returned to a small process-wide
// pool so that building a plan does not page-fault fresh memory every time.
struct HostBuf {
  uint8_t* ptr = nullptr;
  size_t size = 0, cap = 0;
  bool owned = true;  // false: memory lent by an image sink, not returned to the pool
  uint8_t* data() const { return ptr; }
};
HostBuf hostbuf_acquire(size_t n);
void hostbuf_release(HostBuf& b);

// Where pa_plan_create writes the plan image on this thread: by default a
// pooled host buffer; a sink set here lends the memory instead (pa_decode_step
// lends a pinned upload buffer, so the image needs no second copy).  The sink
// returns a buffer of at least n bytes, or nullptr to fall back to the pool.
using ImageSink = uint8_t* (*)(size_t n, void* ctx);
void pa_set_image_sink(ImageSink sink, void* ctx);

struct pa_plan {
  pa_config cfg;
  int B = 0, Hq = 0, Hkv = 0, G = 0, D = 0, P = 0;
  int num_pages_in_pool = 0;
  float scale = 0.f;
  int num_sms = 0;
  uint32_t flags = 0;
  int32_t wait_timeout_us = 0;
  pa_plan_stats stats{};
  pa_image_header hdr{};
  // rows of the largest tensor-core tile (n_queries * G, at most 128): when
  // it is at most 64 the launch holds 64-row Q buffers and a deeper K/V ring
  int mma_max_rows = 0;
  HostBuf image;  // exactly what pa_plan_upload sends (image.size bytes)
  ~pa_plan() { hostbuf_release(image); }
  // cached TMA descriptors (encoded for the last pool pointers seen)
  mutable const void* tma_k_ptr = nullptr;
  mutable const void* tma_v_ptr = nullptr;
  alignas(64) mutable uint8_t tma_k[128] = {};
  alignas(64) mutable uint8_t tma_v[128] = {};
  // whole-tile (3-D) maps of the same pools, used by the small-row class when
  // tma_tiles is set (else it copies each tile as D/64 boxes of the 2-D maps)
  mutable bool tma_tiles = false;
  alignas(64) mutable uint8_t tma_k3[128] = {};
  alignas(64) mutable uint8_t tma_v3[128] = {};
  // optional cudaEvent_t handles recorded around the launches (profiling):
  // [0,1] forward launch (pa_forward / pa_attend), [2,3] merge launch
  void* prof[4] = {};
  // device copy of the image when it lives outside the workspace (a half of
  // pa_decode_step's image buffer); nullptr: at the workspace base.  A later
  // pa_plan_upload or pa_attend_noalloc copies the image again and resets it.
  mutable void* dev_image = nullptr;
  // the pack result (PA_PLAN_KEEP_PACK), from which pa_plan_advance plans the
  // next decode step: items (page_off, n_tokens, n_queries, query_off, simt),
  // their pages and requests, each request's kv_len and one-request item (-1:
  // none), and the pack counters
  bool has_pack = false;
  std::vector<int32_t> pk_items, pk_pages, pk_queries, pk_kv_lens, pk_suffix;
  int64_t pk_unique_tokens = 0, pk_read_tokens = 0;
  int pk_num_nodes = 0, pk_num_shared = 0, pk_num_kept = 0;
};

// Kernel launchers (kernels.cu).  Return 0 or a cudaError_t value.
struct PaDevPtrs {
  const uint16_t* q;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  uint8_t* ws;
  const pa_item* items;
  const pa_seg* segs;
  const int32_t* pages;
  const int32_t* queries;
  const int32_t* seg_prows;
  const int32_t* mma_cta_segs;
  int32_t* counters;
  const int32_t* warp_segs;
  const int32_t* prow_off;
  const int32_t* tail_pairs;
  const int32_t* mix_pairs;
  float* partial_lse;
  float* partial_o;
  int32_t* status;
  int32_t* mma_next;
};

// out == nullptr: partial rows only; else the merge is fused into the launch.
int pa_launch_forward(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream);
int pa_launch_merge(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream, bool out_f32 = false);
// Merge of per-part rows gathered across ranks (pa_merge_rows).
int pa_launch_merge_rows(int n_parts, int rows_per_part, int B, int Hq, int D, const int32_t* req,
                         const float* part_o, const float* part_lse, void* out, float* lse, void* stream);
// Merge of the pairs in the plan's tail list (after a fused forward launch).
int pa_launch_tail_merge(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream);

// Device address of the static workspace of pa_attend_noalloc on the current
// device (looked up on first use), or nullptr on error.
void* pa_noalloc_scratch();

// pa_attend on a workspace whose plan image is already (being) uploaded.
pa_status pa_attend_ws(const pa_plan* plan, const void* q, const void* k_pool, const void* v_pool, void* ws,
                       void* out, float* lse, void* stream);

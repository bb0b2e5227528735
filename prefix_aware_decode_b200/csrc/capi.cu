// C ABI: device-side calls of libpa.so (upload, forward, merge, status).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <vector>

#include "plan.h"

namespace {

// Image tables at `image` (the workspace base unless the image was placed
// elsewhere), partial rows in the workspace.
PaDevPtrs dev_ptrs(const pa_plan& p, void* ws) {
  const pa_image_header& h = p.hdr;
  uint8_t* b = static_cast<uint8_t*>(p.dev_image ? p.dev_image : ws);
  uint8_t* w = static_cast<uint8_t*>(ws);
  PaDevPtrs d{};
  d.ws = w;
  d.items = reinterpret_cast<const pa_item*>(b + h.off_nodes);
  d.segs = reinterpret_cast<const pa_seg*>(b + h.off_segs);
  d.pages = reinterpret_cast<const int32_t*>(b + h.off_pages);
  d.queries = reinterpret_cast<const int32_t*>(b + h.off_queries);
  d.seg_prows = reinterpret_cast<const int32_t*>(b + h.off_seg_prows);
  d.mma_cta_segs = reinterpret_cast<const int32_t*>(b + h.off_mma_segs);
  d.counters = reinterpret_cast<int32_t*>(b + h.off_counters);
  d.warp_segs = reinterpret_cast<const int32_t*>(b + h.off_warp_segs);
  d.prow_off = reinterpret_cast<const int32_t*>(b + h.off_prow_off);
  d.tail_pairs = reinterpret_cast<const int32_t*>(b + h.off_tail_pairs);
  d.mix_pairs = reinterpret_cast<const int32_t*>(b + h.off_mix_pairs);
  d.partial_lse = reinterpret_cast<float*>(w + h.off_partial_lse);
  d.partial_o = reinterpret_cast<float*>(w + h.off_partial_o);
  d.status = reinterpret_cast<int32_t*>(b + offsetof(pa_image_header, status));
  d.mma_next = reinterpret_cast<int32_t*>(b + offsetof(pa_image_header, mma_next));
  return d;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D view of a pool: rows = num_pages * Hkv * P, columns = D bf16; box 64 x 16
// with 128-byte swizzle (one half of a (page, kv head) tile per copy).
bool encode_pool(const pa_plan& p, const void* pool, void* out) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)p.D, (cuuint64_t)p.num_pages_in_pool * p.Hkv * p.P};
  cuuint64_t strides[1] = {(cuuint64_t)p.D * 2};
  cuuint32_t box[2] = {64, 16};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(reinterpret_cast<CUtensorMap*>(out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pool),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Pinned staging buffers for plan uploads.  A copy from pageable memory makes
// the runtime wait for the stream first, which would serialise host planning
// with the device work of the previous step; a copy from pinned memory does
// not.  Each device has a ring of kPinSlots buffers used round-robin; before a
// slot is reused the host waits for the event recorded after its last copy, so
// the host can run at most kPinSlots uploads ahead of the device.
constexpr int kPinSlots = 8;
struct PinnedSlot {
  void* ptr = nullptr;
  size_t bytes = 0;
  cudaEvent_t done = nullptr;
  bool lent = false;  // holds a plan image being built, its copy not yet enqueued
};
struct PinnedRing {
  PinnedSlot slot[kPinSlots];
  int next = 0;
};
std::mutex g_pin_mu;
PinnedRing g_pin[64];

// Replaces the buffer of an idle slot by one of >= n bytes (a power of two, at
// least 64 KiB).
bool pin_grow(PinnedSlot& s, size_t n) {
  if (s.ptr) cudaFreeHost(s.ptr);
  s.ptr = nullptr;
  s.bytes = 0;
  size_t cap = 1 << 16;
  while (cap < n) cap <<= 1;
  if (cudaMallocHost(&s.ptr, cap) != cudaSuccess) {
    s.ptr = nullptr;
    return false;
  }
  s.bytes = cap;
  return true;
}

// Returns a free pinned slot of >= n bytes for the current device, or nullptr.
// A slot that must grow takes every idle slot with it: a pinned allocation
// costs a millisecond or more of host time, and paid one slot per step it
// would stall the steps that follow the first (the host has no lead on the
// device yet).
PinnedSlot* pin_acquire(size_t n, int device) {
  if (device < 0 || device >= 64) return nullptr;
  PinnedRing& r = g_pin[device];
  PinnedSlot& s = r.slot[r.next];
  if (s.lent) return nullptr;
  r.next = (r.next + 1) % kPinSlots;
  if (s.done && cudaEventSynchronize(s.done) != cudaSuccess) return nullptr;
  if (s.bytes < n) {
    if (!pin_grow(s, n)) return nullptr;
    for (PinnedSlot& o : r.slot)
      if (&o != &s && o.bytes < n && !o.lent && (!o.done || cudaEventQuery(o.done) == cudaSuccess)) pin_grow(o, n);
  }
  if (!s.done && cudaEventCreateWithFlags(&s.done, cudaEventDisableTiming) != cudaSuccess) return nullptr;
  return &s;
}

void record_profile(const pa_plan& p, int which, cudaStream_t st) {
  if (p.prof[which]) cudaEventRecord(static_cast<cudaEvent_t>(p.prof[which]), st);
}

// 3-D view of a pool for whole (page, kv head) tiles in one copy: dims (64
// dims, row, half of D) with strides (D * 2 bytes per row, 128 bytes per half);
// box 64 x 16 x 2 with 128-byte swizzle lands as two 16-row x 128-byte boxes,
// the second 2 KB after the first (the layout of two 2-D copies).  Only for
// D = 128; returns false when the driver refuses the view.
bool encode_pool_tiles(const pa_plan& p, const void* pool, void* out) {
  auto fn = encode_fn();
  if (!fn || p.D != 128) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)p.num_pages_in_pool * p.Hkv * p.P, 2};
  cuuint64_t strides[2] = {(cuuint64_t)p.D * 2, 128};
  cuuint32_t box[3] = {64, 16, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(reinterpret_cast<CUtensorMap*>(out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Encoded tensor maps, cached process-wide by (pool pointer, rows, head dim,
// view): a pool keeps its maps for every plan that reads it.
struct TmapEntry {
  const void* ptr = nullptr;
  uint64_t rows = 0;
  int D = 0;
  int view = 0;  // 0: 2-D rows x D; 1: 3-D whole tiles; -1 (in `ok`): refused
  bool ok = false;
  alignas(64) uint8_t map[128];
};
std::mutex g_tmap_mu;
TmapEntry g_tmap[128];  // enough for both pools of every layer of a large model
int g_tmap_next = 0;

bool tmap_get(const pa_plan& p, const void* pool, void* out, int view = 0) {
  const uint64_t rows = (uint64_t)p.num_pages_in_pool * p.Hkv * p.P;
  std::lock_guard<std::mutex> lock(g_tmap_mu);
  for (const TmapEntry& e : g_tmap)
    if (e.ptr == pool && e.rows == rows && e.D == p.D && e.view == view) {
      if (e.ok) std::memcpy(out, e.map, 128);
      return e.ok;
    }
  TmapEntry& e = g_tmap[g_tmap_next];
  e.ok = view == 0 ? encode_pool(p, pool, e.map) : encode_pool_tiles(p, pool, e.map);
  e.ptr = pool;
  e.rows = rows;
  e.D = p.D;
  e.view = view;
  g_tmap_next = (g_tmap_next + 1) % (int)(sizeof(g_tmap) / sizeof(g_tmap[0]));
  if (e.ok) std::memcpy(out, e.map, 128);
  return e.ok;
}

}  // namespace

extern "C" pa_status pa_plan_upload(const pa_plan* plan, void* d_workspace, size_t bytes, void* stream) {
  if (!plan || !d_workspace) return PA_ERR_INVALID;
  if (bytes < plan->hdr.workspace_bytes) return PA_ERR_NOMEM;
  if (reinterpret_cast<uintptr_t>(d_workspace) & 255) return PA_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return PA_ERR_CUDA;
  // from here on the plan's image is the copy at the workspace base (a plan
  // that pa_decode_step returned stops referring to the library's slot)
  plan->dev_image = nullptr;
  std::lock_guard<std::mutex> lock(g_pin_mu);
  PinnedSlot* s = pin_acquire(plan->image.size, device);
  if (!s) {
    // no pinned memory: a pageable copy is still correct, only slower
    cudaError_t e = cudaMemcpyAsync(d_workspace, plan->image.data(), plan->image.size, cudaMemcpyHostToDevice, st);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }
  std::memcpy(s->ptr, plan->image.data(), plan->image.size);
  cudaError_t e = cudaMemcpyAsync(d_workspace, s->ptr, plan->image.size, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  if (cudaEventRecord(s->done, st) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

extern "C" pa_status pa_plan_set_profile_events(pa_plan* plan, void* const* events, int32_t n) {
  if (!plan || n < 0 || n > 4 || (n > 0 && !events)) return PA_ERR_INVALID;
  for (int i = 0; i < 4; ++i) plan->prof[i] = i < n ? events[i] : nullptr;
  return PA_OK;
}

namespace {

pa_status launch(const pa_plan* plan, const void* q, const void* k_pool, const void* v_pool, void* d_workspace,
                 void* out, float* lse, void* stream) {
  if (!plan || !q || !k_pool || !v_pool || !d_workspace) return PA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(k_pool) | reinterpret_cast<uintptr_t>(v_pool) |
       reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15)
    return PA_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(d_workspace) & 255) return PA_ERR_INVALID;
  PaDevPtrs d = dev_ptrs(*plan, d_workspace);
  d.q = static_cast<const uint16_t*>(q);
  d.k_pool = static_cast<const uint16_t*>(k_pool);
  d.v_pool = static_cast<const uint16_t*>(v_pool);
  if (plan->tma_k_ptr != k_pool || plan->tma_v_ptr != v_pool) {
    if (!tmap_get(*plan, k_pool, plan->tma_k) || !tmap_get(*plan, v_pool, plan->tma_v)) return PA_ERR_CUDA;
    // whole-tile maps for the small-row class when the driver takes them
    plan->tma_tiles = tmap_get(*plan, k_pool, plan->tma_k3, 1) && tmap_get(*plan, v_pool, plan->tma_v3, 1);
    plan->tma_k_ptr = k_pool;
    plan->tma_v_ptr = v_pool;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  record_profile(*plan, 0, st);
  if (pa_launch_forward(*plan, d, out, lse, stream) != 0) return PA_ERR_CUDA;
  if (out && plan->hdr.num_tail_pairs > 0 && pa_launch_tail_merge(*plan, d, out, lse, stream) != 0) return PA_ERR_CUDA;
  record_profile(*plan, 1, st);
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_forward(const pa_plan* plan, const void* q, const void* k_pool, const void* v_pool,
                                void* d_workspace, void* stream) {
  return launch(plan, q, k_pool, v_pool, d_workspace, nullptr, nullptr, stream);
}

extern "C" pa_status pa_merge(const pa_plan* plan, void* d_workspace, void* out, float* lse, void* stream) {
  if (!plan || !d_workspace || !out) return PA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(out) & 15) || (reinterpret_cast<uintptr_t>(d_workspace) & 255))
    return PA_ERR_INVALID;
  PaDevPtrs d = dev_ptrs(*plan, d_workspace);
  record_profile(*plan, 2, static_cast<cudaStream_t>(stream));
  const int e = pa_launch_merge(*plan, d, out, lse, stream);
  record_profile(*plan, 3, static_cast<cudaStream_t>(stream));
  return e == 0 ? PA_OK : PA_ERR_CUDA;
}

extern "C" pa_status pa_merge_f32(const pa_plan* plan, void* d_workspace, float* out, float* lse, void* stream) {
  if (!plan || !d_workspace || !out) return PA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(out) & 15) || (reinterpret_cast<uintptr_t>(d_workspace) & 255))
    return PA_ERR_INVALID;
  PaDevPtrs d = dev_ptrs(*plan, d_workspace);
  record_profile(*plan, 2, static_cast<cudaStream_t>(stream));
  const int e = pa_launch_merge(*plan, d, out, lse, stream, true);
  record_profile(*plan, 3, static_cast<cudaStream_t>(stream));
  return e == 0 ? PA_OK : PA_ERR_CUDA;
}

extern "C" pa_status pa_merge_rows(int32_t n_parts, int32_t rows_per_part, int32_t batch, int32_t num_q_heads,
                                   int32_t head_dim, const int32_t* d_part_req, const float* d_part_o,
                                   const float* d_part_lse, void* out, float* lse, void* stream) {
  if (n_parts < 1 || rows_per_part < 1 || batch < 1 || num_q_heads < 1 || !d_part_req || !d_part_o || !d_part_lse ||
      !out)
    return PA_ERR_INVALID;
  if (!(head_dim == 64 || head_dim == 128)) return PA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(d_part_o) | reinterpret_cast<uintptr_t>(out)) & 15) return PA_ERR_INVALID;
  const int e = pa_launch_merge_rows(n_parts, rows_per_part, batch, num_q_heads, head_dim, d_part_req, d_part_o,
                                     d_part_lse, out, lse, stream);
  return e == 0 ? PA_OK : PA_ERR_CUDA;
}

extern "C" pa_status pa_attend(const pa_plan* plan, const void* q, const void* k_pool, const void* v_pool,
                               void* d_workspace, void* out, float* lse, void* stream) {
  if (!out) return PA_ERR_INVALID;
  return launch(plan, q, k_pool, v_pool, d_workspace, out, lse, stream);
}

pa_status pa_attend_ws(const pa_plan* plan, const void* q, const void* k_pool, const void* v_pool, void* ws,
                       void* out, float* lse, void* stream) {
  return pa_attend(plan, q, k_pool, v_pool, ws, out, lse, stream);
}

extern "C" pa_status pa_get_device_status(const pa_plan* plan, const void* d_workspace, void* stream,
                                          pa_status* out) {
  if (!plan || !out) return PA_ERR_INVALID;
  int32_t word = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // NULL workspace: the static array of pa_attend_noalloc
  const void* ws = d_workspace ? d_workspace : pa_noalloc_scratch();
  if (!ws) return PA_ERR_CUDA;
  const uint8_t* base = static_cast<const uint8_t*>(d_workspace && plan->dev_image ? plan->dev_image : ws);
  const uint8_t* src = base + offsetof(pa_image_header, status);
  if (cudaMemcpyAsync(&word, src, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
  *out = static_cast<pa_status>(word);
  return PA_OK;
}

namespace {

// Per-step plan images of pa_decode_step: the two halves of the caller's image
// buffer, used alternately and uploaded on a stream of the library's own so
// that the upload of step k+1 runs while the kernels of step k do.  The compute
// stream waits for the upload (an event) before its launches, and records when
// it has finished reading the slot; the upload that next fills the slot waits
// for that.  Images of at most kStepInlineImageBytes are copied on the compute
// stream itself instead: in stream order after the kernels that last read the
// slot and before the step's launches, with no event to wait on, so the host
// makes three fewer calls per step for a copy on the device's timeline (one
// box, decode-step loops: config 1's 3.8 KB image 21-24 -> 19-22 us per step;
// config 2's 78 KB one 53-56 -> 55-60 us, so it keeps the copy stream).  The library
// holds only the copy stream and the events (per device); the device memory
// is the caller's.
constexpr size_t kStepInlineImageBytes = 16 << 10;
struct StepRing {
  cudaStream_t upload = nullptr;
  cudaEvent_t uploaded[2] = {nullptr, nullptr}, consumed[2] = {nullptr, nullptr};
  bool consumed_set[2] = {false, false};
  int next = 0;
};
std::mutex g_step_mu;
StepRing g_step[64];

StepRing* step_ring(int& device) {
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= 64) return nullptr;
  StepRing& r = g_step[device];
  if (!r.upload) {
    if (cudaStreamCreateWithFlags(&r.upload, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    for (int j = 0; j < 2; ++j)
      if (cudaEventCreateWithFlags(&r.uploaded[j], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&r.consumed[j], cudaEventDisableTiming) != cudaSuccess)
        return nullptr;
  }
  return &r;
}

// Uploads the plan image into the next half of the caller's image buffer and
// makes `stream` wait for it; the plan's kernels then read their tables there.
// pa_decode_step has the planner write the image straight into a pinned
// staging buffer (no second copy); the buffer stays lent until its copy is
// enqueued.
struct ImageInPinned {
  int device = 0;
  PinnedSlot* slot = nullptr;
};
uint8_t* pinned_image_sink(size_t n, void* ctx) {
  ImageInPinned* c = static_cast<ImageInPinned*>(ctx);
  std::lock_guard<std::mutex> lock(g_pin_mu);
  PinnedSlot* s = pin_acquire(n, c->device);
  if (!s) return nullptr;
  s->lent = true;
  c->slot = s;
  return static_cast<uint8_t*>(s->ptr);
}
void pinned_image_return(ImageInPinned& c) {
  std::lock_guard<std::mutex> lock(g_pin_mu);
  if (c.slot) c.slot->lent = false;
  c.slot = nullptr;
}

pa_status step_upload(pa_plan* plan, cudaStream_t stream, uint8_t* images, size_t half, int* slot_out,
                      ImageInPinned* pinned) {
  std::lock_guard<std::mutex> lock(g_step_mu);
  int device = 0;
  StepRing* r = step_ring(device);
  if (!r) return PA_ERR_CUDA;
  const int j = r->next;
  const size_t n = plan->image.size;
  if (n > half) return PA_ERR_NOMEM;
  void* dst = images + (size_t)j * half;
  const bool on_stream = n <= kStepInlineImageBytes;
  cudaStream_t cs = on_stream ? stream : r->upload;
  if (!on_stream && r->consumed_set[j] && cudaStreamWaitEvent(r->upload, r->consumed[j], 0) != cudaSuccess)
    return PA_ERR_CUDA;
  {
    std::lock_guard<std::mutex> pin_lock(g_pin_mu);
    PinnedSlot* lent = pinned && pinned->slot && pinned->slot->ptr == plan->image.data() ? pinned->slot : nullptr;
    PinnedSlot* s = lent ? nullptr : pin_acquire(n, device);
    if (lent) {
      // the image was built in this pinned buffer
      const cudaError_t e1 = cudaMemcpyAsync(dst, lent->ptr, n, cudaMemcpyHostToDevice, cs);
      const cudaError_t e2 = e1 == cudaSuccess ? cudaEventRecord(lent->done, cs) : e1;
      lent->lent = false;
      pinned->slot = nullptr;
      if (e2 != cudaSuccess) return PA_ERR_CUDA;
    } else if (s) {
      std::memcpy(s->ptr, plan->image.data(), n);
      if (cudaMemcpyAsync(dst, s->ptr, n, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
          cudaEventRecord(s->done, cs) != cudaSuccess)
        return PA_ERR_CUDA;
    } else if (cudaMemcpyAsync(dst, plan->image.data(), n, cudaMemcpyHostToDevice, cs) != cudaSuccess) {
      return PA_ERR_CUDA;
    }
  }
  if (!on_stream && (cudaEventRecord(r->uploaded[j], r->upload) != cudaSuccess ||
                     cudaStreamWaitEvent(stream, r->uploaded[j], 0) != cudaSuccess))
    return PA_ERR_CUDA;
  plan->dev_image = dst;
  r->next = j ^ 1;
  *slot_out = j;
  return PA_OK;
}

// After the launches of the step: the slot may be refilled once `stream` gets here.
pa_status step_release(int j, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_step_mu);
  int device = 0;
  StepRing* r = step_ring(device);
  if (!r) return PA_ERR_CUDA;
  if (cudaEventRecord(r->consumed[j], stream) != cudaSuccess) return PA_ERR_CUDA;
  r->consumed_set[j] = true;
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_step(const pa_config* cfg, int32_t batch, const int32_t* kv_lens,
                                    const int32_t* block_table, int32_t max_pages, int32_t num_pages_in_pool,
                                    const void* q, const void* k_pool, const void* v_pool, void* d_workspace,
                                    size_t workspace_bytes, void* d_images, size_t images_bytes, void* out,
                                    float* lse, void* const* profile_events, void* stream, pa_plan** plan_out) {
  if (plan_out) *plan_out = nullptr;
  if (!d_images || (reinterpret_cast<uintptr_t>(d_images) & 255)) return PA_ERR_INVALID;
  const size_t half = (images_bytes / 2) & ~size_t(255);
  if (half == 0) return PA_ERR_NOMEM;
  pa_plan* plan = nullptr;
  ImageInPinned pinned;
  if (cudaGetDevice(&pinned.device) != cudaSuccess) return PA_ERR_CUDA;
  pa_set_image_sink(pinned_image_sink, &pinned);
  pa_status st = pa_plan_create(cfg, batch, kv_lens, block_table, max_pages, num_pages_in_pool, &plan);
  pa_set_image_sink(nullptr, nullptr);
  if (st != PA_OK) {
    pinned_image_return(pinned);
    return st;
  }
  if (profile_events) pa_plan_set_profile_events(plan, profile_events, 4);
  if (workspace_bytes < plan->hdr.workspace_bytes) st = PA_ERR_NOMEM;
  int slot = -1;
  if (st == PA_OK)
    st = step_upload(plan, static_cast<cudaStream_t>(stream), static_cast<uint8_t*>(d_images), half, &slot, &pinned);
  pinned_image_return(pinned);  // no-op once the copy was enqueued
  if (st == PA_OK) st = pa_attend(plan, q, k_pool, v_pool, d_workspace, out, lse, stream);
  if (slot >= 0) {
    const pa_status rs = step_release(slot, static_cast<cudaStream_t>(stream));
    if (st == PA_OK) st = rs;
  }
  if (st == PA_OK && plan_out && !plan->image.owned) {
    // the caller keeps the plan: give it its own copy of the image (the pinned
    // buffer goes back to the staging ring)
    try {
      HostBuf own = hostbuf_acquire(plan->image.size);
      std::memcpy(own.data(), plan->image.data(), plan->image.size);
      plan->image = own;
    } catch (...) {
      pa_plan_destroy(plan);
      return PA_ERR_NOMEM;
    }
  }
  if (st == PA_OK && plan_out) *plan_out = plan;
  else pa_plan_destroy(plan);
  return st;
}

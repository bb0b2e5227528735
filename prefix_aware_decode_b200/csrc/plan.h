// Internal definition of the host plan object and the kernel launch entry points.
#pragma once

#include <cstdint>
#include <vector>

#include "pa.h"

static_assert(sizeof(pa_seg) == 32, "pa_seg must be 32 bytes (vector loads)");
static_assert(sizeof(pa_item) == 16, "pa_item must be 16 bytes");

// Forward launch shapes, one CTA per SM for both classes.  A CUDA-core (SIMT)
// CTA runs 8 independent warps; a tensor-core (MMA) CTA runs 8 consumer warps
// of 16 rows each (128 rows) and one producer warp.
constexpr int kSimtWarpsPerCta = 8;
constexpr int kMmaRowsPerCta = 128;

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
  std::vector<uint8_t> image;  // exactly what pa_plan_upload sends
  // cached TMA descriptors (encoded for the last pool pointers seen)
  mutable const void* tma_k_ptr = nullptr;
  mutable const void* tma_v_ptr = nullptr;
  alignas(64) mutable uint8_t tma_k[128] = {};
  alignas(64) mutable uint8_t tma_v[128] = {};
  // optional cudaEvent_t handles recorded around the launches (profiling):
  // [0,1] forward launch (pa_forward / pa_attend), [2,3] merge launch
  void* prof[4] = {};
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
  const int32_t* warp_loads;
  const int32_t* tiles;
  const int32_t* prow_off;
  float* partial_lse;
  float* partial_o;
  int32_t* status;
};

// out == nullptr: partial rows only; else the merge is fused into the launches.
// The two classes run as two kernels; `side` is a second stream that the
// caller has made wait for `stream` (the MMA kernel goes there).
int pa_launch_forward_mma(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* side);
int pa_launch_forward_simt(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream);
int pa_launch_merge(const pa_plan& p, const PaDevPtrs& d, void* out, float* lse, void* stream);

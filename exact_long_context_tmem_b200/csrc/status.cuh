// Device-side status word and wait limit shared by every kernel of the library.
// The library is one CUDA translation unit, so these globals exist once per device.
#pragma once

#include <cstdint>

namespace attn {

enum DeviceErrorCode : uint32_t {
  ATTN_DEV_OK = 0,
  ATTN_DEV_TIMEOUT = 1,  // a bounded wait ran out
  ATTN_DEV_BAD_PAGE = 2,  // a decode page-table entry outside [0, num_pages)
};

// Wait sites, recorded with the error so a timeout names the wait that gave up.
enum WaitSite : int {
  SITE_PROBE = 1,
  SITE_PF_LOAD_EMPTY = 10,
  SITE_PF_MMA_Q = 11,
  SITE_PF_MMA_K = 12,
  SITE_PF_MMA_V = 13,
  SITE_PF_MMA_P = 14,
  SITE_PF_SM_S = 15,
  SITE_PF_EPI_O = 16,
  SITE_PF_DRAIN = 17,
  SITE_DC_LOAD_EMPTY = 30,
  SITE_DC_MMA_K = 31,
  SITE_DC_MMA_V = 32,
  SITE_DC_MMA_P = 33,
  SITE_DC_SM_S = 34,
  SITE_DC_SM_O = 35,
  SITE_DC_SM_V = 36,
  SITE_DC_DRAIN = 37,
  SITE_DC_SM_K = 38,
  SITE_DC_MMA_POLL = 39,
  SITE_DC_Q = 40,
  SITE_DC_MMA_O = 41,
  SITE_DC_MMA_S = 42,
  SITE_DC_SM_P = 43,
  SITE_DC_PAGE = 44,
};

// (code << 16) | site of the first error since the last reset; 0 when clean.
__device__ uint32_t g_dev_status = 0;
// Upper bound for any single mbarrier wait, in nanoseconds of %globaltimer.
__device__ uint64_t g_wait_limit_ns = 2000000000ull;

__device__ __forceinline__ void record_device_error(uint32_t code, int site) {
  atomicCAS(&g_dev_status, 0u, (code << 16) | (uint32_t)(site & 0xFFFF));
}

__device__ __forceinline__ bool device_error_set() {
  return *reinterpret_cast<volatile uint32_t*>(&g_dev_status) != 0u;
}

// Optional progress trace for diagnosing a stalled kernel (compiled in only with -DATTN_TRACE):
// each role writes (stage << 16 | iteration) into host-mapped memory that the host can read
// while the kernel is still running.
#ifdef ATTN_TRACE
__device__ uint32_t* g_trace = nullptr;
#define ATTN_TRACE_AT(slot, stage, iter)                                                  \
  do {                                                                                    \
    volatile uint32_t* t_ = g_trace;                                                      \
    if (t_) {                                                                             \
      t_[blockIdx.x * 16 + (slot)] = ((uint32_t)(stage) << 16) | ((uint32_t)(iter) & 0xFFFFu); \
      __threadfence_system();                                                             \
    }                                                                                     \
  } while (0)
#else
#define ATTN_TRACE_AT(slot, stage, iter) \
  do {                                   \
  } while (0)
#endif

// Optional cycle profile (compiled in only with -DATTN_PROF): roles add clock64() spans per
// category into a device buffer of 64 counters that the host reads after the kernel.
#ifdef ATTN_PROF
__device__ unsigned long long* g_prof = nullptr;
#define ATTN_PROF_DECL(name) long long name = 0
#define ATTN_PROF_T0(v) const long long v = clock64()
#define ATTN_PROF_ADD(acc, t0) (acc) += clock64() - (t0)
#define ATTN_PROF_FLUSH(slot, acc)                                    \
  do {                                                                \
    if (g_prof) atomicAdd(g_prof + (slot), (unsigned long long)(acc)); \
  } while (0)
// Event timeline of CTA 0: clock64() of event `kind` (< 16) for tile `tile` (< 64).  The buffer
// pointer is read once per thread (ATTN_EVT_INIT), so an event costs one store.
__device__ long long* g_evt = nullptr;
#define ATTN_EVT_INIT() long long* const evt_base_ = (blockIdx.x == 0) ? g_evt : nullptr
#define ATTN_EVT(tile, kind)                                                      \
  do {                                                                            \
    if (evt_base_ && (tile) < 64) evt_base_[(tile) * 16 + (kind)] = clock64();    \
  } while (0)
#else
#define ATTN_PROF_DECL(name)
#define ATTN_PROF_T0(v)
#define ATTN_PROF_ADD(acc, t0)
#define ATTN_PROF_FLUSH(slot, acc)
#define ATTN_EVT_INIT()
#define ATTN_EVT(tile, kind)
#endif

}  // namespace attn

// Shared host/device helpers of the PBSA library: status handling, argument
// checks, bf16 helpers, order-preserving sort keys and the bounded wait.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string>

#include "../../include/pbsa.h"

namespace pbsa {

// ---------------------------------------------------------------- host side
void set_error(const std::string& msg);
int* device_status_ptr();           // address of this device's status word
int debug_flags();
int64_t wait_limit_ns();

#define PBSA_CHECK_ARG(cond, code, msg)            \
  do {                                             \
    if (!(cond)) {                                 \
      ::pbsa::set_error(msg);                      \
      return (code);                               \
    }                                              \
  } while (0)

#define PBSA_CHECK_LAUNCH(what)                                              \
  do {                                                                       \
    cudaError_t e_ = cudaGetLastError();                                     \
    if (e_ != cudaSuccess) {                                                 \
      ::pbsa::set_error(std::string(what) + ": " + cudaGetErrorString(e_));  \
      return PBSA_ERR_CUDA;                                                  \
    }                                                                        \
  } while (0)

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int common_dims_check(const pbsa_dims* d) {
  PBSA_CHECK_ARG(d != nullptr, PBSA_ERR_ARG, "dims is NULL");
  PBSA_CHECK_ARG(d->B >= 1 && d->H >= 1, PBSA_ERR_SHAPE, "B and H must be >= 1");
  PBSA_CHECK_ARG(d->D == 64 || d->D == 128, PBSA_ERR_SHAPE, "D must be 64 or 128");
  PBSA_CHECK_ARG(d->bs == 64 || d->bs == 128, PBSA_ERR_SHAPE, "bs must be 64 or 128");
  PBSA_CHECK_ARG(d->dtype == PBSA_BF16 || d->dtype == PBSA_FP32, PBSA_ERR_DTYPE,
                 "dtype must be PBSA_BF16 or PBSA_FP32");
  PBSA_CHECK_ARG(d->q_chunk >= 0, PBSA_ERR_SHAPE, "q_chunk must be >= 0");
  return PBSA_OK;
}

// Query rows are chunks of qc rows (qc <= 0: one chunk), each tiled into
// blocks of bs rows on its own.
__host__ __device__ inline int qb_count(int Tq, int qc, int bs) {
  qc = qc > 0 ? qc : Tq;
  const int per = (qc + bs - 1) / bs;
  const int full = Tq / qc;
  const int rem = Tq - full * qc;
  return full * per + (rem + bs - 1) / bs;
}
__host__ __device__ inline void qb_rows(int i, int Tq, int qc, int bs, int& row0, int& len) {
  qc = qc > 0 ? qc : Tq;
  const int per = (qc + bs - 1) / bs;
  const int c = i / per, b = i - c * per;
  const int crow = c * qc;
  const int clen = min(qc, Tq - crow);
  row0 = crow + b * bs;
  len = min(bs, clen - b * bs);
}

inline size_t elem_size(int dtype) { return dtype == PBSA_BF16 ? 2 : 4; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// -------------------------------------------------------------- device side
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Map a float to a uint32 whose unsigned order is the float order.
__device__ __forceinline__ uint32_t orderable(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 64-bit sort key: score descending, then id ascending, under a DESCENDING sort.
__device__ __forceinline__ uint64_t score_key(float s, uint32_t id) {
  return (static_cast<uint64_t>(orderable(s)) << 32) | static_cast<uint64_t>(0xffffffffu - id);
}
__device__ __forceinline__ uint32_t key_id(uint64_t k) {
  return 0xffffffffu - static_cast<uint32_t>(k & 0xffffffffu);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

// Programmatic dependent launch.  Every library kernel is launched with the
// programmatic-serialisation attribute (see launch.h), so its CTAs may start
// while the previous kernel on the stream is still running.  pdl_wait() blocks
// until that kernel has completed and its memory is visible; every kernel calls
// it before its first global-memory access.  pdl_trigger() lets the next
// kernel's CTAs be scheduled once every CTA of this grid has started.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Warp-wide bitonic sort of 32*KPL 64-bit keys, DESCENDING.  Element e of the
// virtual array lives in lane (e / KPL), register (e % KPL).
template <int KPL>
__device__ __forceinline__ void warp_bitonic_sort_desc(uint64_t (&v)[KPL]) {
  const int lane = threadIdx.x & 31;
  constexpr int N = 32 * KPL;
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= KPL) {
        const int lane_stride = stride / KPL;
#pragma unroll
        for (int r = 0; r < KPL; ++r) {
          const int e = lane * KPL + r;
          uint64_t other = __shfl_xor_sync(0xffffffffu, v[r], lane_stride);
          const bool desc_block = ((e & size) == 0);   // this run sorts descending
          const bool lower = ((e & stride) == 0);
          // keep max at lower index for a descending run
          const bool take_max = (lower == desc_block);
          const uint64_t mx = v[r] > other ? v[r] : other;
          const uint64_t mn = v[r] > other ? other : v[r];
          v[r] = take_max ? mx : mn;
        }
      } else {
#pragma unroll
        for (int r = 0; r < KPL; ++r) {
          const int partner = r ^ stride;
          if (partner > r) {
            const int e = lane * KPL + r;
            const bool desc_block = ((e & size) == 0);
            const uint64_t a = v[r], b = v[partner];
            const bool swap = desc_block ? (a < b) : (a > b);
            v[r] = swap ? b : a;
            v[partner] = swap ? a : b;
          }
        }
      }
    }
  }
}

}  // namespace pbsa

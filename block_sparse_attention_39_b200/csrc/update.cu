// a3: persistent-memory update as three kernels per call: one plan CTA per
// (b,h), then (merge policy only) a stash CTA and an apply CTA per (slot, b,h).
// The device code is in update_dev.cuh.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "update_dev.cuh"

namespace pbsa {
namespace {

using namespace dev;

__global__ void __launch_bounds__(256) update_plan_kernel(UpdArgs a) {
  __shared__ PlanSmem sm;
  extern __shared__ __align__(16) float sk[];   // [P][D] kept pooled keys (merge policy)
  pdl_wait();
  pdl_trigger();
  plan_head(a, blockIdx.x, sm, sk);
}

template <typename T>
__global__ void __launch_bounds__(256)
update_stash_kernel(UpdArgs a, const T* __restrict__ kpool, const T* __restrict__ vpool,
                    T* __restrict__ stash) {
  pdl_wait();
  pdl_trigger();
  stash_item<T>(a, static_cast<int>(blockIdx.x), blockIdx.y, kpool, vpool, stash);
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
update_apply_kernel(UpdArgs a, T* __restrict__ kpool, T* __restrict__ vpool,
                    const T* __restrict__ stash, int32_t* __restrict__ blk_len,
                    int32_t* __restrict__ blk_pos, float* __restrict__ k_bar,
                    int32_t* __restrict__ slot_src, float* __restrict__ slot_w) {
  __shared__ float red[8][D];
  __shared__ int s_mref[kMaxItems], s_mlen[kMaxItems];
  __shared__ float s_mw[kMaxItems];
  pdl_wait();
  pdl_trigger();
  apply_item<T, D>(a, static_cast<int>(blockIdx.x), blockIdx.y, kpool, vpool, stash, blk_len,
                   blk_pos, k_bar, slot_src, slot_w, red, s_mref, s_mlen, s_mw);
}

template <typename T, int D>
cudaError_t launch_apply(const UpdArgs& a, void* kpool, void* vpool, const void* stash,
                         int32_t* blk_len, int32_t* blk_pos, float* k_bar, int32_t* slot_src,
                         float* slot_w, cudaStream_t s) {
  dim3 grid(a.P, a.B * a.H);
  if (a.policy == PBSA_MERGE_MEAN) {
    cudaError_t e = launch(update_stash_kernel<T>, grid, dim3(256), 0, s, a,
                           static_cast<const T*>(kpool), static_cast<const T*>(vpool),
                           static_cast<T*>(const_cast<void*>(stash)));
    if (e != cudaSuccess) return e;
  }
  return launch(update_apply_kernel<T, D>, grid, dim3(256), 0, s, a, static_cast<T*>(kpool),
                static_cast<T*>(vpool), static_cast<const T*>(stash), blk_len, blk_pos, k_bar,
                slot_src, slot_w);
}

}  // namespace
}  // namespace pbsa

extern "C" size_t pbsa_update_memory_workspace(const pbsa_dims* d, int P, int n_cand) {
  using namespace pbsa;
  if (d == nullptr || P < 1 || n_cand < 0 || d->B < 1 || d->H < 1) return 0;
  const int M = P + n_cand;
  return static_cast<size_t>(d->B) * d->H * plan_bytes(P, M) + stash_bytes(d, P);
}

extern "C" int pbsa_update_memory(const pbsa_dims* d, void* kpool, void* vpool, int NB,
                                  int32_t* blk_len, int32_t* blk_pos, float* k_bar, int P,
                                  int n_sink, int32_t* slot_src, float* slot_w,
                                  const int32_t* cand_ids, const int32_t* cand_src, int n_cand,
                                  const float* mem_score, int policy, void* workspace,
                                  size_t ws_bytes, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(kpool && vpool && blk_len && blk_pos && k_bar && slot_src && slot_w && mem_score,
                 PBSA_ERR_ARG, "update_memory: NULL buffer");
  PBSA_CHECK_ARG(n_cand >= 0 && (n_cand == 0 || (cand_ids && cand_src)), PBSA_ERR_ARG,
                 "update_memory: candidate lists are NULL");
  PBSA_CHECK_ARG(P >= 1 && P <= 256 && NB >= P, PBSA_ERR_SHAPE,
                 "update_memory: need 1 <= P <= 256 and NB >= P");
  PBSA_CHECK_ARG(n_sink >= 0 && n_sink <= P, PBSA_ERR_SHAPE, "update_memory: bad n_sink");
  PBSA_CHECK_ARG((P - n_sink) + n_cand <= kMaxItems, PBSA_ERR_SHAPE,
                 "update_memory: (P - n_sink) + n_cand must be <= 256");
  PBSA_CHECK_ARG(policy == PBSA_EVICT || policy == PBSA_MERGE_MEAN, PBSA_ERR_ARG,
                 "update_memory: bad policy");
  PBSA_CHECK_ARG(aligned(kpool, 16) && aligned(vpool, 16), PBSA_ERR_ALIGN,
                 "update_memory: kpool/vpool must be 16-byte aligned");
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "update_memory: B*H must be <= 65535");
  const size_t need = pbsa_update_memory_workspace(d, P, n_cand);
  PBSA_CHECK_ARG(workspace != nullptr && ws_bytes >= need && aligned(workspace, 256),
                 PBSA_ERR_WORKSPACE,
                 "update_memory: workspace missing, too small or not 256-byte aligned (need " +
                     std::to_string(need) + " bytes)");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "update_memory: no device status word");
  UpdArgs a;
  a.B = d->B; a.H = d->H; a.D = d->D; a.bs = d->bs; a.NB = NB; a.P = P; a.n_sink = n_sink;
  a.n_cand = n_cand; a.policy = policy; a.M = P + n_cand;
  a.blk_len = blk_len; a.blk_pos = blk_pos; a.k_bar = k_bar; a.slot_src = slot_src;
  a.slot_w = slot_w; a.cand_ids = cand_ids; a.cand_src = cand_src; a.mem = mem_score;
  a.ws = workspace; a.status = status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t plan_smem = policy == PBSA_MERGE_MEAN ? merge_key_smem(P, d->D) : 0;
  {
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
      cudaFuncSetAttribute(update_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(merge_key_smem(256, 128)));
      attr_set[dev] = true;
    }
  }
  if (launch(update_plan_kernel, dim3(d->B * d->H), dim3(256), plan_smem, s, a) != cudaSuccess)
    PBSA_CHECK_LAUNCH("update_plan_kernel");
  const void* stash =
      static_cast<const char*>(workspace) + static_cast<size_t>(d->B) * d->H * plan_bytes(P, a.M);
  cudaError_t e;
  if (d->dtype == PBSA_BF16) {
    if (d->D == 128)
      e = launch_apply<__nv_bfloat16, 128>(a, kpool, vpool, stash, blk_len, blk_pos, k_bar,
                                           slot_src, slot_w, s);
    else
      e = launch_apply<__nv_bfloat16, 64>(a, kpool, vpool, stash, blk_len, blk_pos, k_bar,
                                          slot_src, slot_w, s);
  } else {
    if (d->D == 128)
      e = launch_apply<float, 128>(a, kpool, vpool, stash, blk_len, blk_pos, k_bar, slot_src,
                                   slot_w, s);
    else
      e = launch_apply<float, 64>(a, kpool, vpool, stash, blk_len, blk_pos, k_bar, slot_src,
                                  slot_w, s);
  }
  if (e != cudaSuccess) PBSA_CHECK_LAUNCH("update_apply_kernel");
  return PBSA_OK;
}

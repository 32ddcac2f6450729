// Backward of a3, the persistent-memory update, for the key and value rows:
// the recurrent trainable path.
//
// Sparse Forcing trains with the dynamically updated cache (gist.science/es,
// section 2 "Entrenamiento"), and its memory learns to compress, keep and
// refresh persistent blocks (the abstract), so the loss reaches a block's keys
// and values also through the slots it was copied or merged into.  After an
// update every slot is a weighted row-wise sum of pre-update blocks, which the
// update's plan (update_dev.cuh) records:
//   op NONE   the slot keeps its content (identity);
//   op CLEAR  the slot is emptied (no term);
//   op WRITE  a copy of the base block (the whole block, weight 1), or the
//             merge  (bw * base[r < blen] + sum_m w_m * src_m[r < len_m]) / W
//             with W = bw + sum_m w_m; a merge source is a pool id or a stashed
//             pre-update slot (stash entry so = slot so before the update).
// The vector-Jacobian product is that sum transposed: every term (j, weight,
// rows) adds weight * dSlot[r] to d(pre-update block j)[r] for r < rows.  The
// selection and merge decisions are constants.  Each pre-update block appears
// in at most one term (a kept item is one slot's base, a loser one slot's
// merge source), so the scatter needs no atomics.
//
// Two kernels: update_bwd_stage_kernel copies every slot's incoming gradient
// to the workspace and clears the slots whose content the update replaced;
// update_bwd_scatter_kernel adds each written slot's terms.
#include <cuda_runtime.h>

#include <string>

#include "common.cuh"
#include "launch.h"
#include "update_dev.cuh"

namespace pbsa {
namespace {

using namespace dev;

struct BwdArgs {
  const void* plan;
  float* dk;
  float* dv;
  float* scratch;       // [BH][P][2][bs*D]
  int NB, P, M, bs, D;
};

__global__ void __launch_bounds__(256) update_bwd_stage_kernel(BwdArgs a) {
  pdl_wait();
  pdl_trigger();
  const int s = static_cast<int>(blockIdx.x);
  const long bh = blockIdx.y;
  const PlanView pv = plan_view(const_cast<void*>(a.plan), bh, a.P, a.M);
  const int op = pv.op[s];
  const long n4 = static_cast<long>(a.bs) * a.D / 4;
  float4* gk = reinterpret_cast<float4*>(a.dk + (bh * a.NB + s) * a.bs * static_cast<long>(a.D));
  float4* gv = reinterpret_cast<float4*>(a.dv + (bh * a.NB + s) * a.bs * static_cast<long>(a.D));
  float4* sk = reinterpret_cast<float4*>(a.scratch + ((bh * a.P + s) * 2 + 0) * n4 * 4);
  float4* sv = reinterpret_cast<float4*>(a.scratch + ((bh * a.P + s) * 2 + 1) * n4 * 4);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long e = threadIdx.x; e < n4; e += blockDim.x) {
    const float4 x = gk[e], y = gv[e];
    sk[e] = x;
    sv[e] = y;
    if (op != OP_NONE) {        // the slot's pre-update content gets only its terms
      gk[e] = z;
      gv[e] = z;
    }
  }
}

// rows [0, n) of block j += coef * (staged slot gradient)
__device__ __forceinline__ void add_term(const BwdArgs& a, long bh, int j, float coef, int n,
                                         const float* sk, const float* sv) {
  if (j < 0 || j >= a.NB || n <= 0) return;
  n = min(n, a.bs);
  const long n4 = static_cast<long>(n) * a.D / 4;
  float4* dk = reinterpret_cast<float4*>(a.dk + (bh * a.NB + j) * a.bs * static_cast<long>(a.D));
  float4* dv = reinterpret_cast<float4*>(a.dv + (bh * a.NB + j) * a.bs * static_cast<long>(a.D));
  const float4* gk = reinterpret_cast<const float4*>(sk);
  const float4* gv = reinterpret_cast<const float4*>(sv);
  for (long e = threadIdx.x; e < n4; e += blockDim.x) {
    float4 x = dk[e], y = dv[e];
    const float4 p = gk[e], q = gv[e];
    x.x = fmaf(coef, p.x, x.x); x.y = fmaf(coef, p.y, x.y);
    x.z = fmaf(coef, p.z, x.z); x.w = fmaf(coef, p.w, x.w);
    y.x = fmaf(coef, q.x, y.x); y.y = fmaf(coef, q.y, y.y);
    y.z = fmaf(coef, q.z, y.z); y.w = fmaf(coef, q.w, y.w);
    dk[e] = x;
    dv[e] = y;
  }
}

__global__ void __launch_bounds__(256) update_bwd_scatter_kernel(BwdArgs a) {
  pdl_wait();
  pdl_trigger();
  const int s = static_cast<int>(blockIdx.x);
  const long bh = blockIdx.y;
  const PlanView pv = plan_view(const_cast<void*>(a.plan), bh, a.P, a.M);
  if (pv.op[s] != OP_WRITE) return;
  const long n = static_cast<long>(a.bs) * a.D;
  const float* sk = a.scratch + ((bh * a.P + s) * 2 + 0) * n;
  const float* sv = a.scratch + ((bh * a.P + s) * 2 + 1) * n;
  const int m0 = pv.moff[s], m1 = pv.moff[s + 1];
  if (m0 == m1) {
    add_term(a, bh, pv.base[s], 1.f, a.bs, sk, sv);     // a copy: the whole block
    return;
  }
  // the weights as apply_item sums them: base first, then the list in order
  float wsum = pv.base_w[s];
  for (int m = m0; m < m1; ++m) wsum += pv.mw[m];
  const float inv = 1.f / wsum;
  add_term(a, bh, pv.base[s], pv.base_w[s] * inv, pv.base_len[s], sk, sv);
  for (int m = m0; m < m1; ++m) {
    const int ref = pv.mref[m];
    const int j = ref >= 0 ? ref : -(ref + 1);          // stash entry so: slot so before
    add_term(a, bh, j, pv.mw[m] * inv, pv.mlen[m], sk, sv);
  }
}

}  // namespace
}  // namespace pbsa

extern "C" size_t pbsa_update_plan_bytes(const pbsa_dims* d, int P, int n_cand) {
  if (d == nullptr || P < 1 || n_cand < 0 || d->B < 1 || d->H < 1) return 0;
  return static_cast<size_t>(d->B) * d->H * pbsa::dev::plan_bytes(P, P + n_cand);
}

extern "C" size_t pbsa_update_memory_bwd_workspace(const pbsa_dims* d, int P) {
  if (d == nullptr || P < 1 || d->B < 1 || d->H < 1) return 0;
  return pbsa::align_up(static_cast<size_t>(d->B) * d->H * P * 2 * d->bs * d->D * sizeof(float),
                        256);
}

extern "C" int pbsa_update_memory_bwd(const pbsa_dims* d, int NB, int P, int n_cand,
                                      const void* plan, float* dk, float* dv, void* workspace,
                                      size_t ws_bytes, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(plan && dk && dv, PBSA_ERR_ARG, "update_memory_bwd: NULL buffer");
  PBSA_CHECK_ARG(P >= 1 && P <= 256 && NB >= P && n_cand >= 0 && P + n_cand <= 512,
                 PBSA_ERR_SHAPE, "update_memory_bwd: need 1 <= P <= 256, NB >= P, n_cand >= 0");
  PBSA_CHECK_ARG(aligned(dk, 16) && aligned(dv, 16) && aligned(plan, 16), PBSA_ERR_ALIGN,
                 "update_memory_bwd: dk, dv and plan must be 16-byte aligned");
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "update_memory_bwd: B*H must be <= 65535");
  const size_t need = pbsa_update_memory_bwd_workspace(d, P);
  PBSA_CHECK_ARG(workspace != nullptr && ws_bytes >= need && aligned(workspace, 256),
                 PBSA_ERR_WORKSPACE,
                 "update_memory_bwd: workspace missing, too small or not 256-byte aligned (need " +
                     std::to_string(need) + " bytes)");
  BwdArgs a;
  a.plan = plan; a.dk = dk; a.dv = dv; a.scratch = static_cast<float*>(workspace);
  a.NB = NB; a.P = P; a.M = P + n_cand; a.bs = d->bs; a.D = d->D;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dim3 grid(P, d->B * d->H);
  if (launch(update_bwd_stage_kernel, grid, dim3(256), 0, s, a) != cudaSuccess)
    PBSA_CHECK_LAUNCH("update_bwd_stage_kernel");
  if (launch(update_bwd_scatter_kernel, grid, dim3(256), 0, s, a) != cudaSuccess)
    PBSA_CHECK_LAUNCH("update_bwd_scatter_kernel");
  return PBSA_OK;
}

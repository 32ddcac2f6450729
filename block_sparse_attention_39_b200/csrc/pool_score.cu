// a1 + a2: block pooling and coarse block scoring, as two kernels per call:
// a persistent pooling grid (two CTAs per SM) and one 64-thread scoring CTA
// per (b,h, 32 query blocks, 32 key blocks) tile of S.  The device code is in pool_score_dev.cuh.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "pool_score_dev.cuh"

namespace pbsa {
namespace {

using namespace dev;

template <typename T, int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(PoolArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_wait();
  pdl_trigger();
  pool_phase<T, D>(a, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x), smem);
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(ScoreArgs a) {
  extern __shared__ __align__(16) float ssm[];
  pdl_wait();
  pdl_trigger();
  const int n_jblk = (a.NB + kScoreTile - 1) / kScoreTile;
  const int x = static_cast<int>(blockIdx.x);
  score_item<D, kScoreTile>(a, blockIdx.y, x % n_jblk, x / n_jblk, ssm);
}

template <typename T, int D>
int launch_pool(PoolArgs a, cudaStream_t s) {
  a.stages = pool_stages<T, D>(a.bs);
  const size_t smem = pool_smem_bytes<T, D>(a.stages, a.bs);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaFuncSetAttribute(pool_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         200 * 1024);
    attr_set[dev] = true;
  }
  const int grid = max(1, min(a.n_items, kPoolCtasPerSm * sm_count()));
  cudaError_t e = launch(pool_kernel<T, D>, dim3(grid), dim3(kPoolThreads), smem, s, a);
  if (e != cudaSuccess) {
    set_error(std::string("pool_kernel: ") + cudaGetErrorString(e));
    return PBSA_ERR_CUDA;
  }
  return PBSA_OK;
}

template <int D>
int launch_score(const ScoreArgs& a, int BH, cudaStream_t s) {
  const size_t smem = score_smem_bytes<D, kScoreTile>();
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    // the whole unified L1 as shared memory, so that six 34 KB tiles fit per SM
    cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    attr_set[dev] = true;
  }
  dim3 grid(((a.NB + kScoreTile - 1) / kScoreTile) * ((a.nQB + kScoreTile - 1) / kScoreTile), BH);
  cudaError_t e = launch(score_kernel<D>, grid, dim3(kScoreThreads), smem, s, a);
  if (e != cudaSuccess) {
    set_error(std::string("score_kernel: ") + cudaGetErrorString(e));
    return PBSA_ERR_CUDA;
  }
  return PBSA_OK;
}

}  // namespace
}  // namespace pbsa

extern "C" int pbsa_score_blocks(const pbsa_dims* d, const void* q, int Tq, const void* kpool,
                                 int NB, const int32_t* blk_len, const int32_t* pool_ids,
                                 int n_pool, float* q_bar, float* k_bar, float* scores,
                                 float* mem_score, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(Tq >= 1 && NB >= 1 && n_pool >= 0, PBSA_ERR_SHAPE,
                 "score_blocks: need Tq >= 1, NB >= 1, n_pool >= 0");
  PBSA_CHECK_ARG(q && kpool && blk_len && q_bar && k_bar && scores && mem_score, PBSA_ERR_ARG,
                 "score_blocks: NULL buffer");
  PBSA_CHECK_ARG(n_pool == 0 || pool_ids, PBSA_ERR_ARG, "score_blocks: pool_ids is NULL");
  PBSA_CHECK_ARG(aligned(q, 16) && aligned(kpool, 16), PBSA_ERR_ALIGN,
                 "score_blocks: q and kpool must be 16-byte aligned");
  PBSA_CHECK_ARG(aligned(q_bar, 16) && aligned(k_bar, 16) && aligned(scores, 4) &&
                     aligned(mem_score, 4) && aligned(blk_len, 4),
                 PBSA_ERR_ALIGN,
                 "score_blocks: q_bar/k_bar must be 16-byte aligned, scores/mem 4-byte aligned");
  const int nQB = qb_count(Tq, d->q_chunk, d->bs);
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "score_blocks: B*H must be <= 65535");
  const long n_items = static_cast<long>(d->B) * d->H * (nQB + n_pool);
  PBSA_CHECK_ARG(n_items < (1L << 31), PBSA_ERR_SHAPE, "score_blocks: too many blocks to pool");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "score_blocks: no device status word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PoolArgs pa;
  pa.q = q; pa.kpool = kpool; pa.blk_len = blk_len; pa.pool_ids = pool_ids;
  pa.q_bar = q_bar; pa.k_bar = k_bar;
  pa.Tq = Tq; pa.qc = d->q_chunk; pa.NB = NB; pa.bs = d->bs; pa.nQB = nQB; pa.n_pool = n_pool;
  pa.n_items = static_cast<int>(n_items); pa.stages = 0;
  pa.status = status; pa.limit_ns = wait_limit_ns();
  if (d->dtype == PBSA_BF16)
    rc = d->D == 128 ? launch_pool<__nv_bfloat16, 128>(pa, s) : launch_pool<__nv_bfloat16, 64>(pa, s);
  else
    rc = d->D == 128 ? launch_pool<float, 128>(pa, s) : launch_pool<float, 64>(pa, s);
  if (rc) return rc;
  const int qc = d->q_chunk > 0 ? d->q_chunk : Tq;
  ScoreArgs sa;
  sa.q_bar = q_bar; sa.k_bar = k_bar; sa.scores = scores; sa.mem = mem_score;
  sa.nQB = nQB; sa.NB = NB;
  sa.per_group = (qc + d->bs - 1) / d->bs;
  sa.groups = (Tq + qc - 1) / qc;
  sa.scale = d->scale;
  return d->D == 128 ? launch_score<128>(sa, d->B * d->H, s) : launch_score<64>(sa, d->B * d->H, s);
}

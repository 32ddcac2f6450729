// a0: append one chunk's K and V to the block pool, pooling the keys in the
// same pass.
//
// The pooled key of a block is what the coarse scoring reads (gist.science/es,
// section 2, PBSA item "Compresión de Bloques"; item "Optimización" names
// selective cache updates as part of the kernel's job).  Computing it while the
// chunk is written into its blocks means the chunk's keys are read from HBM
// once; pbsa_score_blocks then only has to pool the query blocks.
//
// One persistent grid (two CTAs per SM) walks the items (b, h, block, K or V).
// Each item's rows are one contiguous run in the chunk tensor and in the
// destination block: an untiled bulk copy brings them into a shared-memory
// stage, an untiled bulk store writes them to the pool block, the padding rows
// of a partial block are zero-filled, and for a K item the rows are summed
// (row_sums / row_mean, the same code as pbsa_score_blocks' pooling, so the two
// give identical means) while the store drains.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "pool_score_dev.cuh"

namespace pbsa {
namespace {

using namespace dev;

struct AppendArgs {
  const void* k;
  const void* v;
  void* kpool;
  void* vpool;
  const int32_t* blk_ids;
  int32_t* blk_len;
  int32_t* blk_pos;
  float* k_bar;
  int Tc, pos0, NB, bs, nb, n_items, stages;
  int* status;
  int64_t limit_ns;
};

template <typename T, int D>
__global__ void __launch_bounds__(kPoolThreads) append_kernel(AppendArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_wait();
  pdl_trigger();
  constexpr int ROW = D * static_cast<int>(sizeof(T));
  const int S = a.stages;
  const int stage_bytes = a.bs * ROW;
  float* red = reinterpret_cast<float*>(smem + S * stage_bytes);        // [2][8][D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * 8 * D);         // [S]
  int* s_item = reinterpret_cast<int*>(bars + S);                        // [S] item of the stage
  volatile int* abort_flag = s_item + S;
  const int t = threadIdx.x;
  const int cta = static_cast<int>(blockIdx.x), G = static_cast<int>(gridDim.x);
  const int mine = a.n_items > cta ? (a.n_items - cta + G - 1) / G : 0;
  if (t == 0) {
    for (int s = 0; s < S; ++s) mbar_init(smem_u32(&bars[s]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // item it = ((b*H + h) * nb + block) * 2 + (0: K, 1: V)
  auto rows_of = [&](int it, int& blk, int& id, int& n) -> long {
    const long bh = it / (2 * a.nb);
    blk = (it >> 1) % a.nb;
    id = a.blk_ids[blk];
    n = min(a.bs, a.Tc - blk * a.bs);
    return bh;
  };
  auto issue = [&](int k) {             // thread 0: item k of this CTA into stage k % S
    const int s = k % S;
    const int it = cta + k * G;
    int blk, id, n;
    const long bh = rows_of(it, blk, id, n);
    s_item[s] = it;
    const uint32_t bar = smem_u32(&bars[s]);
    if (id < 0 || id >= a.NB) {
      report_status(a.status, PBSA_ERR_ARG);
      mbar_arrive(bar);
      return;
    }
    const T* src = static_cast<const T*>((it & 1) ? a.v : a.k) +
                   (bh * a.Tc + static_cast<long>(blk) * a.bs) * D;
    mbar_expect_tx(bar, static_cast<uint32_t>(n * ROW));
    bulk_load(smem_u32(smem + s * stage_bytes), src, static_cast<uint32_t>(n * ROW), bar);
  };

  int issued = 0;
  if (t == 0) {
    const int first = min(S, mine);
    for (int k = 0; k < first; ++k) issue(k);
    issued = first;
  }
  bool ok = true;
  for (int k = 0; k < mine; ++k) {
    const int s = k % S;
    ok = mbar_wait(smem_u32(&bars[s]), static_cast<uint32_t>((k / S) & 1), abort_flag, a.status,
                   a.limit_ns);
    if (__syncthreads_or(!ok)) { ok = false; break; }
    const int it = s_item[s];
    int blk, id, n;
    const long bh = rows_of(it, blk, id, n);
    const bool valid = id >= 0 && id < a.NB;
    const bool is_k = (it & 1) == 0;
    T* dst = static_cast<T*>(is_k ? a.kpool : a.vpool) +
             (bh * a.NB + (valid ? id : 0)) * static_cast<long>(a.bs) * D;
    if (valid) {
      if (t == 0) {                      // the rows, straight from the stage
        bulk_store(dst, smem_u32(smem + s * stage_bytes), static_cast<uint32_t>(n * ROW));
        bulk_commit();
        if (is_k) {
          a.blk_len[bh * a.NB + id] = n;
          a.blk_pos[bh * a.NB + id] = a.pos0 + blk * a.bs;
        }
      }
      // padding rows of a partial block are zero
      const int pad16 = (a.bs - n) * ROW / 16;
      uint4* pdst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(dst) + n * ROW);
      for (int e = t; e < pad16; e += kPoolThreads) pdst[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    float* rb = red + (k & 1) * 8 * D;
    if (is_k && valid) row_sums<T, D>(smem + s * stage_bytes, n, rb);
    __syncthreads();                     // stage s read by every thread
    if (t == 0 && k + S < mine) {
      bulk_wait_read_all();              // ... and by the bulk store
      issue(k + S);
      ++issued;
    }
    if (is_k && valid && t < D) a.k_bar[(bh * a.NB + id) * D + t] = row_mean<D>(rb, n);
  }
  if (t == 0) {
    if (!ok)
      for (int k = max(0, issued - S); k < issued; ++k)
        mbar_drain(smem_u32(&bars[k % S]), static_cast<uint32_t>((k / S) & 1), a.status,
                   a.limit_ns);
    bulk_wait_all();                     // every row written before the CTA leaves
  }
  __syncthreads();
  if (t < S) mbar_inval(smem_u32(&bars[t]));
}

template <typename T, int D>
int launch_append(AppendArgs a, cudaStream_t s) {
  a.stages = pool_stages<T, D>(a.bs);
  const size_t smem = static_cast<size_t>(a.stages) * a.bs * D * sizeof(T) +
                      2 * 8 * D * sizeof(float) + a.stages * (sizeof(uint64_t) + sizeof(int)) + 16;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaFuncSetAttribute(append_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         200 * 1024);
    attr_set[dev] = true;
  }
  const int grid = max(1, min(a.n_items, 2 * sm_count()));
  cudaError_t e = launch(append_kernel<T, D>, dim3(grid), dim3(kPoolThreads), smem, s, a);
  if (e != cudaSuccess) {
    set_error(std::string("append_kernel: ") + cudaGetErrorString(e));
    return PBSA_ERR_CUDA;
  }
  return PBSA_OK;
}

}  // namespace
}  // namespace pbsa

extern "C" int pbsa_append_chunk(const pbsa_dims* d, const void* k, const void* v, int Tc,
                                 int pos0, void* kpool, void* vpool, int NB,
                                 const int32_t* blk_ids, int32_t* blk_len, int32_t* blk_pos,
                                 float* k_bar, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(Tc >= 1 && NB >= 1, PBSA_ERR_SHAPE, "append_chunk: need Tc >= 1, NB >= 1");
  PBSA_CHECK_ARG(k && v && kpool && vpool && blk_ids && blk_len && blk_pos && k_bar,
                 PBSA_ERR_ARG, "append_chunk: NULL buffer");
  PBSA_CHECK_ARG(aligned(k, 16) && aligned(v, 16) && aligned(kpool, 16) && aligned(vpool, 16),
                 PBSA_ERR_ALIGN, "append_chunk: k, v, kpool and vpool must be 16-byte aligned");
  PBSA_CHECK_ARG(aligned(k_bar, 4) && aligned(blk_len, 4) && aligned(blk_pos, 4) &&
                     aligned(blk_ids, 4),
                 PBSA_ERR_ALIGN, "append_chunk: misaligned int/float buffer");
  const int nb = (Tc + d->bs - 1) / d->bs;
  PBSA_CHECK_ARG(nb <= NB, PBSA_ERR_SHAPE, "append_chunk: the chunk has more blocks than the pool");
  const long n_items = static_cast<long>(d->B) * d->H * nb * 2;
  PBSA_CHECK_ARG(n_items < (1L << 31), PBSA_ERR_SHAPE, "append_chunk: too many blocks");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "append_chunk: no device status word");
  AppendArgs a;
  a.k = k; a.v = v; a.kpool = kpool; a.vpool = vpool; a.blk_ids = blk_ids; a.blk_len = blk_len;
  a.blk_pos = blk_pos; a.k_bar = k_bar; a.Tc = Tc; a.pos0 = pos0; a.NB = NB; a.bs = d->bs;
  a.nb = nb; a.n_items = static_cast<int>(n_items); a.stages = 0;
  a.status = status; a.limit_ns = wait_limit_ns();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d->dtype == PBSA_BF16)
    return d->D == 128 ? launch_append<__nv_bfloat16, 128>(a, s) : launch_append<__nv_bfloat16, 64>(a, s);
  return d->D == 128 ? launch_append<float, 128>(a, s) : launch_append<float, 64>(a, s);
}

// a6: hybrid block-sparse attention, forward, on sm_100a tensor cores.
//
// PBSA computes attention densely over the persistent memory and sparsely
// over the selected local blocks, in one kernel (gist.science/es, section 2
// PBSA, item "Atención Híbrida"), handling irregular sparsity (item
// "Optimización").  Here both parts are one list of physical block ids per
// query block, and one softmax runs over their union.
//
// Design (one CTA per 128-row query tile, 7 warps):
//   warp 4      TMA producer of the Q tile and of K_j for every listed block j,
//               gathered by row coordinate from the block pool through an
//               NSK-stage ring (128-byte swizzle); a K stage is released as
//               soon as its QK^T has run; also allocates / frees TMEM;
//   warp 6      TMA producer of V_j through an NSV-stage ring;
//   warp 5      tcgen05 issuer (one thread): S_0, S_1 first; then for each j,
//               O += P_j V_j (P_j read from TMEM) as soon as the softmax has
//               written it, followed by S_{j+2} = Q K_{j+2}^T into the score
//               buffer just freed -- so the tensor core runs PV_j and QK_{j+2}
//               while the softmax warps handle block j+1;
//   warps 0-3   softmax (thread = query row = TMEM lane): fp32 online softmax
//               in the log2 domain with a lazily moved reference maximum
//               (O in TMEM is rescaled only when the row maximum grows by
//               more than 2^8), P packed to bf16 into TMEM, then the
//               epilogue O / l and LSE.
// TMEM (D = bs = 128): S0 | S1 | O | P0 | P1 = 128+128+128+64+64 columns.
// Every mbarrier wait is bounded; on time-out the CTA raises an abort flag,
// records PBSA_ERR_TIMEOUT, drains its copies and MMAs, frees TMEM, returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_sm100.cuh"
#include "tmap.h"

namespace pbsa {
namespace {

using namespace tc;

struct FwdParams {
  const int32_t* blk_len;
  const int32_t* blk_pos;
  const int32_t* idx;
  const int32_t* cnt;
  __nv_bfloat16* o;
  float* lse;
  int B, H, Tq, q_chunk, q_pos0, NB, Amax, nQB, mask;
  float scale_log2;
  int* status;
  int64_t limit_ns;
  int debug;
};

template <int D, int BS, int NSK, int NSV>
struct FwdCfg {
  static constexpr int BM = 128;
  static constexpr int KB = D / 64;            // 64-column (128-byte) boxes per row
  static constexpr int BOX_Q = BM * 128;
  static constexpr int BOX_KV = BS * 128;
  static constexpr int Q_BYTES = KB * BOX_Q;
  static constexpr int KV_BYTES = KB * BOX_KV;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NSK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NSV * KV_BYTES;
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KF = 1;                         // + K stage
  static constexpr int B_KE = B_KF + NSK;                // + K stage
  static constexpr int B_VF = B_KE + NSK;                // + V stage
  static constexpr int B_VE = B_VF + NSV;                // + V stage
  static constexpr int B_SF = B_VE + NSV;                // + S buffer (2)
  static constexpr int B_PF = B_SF + 2;                  // + P buffer (2)
  static constexpr int B_OD = B_PF + 2;                  // + parity of the PV (2)
  static constexpr int B_MMA = B_OD + 2;
  static constexpr int NBAR = B_MMA + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_IDS = OFF_MISC + 16;
  // tensor-memory columns
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = BS;
  static constexpr int TM_O = 2 * BS;
  static constexpr int TM_P0 = 2 * BS + D;
  static constexpr int TM_P1 = TM_P0 + BS / 2;
  static constexpr int TM_USED = TM_P1 + BS / 2;
  static constexpr int TM_COLS = TM_USED <= 256 ? 256 : 512;
  static_assert(TM_USED <= 512, "tensor memory budget");
  static size_t smem_bytes(int Amax) { return 1024 + OFF_IDS + 3 * 4 * static_cast<size_t>(Amax); }
};

// Warp roles: 0-3 softmax / epilogue, 4 K producer + TMEM owner, 5 MMA issuer,
// 6 V producer.
constexpr int kFwdThreads = 224;

template <int D, int BS, int NSK, int NSV>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, FwdParams p) {
  using C = FwdCfg<D, BS, NSK, NSV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int bh = tile / p.nQB;
  const int qi = tile - bh * p.nQB;
  int n = p.cnt[static_cast<long>(bh) * p.nQB + qi];
  if (n < 0 || n > p.Amax) {
    if (tid == 0) report_status(p.status, PBSA_ERR_ARG);
    n = n < 0 ? 0 : p.Amax;
  }
  int qrow0, qlen;                  // first row and rows of this query block
  qb_rows(qi, p.Tq, p.q_chunk, BS, qrow0, qlen);

  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sK = smem_u32(smem + C::OFF_K);
  const uint32_t sV = smem_u32(smem + C::OFF_V);
  const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* s_ids = reinterpret_cast<int*>(smem + C::OFF_IDS);
  int* s_len = s_ids + p.Amax;
  int* s_pos = s_len + p.Amax;

  if (tid == 0) {
    mbar_init(BAR(C::B_Q), 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(BAR(C::B_KF + s), 1);
      mbar_init(BAR(C::B_KE + s), 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(BAR(C::B_VF + s), 1);
      mbar_init(BAR(C::B_VE + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(C::B_SF + b), 1);
      mbar_init(BAR(C::B_PF + b), 128);
      mbar_init(BAR(C::B_OD + b), 1);
    }
    mbar_init(BAR(C::B_MMA), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const int32_t* row_ids = p.idx + (static_cast<long>(bh) * p.nQB + qi) * p.Amax;
  for (int e = tid; e < n; e += blockDim.x) {
    int id = row_ids[e];
    int len = 0, pos = 0;
    if (id < 0 || id >= p.NB) {
      report_status(p.status, PBSA_ERR_ARG);
      id = 0;                                   // loaded but fully masked
    } else {
      len = min(max(p.blk_len[static_cast<long>(bh) * p.NB + id], 0), BS);
      pos = p.blk_pos ? p.blk_pos[static_cast<long>(bh) * p.NB + id] : 0;
    }
    s_ids[e] = id;
    s_len[e] = len;
    s_pos[e] = pos;
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_holder), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4) {
    // ------------------------------------------------------------ K producer
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      const int q_row = bh * p.Tq + qrow0;
      mbar_expect_tx(BAR(C::B_Q), C::Q_BYTES);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) tma_load_2d(sQ + kb * C::BOX_Q, &tmQ, BAR(C::B_Q), kb * 64, q_row);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % NSK;
        if (j >= NSK &&
            !mbar_wait(BAR(C::B_KE + s), ((j / NSK) & 1) ^ 1, abort_flag, p.status, p.limit_ns))
          break;
        const int kv_row = (bh * p.NB + s_ids[j]) * BS;
        mbar_expect_tx(BAR(C::B_KF + s), C::KV_BYTES);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(sK + s * C::KV_BYTES + kb * C::BOX_KV, &tmK, BAR(C::B_KF + s), kb * 64, kv_row);
        issued = j + 1;
      }
      // no copy may still be in flight when the CTA leaves
      mbar_drain(BAR(C::B_Q), 0, p.status, p.limit_ns);
      for (int s = 0; s < NSK && s < issued; ++s) {
        const int jl = s + ((issued - 1 - s) / NSK) * NSK;   // last load issued to stage s
        mbar_drain(BAR(C::B_KF + s), (jl / NSK) & 1, p.status, p.limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------------ V producer
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tmV);
      const bool skip_v0 = (p.debug & 1) != 0;
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % NSV;
        if (j >= NSV &&
            !mbar_wait(BAR(C::B_VE + s), ((j / NSV) & 1) ^ 1, abort_flag, p.status, p.limit_ns))
          break;
        if (!(skip_v0 && j == 0)) {
          const int kv_row = (bh * p.NB + s_ids[j]) * BS;
          mbar_expect_tx(BAR(C::B_VF + s), C::KV_BYTES);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(sV + s * C::KV_BYTES + kb * C::BOX_KV, &tmV, BAR(C::B_VF + s), kb * 64,
                        kv_row);
        }
        issued = j + 1;
      }
      for (int s = 0; s < NSV && s < issued; ++s) {
        const int jl = s + ((issued - 1 - s) / NSV) * NSV;
        if (!(skip_v0 && jl == 0)) mbar_drain(BAR(C::B_VF + s), (jl / NSV) & 1, p.status, p.limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BS, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      // S_j = Q K_j^T into S buffer (j & 1); frees K stage j % NSK when done
      auto issue_qk = [&](int j) -> bool {
        const int s = j % NSK;
        if (!mbar_wait(BAR(C::B_KF + s), (j / NSK) & 1, abort_flag, p.status, p.limit_ns))
          return false;
        tc_fence_after();
        const uint32_t d_tm = tmem + ((j & 1) ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t koff = (k & 3) * 32;
          const uint64_t a = smem_desc_sw128(sQ + (k >> 2) * C::BOX_Q + koff, 16, 1024);
          const uint64_t b =
              smem_desc_sw128(sK + s * C::KV_BYTES + (k >> 2) * C::BOX_KV + koff, 16, 1024);
          mma_ss(d_tm, a, b, idesc_qk, k > 0 ? 1u : 0u);
        }
        mma_commit(BAR(C::B_SF + (j & 1)));
        mma_commit(BAR(C::B_KE + s));
        return true;
      };
      bool ok = mbar_wait(BAR(C::B_Q), 0, abort_flag, p.status, p.limit_ns) && issue_qk(0) &&
                (n < 2 || issue_qk(1));
      for (int j = 0; ok && j < n; ++j) {
        // O += P_j V_j once the softmax has written P_j
        if (!mbar_wait(BAR(C::B_PF + (j & 1)), (j >> 1) & 1, abort_flag, p.status, p.limit_ns))
          break;
        const int sv = j % NSV;
        if (!mbar_wait(BAR(C::B_VF + sv), (j / NSV) & 1, abort_flag, p.status, p.limit_ns)) break;
        tc_fence_after();
        const uint32_t p_tm = tmem + ((j & 1) ? C::TM_P1 : C::TM_P0);
#pragma unroll
        for (int k = 0; k < BS / 16; ++k) {
          const uint64_t b = smem_desc_sw128(sV + sv * C::KV_BYTES + k * 2048, C::BOX_KV, 1024);
          mma_ts(tmem + C::TM_O, p_tm + k * 8, b, idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(BAR(C::B_OD + (j & 1)));
        mma_commit(BAR(C::B_VE + sv));
        // S buffer (j & 1) is free again: start S_{j+2}
        if (j + 2 < n && !issue_qk(j + 2)) break;
      }
      // every MMA issued so far must finish before TMEM is freed
      mma_commit(BAR(C::B_MMA));
      mbar_drain(BAR(C::B_MMA), 0, p.status, p.limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int row = tid;                         // query row inside the tile
    const int qpos = p.q_pos0 + qrow0 + row;
    const int qpos_first = p.q_pos0 + qrow0;
    const float c_l2 = p.scale_log2;             // logits in log2 units: s * c_l2
    float m_use = -INFINITY;                     // reference maximum, log2 units
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = mbar_wait(BAR(C::B_SF + (j & 1)), (j >> 1) & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_tm = tmem + lane_base + ((j & 1) ? C::TM_S1 : C::TM_S0);
      uint32_t sr[BS];
#pragma unroll
      for (int c = 0; c < BS / 32; ++c)
        tmem_ld32(s_tm + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      const int len = s_len[j];
      const int kpos0 = s_pos[j];
      // masking only for partial blocks and blocks that reach past the first query
      const bool tok = p.mask == PBSA_MASK_TOKEN && kpos0 + BS - 1 > qpos_first;
      if (len < BS || tok) {
#pragma unroll
        for (int c = 0; c < BS; ++c) {
          bool vis = c < len;
          if (tok) vis = vis && (kpos0 + c <= qpos);
          if (!vis) sr[c] = __float_as_uint(-INFINITY);
        }
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < BS; ++c) mx4[c & 3] = fmaxf(mx4[c & 3], __uint_as_float(sr[c]));
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c_l2;
      const float m_new = fmaxf(m_use, mx);
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_use = m_new;
      } else if (m_new > m_use + 8.f) {
        alpha = ex2(m_use - m_new);
        m_use = m_new;
        rescale = true;
      }
      const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < BS; c += 2) {
        const float p0 = ex2(fmaf(__uint_as_float(sr[c]), c_l2, neg_m));
        const float p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), c_l2, neg_m));
        rs4[(c >> 1) & 3] += p0 + p1;
        sr[c >> 1] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds PV_0..PV_{j-1}: wait for the last of them, scale in place
        ok = mbar_wait(BAR(C::B_OD + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag, p.status,
                       p.limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(tmem + lane_base + C::TM_O + c * 32, orr);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st32(tmem + lane_base + C::TM_O + c * 32, orr);
        }
      }
      // P buffer (j & 1) was last read by PV_{j-2}, which completed before S_j
      // (issued after it) was signalled.
      const uint32_t p_tm = tmem + lane_base + ((j & 1) ? C::TM_P1 : C::TM_P0);
#pragma unroll
      for (int c = 0; c < BS / 64; ++c)
        tmem_st32(p_tm + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(C::B_PF + (j & 1)));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n > 0) {
      ok = mbar_wait(BAR(C::B_OD + ((n - 1) & 1)), ((n - 1) >> 1) & 1, abort_flag, p.status,
                     p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const bool valid = row < qlen;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.o + (static_cast<long>(bh) * p.Tq + qrow0 + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        if (n > 0) {
          tmem_ld32(tmem + lane_base + C::TM_O + c * 32, orr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = 0u;
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(orr[8 * v + 0]) * inv, __uint_as_float(orr[8 * v + 1]) * inv);
            u.y = pack_bf16x2(__uint_as_float(orr[8 * v + 2]) * inv, __uint_as_float(orr[8 * v + 3]) * inv);
            u.z = pack_bf16x2(__uint_as_float(orr[8 * v + 4]) * inv, __uint_as_float(orr[8 * v + 5]) * inv);
            u.w = pack_bf16x2(__uint_as_float(orr[8 * v + 6]) * inv, __uint_as_float(orr[8 * v + 7]) * inv);
            dst[v] = u;
          }
        }
      }
      if (valid)
        p.lse[static_cast<long>(bh) * p.Tq + qrow0 + row] =
            l > 0.f ? (m_use + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

template <int D, int BS, int NSK, int NSV>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const FwdParams& prm, cudaStream_t s) {
  using C = FwdCfg<D, BS, NSK, NSV>;
  const size_t smem = C::smem_bytes(prm.Amax);
  PBSA_CHECK_ARG(smem <= 227 * 1024, PBSA_ERR_SHAPE, "attn_fwd: Amax too large for shared memory");
  auto kern = attn_fwd_kernel<D, BS, NSK, NSV>;
  // opt in to the full 227 KB once per device (not a stream operation, so it
  // also happens outside any graph capture after the first call)
  static bool opted[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !opted[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
        cudaSuccess) {
      PBSA_CHECK_LAUNCH("attn_fwd: cudaFuncSetAttribute");
    }
    if (dev >= 0 && dev < 64) opted[dev] = true;
  }
  const long tiles = static_cast<long>(prm.B) * prm.H * prm.nQB;
  kern<<<static_cast<unsigned>(tiles), kFwdThreads, smem, s>>>(mq, mk, mv, prm);
  PBSA_CHECK_LAUNCH("attn_fwd_kernel");
  return PBSA_OK;
}

}  // namespace
}  // namespace pbsa

extern "C" int pbsa_attn_fwd(const pbsa_dims* d, const void* q, int Tq, int q_pos0,
                             const void* kpool, const void* vpool, int NB,
                             const int32_t* blk_len, const int32_t* blk_pos, const int32_t* idx,
                             const int32_t* cnt, int Amax, int mask, void* o, float* lse,
                             void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(d->dtype == PBSA_BF16, PBSA_ERR_DTYPE, "attn_fwd: q/k/v must be bf16");
  PBSA_CHECK_ARG(q && kpool && vpool && blk_len && idx && cnt && o && lse, PBSA_ERR_ARG,
                 "attn_fwd: NULL buffer");
  PBSA_CHECK_ARG(mask == PBSA_MASK_CHUNK || (mask == PBSA_MASK_TOKEN && blk_pos), PBSA_ERR_ARG,
                 "attn_fwd: bad mask, or token mask without blk_pos");
  PBSA_CHECK_ARG(Tq >= 1 && NB >= 1 && Amax >= 1, PBSA_ERR_SHAPE,
                 "attn_fwd: need Tq >= 1, NB >= 1, Amax >= 1");
  PBSA_CHECK_ARG(aligned(q, 16) && aligned(kpool, 16) && aligned(vpool, 16) && aligned(o, 16),
                 PBSA_ERR_ALIGN, "attn_fwd: q, kpool, vpool and o must be 16-byte aligned");
  const long BH = static_cast<long>(d->B) * d->H;
  const int nQB = qb_count(Tq, d->q_chunk, d->bs);
  PBSA_CHECK_ARG(BH * Tq < (1L << 31) && BH * NB * d->bs < (1L << 31), PBSA_ERR_SHAPE,
                 "attn_fwd: tensor rows must be < 2^31");
  PBSA_CHECK_ARG(BH * nQB < (1L << 31), PBSA_ERR_SHAPE, "attn_fwd: too many query tiles");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "attn_fwd: no device status word");
  CUtensorMap mq, mk, mv;
  rc = make_tmap_bf16_2d(&mq, q, BH * Tq, d->D, 128, 64);
  if (rc) return rc;
  rc = make_tmap_bf16_2d(&mk, kpool, BH * NB * d->bs, d->D, d->bs, 64);
  if (rc) return rc;
  rc = make_tmap_bf16_2d(&mv, vpool, BH * NB * d->bs, d->D, d->bs, 64);
  if (rc) return rc;
  FwdParams prm;
  prm.blk_len = blk_len; prm.blk_pos = blk_pos; prm.idx = idx; prm.cnt = cnt;
  prm.o = static_cast<__nv_bfloat16*>(o); prm.lse = lse;
  prm.B = d->B; prm.H = d->H; prm.Tq = Tq; prm.q_chunk = d->q_chunk; prm.q_pos0 = q_pos0; prm.NB = NB; prm.Amax = Amax;
  prm.nQB = nQB; prm.mask = mask;
  prm.scale_log2 = d->scale * 1.4426950408889634f;
  prm.status = status; prm.limit_ns = wait_limit_ns(); prm.debug = debug_flags();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d->D == 128 && d->bs == 128) return launch_fwd<128, 128, 3, 2>(mq, mk, mv, prm, s);
  if (d->D == 64 && d->bs == 128) return launch_fwd<64, 128, 4, 3>(mq, mk, mv, prm, s);
  if (d->D == 128 && d->bs == 64) return launch_fwd<128, 64, 4, 3>(mq, mk, mv, prm, s);
  return launch_fwd<64, 64, 4, 4>(mq, mk, mv, prm, s);
}

// a6: hybrid block-sparse attention, forward, on sm_100a tensor cores.
//
// PBSA computes attention densely over the persistent memory and sparsely
// over the selected local blocks, in one kernel (gist.science/es, section 2
// PBSA, item "Atención Híbrida"), handling irregular sparsity (item
// "Optimización").  Here both parts are one list of physical block ids per
// query block, and one softmax runs over their union.
//
// Design (one CTA per 128-row query tile, 12 warps):
//   warp 8      TMA producer of the Q tile and of K_j / V_j for every listed
//               block j, gathered by row coordinate from the block pool through
//               NSK- and NSV-stage rings (128-byte swizzle); a K stage is
//               released as soon as its QK^T has run, a V stage after its PV;
//               also allocates / frees TMEM;
//   warp 9      tcgen05 issuer (one thread): the blocks of the list are split
//               into two streams (even and odd positions).  S_0, S_1 first; then
//               for each j, O_{j&1} += P_j V_j as soon as stream j&1 has written
//               P_j, followed by S_{j+2} = Q K_{j+2}^T into the same score
//               buffer (MMAs issued by one thread run in order);
//   warps 0-3   softmax of stream 0, warps 4-7 softmax of stream 1 (thread =
//               query row = TMEM lane): fp32 online softmax in the log2 domain
//               with a lazily moved reference maximum (O_h in TMEM is rescaled
//               only when the row maximum grows by more than 2^8), P packed to
//               bf16 over the stream's score buffer;
//   epilogue    warps 0-3 merge the two streams' (m, l, O) and write O, LSE.
// TMEM (D = bs = 128): S0 | S1 | O0 | O1 = 4 x 128 columns.
// Every mbarrier wait is bounded; on time-out the CTA raises an abort flag,
// records PBSA_ERR_TIMEOUT, drains its copies and MMAs, frees TMEM, returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "tc_sm100.cuh"
#include "tmap.h"

#include <string>

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
  static constexpr int OFF_STAT = OFF_V + NSV * KV_BYTES;  // stream 1's m and l per row
  static constexpr int OFF_BAR = OFF_STAT + 2 * 128 * 4;
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KF = 1;                         // + K stage
  static constexpr int B_KE = B_KF + NSK;                // + K stage
  static constexpr int B_VF = B_KE + NSK;                // + V stage
  static constexpr int B_VE = B_VF + NSV;                // + V stage
  static constexpr int B_SF = B_VE + NSV;                // + stream (2)
  static constexpr int B_PF = B_SF + 2;                  // + stream (2)
  static constexpr int B_OD = B_PF + 2;                  // + stream (2)
  static constexpr int B_ST = B_OD + 2;                  // stream 1's statistics written
  static constexpr int B_ST2 = B_ST + 1;                 // merge weights written back
  static constexpr int B_MMA = B_ST2 + 1;
  static constexpr int NBAR = B_MMA + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_IDS = OFF_MISC + 16;
  // tensor-memory columns: per stream h a score buffer S_h (P_h written over
  // its first BS/2 columns as packed bf16) and an output accumulator O_h
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = BS;
  static constexpr int TM_O0 = 2 * BS;
  static constexpr int TM_O1 = 2 * BS + D;
  static constexpr int TM_USED = 2 * BS + 2 * D;
  static constexpr int TM_COLS = TM_USED <= 256 ? 256 : 512;
  static_assert(TM_USED <= 512, "tensor memory budget");
  static size_t smem_bytes(int Amax) { return 1024 + OFF_IDS + 3 * 4 * static_cast<size_t>(Amax); }
};

// Warp roles: 0-3 softmax stream 0 and epilogue, 4-7 softmax stream 1,
// 8 TMA producer (Q, K and V) + TMEM owner, 9 MMA issuer, 10-11 idle.
// Registers: launched with kFwdLaunchRegs per thread (384 x 168 = 64,512 of
// the 65,536); the producer warpgroup (8-11) gives back down to kRegsLow and
// the two softmax warpgroups take kRegsHigh: 8 x 32 x 224 + 4 x 32 x 56 =
// 64,512, and per scheduler (warps w, w+4, w+8) 224 + 224 + 56 <= 512.  The
// host refuses to launch unless the kernel was built with kFwdLaunchRegs.
constexpr int kFwdThreads = 384;
constexpr int kFwdLaunchRegs = 168;
constexpr uint32_t kRegsLow = 56, kRegsHigh = 224;
static_assert(kFwdThreads / 128 * 128 == kFwdThreads, "whole warpgroups");
static_assert(8 * 32 * kRegsHigh + 4 * 32 * kRegsLow == kFwdThreads * kFwdLaunchRegs,
              "register split must equal the launch allocation");

template <int D, int BS, int NSK, int NSV>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, FwdParams p) {
  using C = FwdCfg<D, BS, NSK, NSV>;
  pdl_wait();
  pdl_trigger();
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
  float* st_m1 = reinterpret_cast<float*>(smem + C::OFF_STAT);
  float* st_l1 = st_m1 + 128;
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
    for (int h = 0; h < 2; ++h) {
      mbar_init(BAR(C::B_SF + h), 1);
      mbar_init(BAR(C::B_PF + h), 4);   // one arrival per softmax warp
      mbar_init(BAR(C::B_OD + h), 1);
    }
    mbar_init(BAR(C::B_ST), 128);
    mbar_init(BAR(C::B_ST2), 128);
    mbar_init(BAR(C::B_MMA), 1);
    *abort_flag = 0;
    fence_mbar_init();
    // Q does not depend on the list: its load overlaps the list staging below
    if (n > 0) {
      prefetch_tmap(&tmQ);
      mbar_expect_tx(BAR(C::B_Q), C::Q_BYTES);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_2d(sQ + kb * C::BOX_Q, &tmQ, BAR(C::B_Q), kb * 64, bh * p.Tq + qrow0);
    }
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
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_holder), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (warp >= 8) {
  regs_dec<kRegsLow>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // K_j and V_j in list order.  V_j waits for PV_{j-NSV}, which always
    // completes before K_{j+1} is needed (QK_{j+1} is issued after PV_{j-1}).
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const bool skip_v0 = (p.debug & 1) != 0;
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n; ++j) {
        const int kv_row = (bh * p.NB + s_ids[j]) * BS;
        const int s = j % NSK;
        if (j >= NSK &&
            !mbar_wait(BAR(C::B_KE + s), ((j / NSK) & 1) ^ 1, abort_flag, p.status, p.limit_ns))
          break;
        mbar_expect_tx(BAR(C::B_KF + s), C::KV_BYTES);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(sK + s * C::KV_BYTES + kb * C::BOX_KV, &tmK, BAR(C::B_KF + s), kb * 64, kv_row);
        k_issued = j + 1;
        const int sv = j % NSV;
        if (j >= NSV &&
            !mbar_wait(BAR(C::B_VE + sv), ((j / NSV) & 1) ^ 1, abort_flag, p.status, p.limit_ns))
          break;
        if (!(skip_v0 && j == 0)) {
          mbar_expect_tx(BAR(C::B_VF + sv), C::KV_BYTES);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(sV + sv * C::KV_BYTES + kb * C::BOX_KV, &tmV, BAR(C::B_VF + sv), kb * 64,
                        kv_row);
        }
        v_issued = j + 1;
      }
      // no copy may still be in flight when the CTA leaves
      mbar_drain(BAR(C::B_Q), 0, p.status, p.limit_ns);
      for (int s = 0; s < NSK && s < k_issued; ++s) {
        const int jl = s + ((k_issued - 1 - s) / NSK) * NSK;   // last K load to stage s
        mbar_drain(BAR(C::B_KF + s), (jl / NSK) & 1, p.status, p.limit_ns);
      }
      for (int s = 0; s < NSV && s < v_issued; ++s) {
        const int jl = s + ((v_issued - 1 - s) / NSV) * NSV;
        if (!(skip_v0 && jl == 0)) mbar_drain(BAR(C::B_VF + s), (jl / NSV) & 1, p.status, p.limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BS, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      // S_j = Q K_j^T into the score buffer of stream j & 1; frees K stage j % NSK
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
        const int h = j & 1;
        // O_h += P_j V_j once stream h has written P_j (over S_h).  V_j is
        // normally loaded long before, so it is checked first and PV_j goes
        // out as soon as P_j lands.
        const int sv = j % NSV;
        if (!mbar_wait(BAR(C::B_VF + sv), (j / NSV) & 1, abort_flag, p.status, p.limit_ns)) break;
        if (!mbar_wait(BAR(C::B_PF + h), (j >> 1) & 1, abort_flag, p.status, p.limit_ns)) break;
        tc_fence_after();
        const uint32_t p_tm = tmem + (h ? C::TM_S1 : C::TM_S0);
        const uint32_t o_tm = tmem + (h ? C::TM_O1 : C::TM_O0);
#pragma unroll
        for (int k = 0; k < BS / 16; ++k) {
          const uint64_t b = smem_desc_sw128(sV + sv * C::KV_BYTES + k * 2048, C::BOX_KV, 1024);
          mma_ts(o_tm, p_tm + k * 8, b, idesc_pv, (j >= 2 || k > 0) ? 1u : 0u);
        }
        mma_commit(BAR(C::B_OD + h));
        mma_commit(BAR(C::B_VE + sv));
        // S_{j+2} reuses S_h: tcgen05 MMAs from one thread run in issue order,
        // so it is written only after PV_j has read P_j
        if (j + 2 < n && !issue_qk(j + 2)) break;
      }
      // every MMA issued so far must finish before TMEM is freed
      mma_commit(BAR(C::B_MMA));
      mbar_drain(BAR(C::B_MMA), 0, p.status, p.limit_ns);
    }
    __syncwarp();
  }
  } else {
    regs_inc<kRegsHigh>();
    // ------------------------------------------------------------ softmax
    const int h = warp >> 2;                     // stream: blocks j with j & 1 == h
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t S_tm = tmem + lane_base + (h ? C::TM_S1 : C::TM_S0);
    const uint32_t O_tm = tmem + lane_base + (h ? C::TM_O1 : C::TM_O0);
    const int row = tid & 127;                   // query row inside the tile
    const int qpos = p.q_pos0 + qrow0 + row;
    const int qpos_first = p.q_pos0 + qrow0;
    const float c_l2 = p.scale_log2;             // logits in log2 units: s * c_l2
    float m_use = -INFINITY;                     // reference maximum, log2 units
    float l = 0.f;
    bool ok = true;
    int jj = 0;                                  // index of the block within the stream
    for (int j = h; j < n; j += 2, ++jj) {
      ok = mbar_wait(BAR(C::B_SF + h), jj & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[BS];
#pragma unroll
      for (int c = 0; c < BS / 32; ++c)
        tmem_ld32(S_tm + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      const int len = s_len[j];
      const int kpos0 = s_pos[j];
      // masking only for partial blocks and blocks that reach past the first query
      const bool tok = p.mask == PBSA_MASK_TOKEN && kpos0 + BS - 1 > qpos_first;
      {
        // visible keys are c < lim: one bound per row and a select per element,
        // on every block.  A separate branch taken only by partial blocks cost
        // about 8k cycles each time it ran (measured with clock stamps).
        int lim = len;
        if (tok) lim = min(lim, max(0, qpos - kpos0 + 1));
        if (__any_sync(0xffffffffu, lim < BS)) {
#pragma unroll
          for (int c = 0; c < BS; ++c) sr[c] = c < lim ? sr[c] : __float_as_uint(-INFINITY);
        }
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < BS; c += 8) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          mx4[u] = max3(mx4[u], __uint_as_float(sr[c + 2 * u]), __uint_as_float(sr[c + 2 * u + 1]));
      }
      const float mx = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * c_l2;
      const float m_new = fmaxf(m_use, mx);
      float alpha = 1.f;
      bool rescale = false;
      if (jj == 0) {
        m_use = m_new;
      } else if (m_new > m_use + 8.f) {
        alpha = ex2(m_use - m_new);
        m_use = m_new;
        rescale = true;
      }
      const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;
      const uint64_t negm2 = f2(neg_m, neg_m);
      const uint64_t cl2 = f2(c_l2, c_l2);
      uint64_t rs2[2] = {0ull, 0ull};
      if (len == BS && !tok) {
        // no masked key: one pair in four takes the FMA-pipe exp2
#pragma unroll
        for (int c = 0; c < BS; c += 2) {
          const uint64_t x2 =
              fma2(f2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), cl2, negm2);
          uint64_t p2;
          if (((c >> 1) & 3) == 3) {
            p2 = exp2_poly2(x2);
          } else {
            float x0, x1;
            f2_split(x2, x0, x1);
            p2 = f2(ex2(x0), ex2(x1));
          }
          rs2[(c >> 1) & 1] = add2(rs2[(c >> 1) & 1], p2);
          float p0, p1;
          f2_split(p2, p0, p1);
          sr[c >> 1] = pack_bf16x2(p0, p1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BS; c += 2) {
          const uint64_t x2 =
              fma2(f2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), cl2, negm2);
          float x0, x1;
          f2_split(x2, x0, x1);
          const uint64_t p2 = f2(ex2(x0), ex2(x1));
          rs2[(c >> 1) & 1] = add2(rs2[(c >> 1) & 1], p2);
          float p0, p1;
          f2_split(p2, p0, p1);
          sr[c >> 1] = pack_bf16x2(p0, p1);
        }
      }
      float ra, rb, rc, rd;
      f2_split(rs2[0], ra, rb);
      f2_split(rs2[1], rc, rd);
      l = l * alpha + ((ra + rb) + (rc + rd));
      if (__any_sync(0xffffffffu, rescale)) {
        // O_h holds this stream's earlier blocks; their last PV (block j-2) was
        // issued before S_j, whose completion was just observed.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(O_tm + c * 32, orr);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st32(O_tm + c * 32, orr);
        }
      }
      // P_j over the first BS/2 columns of S_h (its scores are in registers now)
#pragma unroll
      for (int c = 0; c < BS / 64; ++c)
        tmem_st32(S_tm + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_PF + h));
    }
    // ------------------------------------------------------------ epilogue
    const int n_h = (n - h + 1) / 2;             // blocks of this stream
    if (ok && n_h > 0) {
      ok = mbar_wait(BAR(C::B_OD + h), (n_h - 1) & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    // Merge the two streams: stream 1 hands its (m, l) to stream 0, which
    // writes back the weights of O0 and O1; then each stream normalises and
    // stores half of the row's columns (and stream 0 the LSE).
    const int n1 = n / 2;
    float w0 = 0.f, w1 = 0.f, m = -INFINITY, lt = 0.f;
    if (h == 1) {
      st_m1[row] = m_use;
      st_l1[row] = l;
      tc_fence_before();
      mbar_arrive(BAR(C::B_ST));
      bool ok2 = mbar_wait(BAR(C::B_ST2), 0, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok && ok2);
      if (ok) {
        w0 = st_m1[row];
        w1 = st_l1[row];
      }
    } else {
      bool ok1 = mbar_wait(BAR(C::B_ST), 0, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok && ok1);
      if (ok) {
        const float m1 = st_m1[row], l1 = st_l1[row];
        m = fmaxf(m_use, m1);
        const float a0 = (m_use == -INFINITY) ? 0.f : ex2(m_use - m);
        const float a1 = (m1 == -INFINITY || n1 == 0) ? 0.f : ex2(m1 - m);
        lt = a0 * l + a1 * l1;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        w0 = a0 * inv;
        w1 = a1 * inv;
        st_m1[row] = w0;
        st_l1[row] = w1;
      }
      tc_fence_before();
      mbar_arrive(BAR(C::B_ST2));
    }
    if (ok) {
      tc_fence_after();
      const bool valid = row < qlen;
      __nv_bfloat16* orow = p.o + (static_cast<long>(bh) * p.Tq + qrow0 + row) * D;
      constexpr int HALF = D / 64;             // 32-column chunks per stream
#pragma unroll
      for (int cc = 0; cc < HALF; ++cc) {
        const int c = h * HALF + cc;
        uint32_t o0[32], o1[32];
        if (n > 0) tmem_ld32(tmem + lane_base + C::TM_O0 + c * 32, o0);
        if (n1 > 0) tmem_ld32(tmem + lane_base + C::TM_O1 + c * 32, o1);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float x = n > 0 ? __uint_as_float(o0[e]) * w0 : 0.f;
          if (n1 > 0) x = fmaf(__uint_as_float(o1[e]), w1, x);
          v[e] = x;
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 u;
            u.x = pack_bf16x2(v[8 * q4 + 0], v[8 * q4 + 1]);
            u.y = pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]);
            u.z = pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]);
            u.w = pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]);
            dst[q4] = u;
          }
        }
      }
      if (h == 0 && valid)
        p.lse[static_cast<long>(bh) * p.Tq + qrow0 + row] =
            lt > 0.f ? (m + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
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
  // the register split inside the kernel assumes this launch allocation
  static int launch_regs[64] = {0};
  int rdev = 0;
  cudaGetDevice(&rdev);
  if (rdev < 0 || rdev >= 64 || launch_regs[rdev] == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) PBSA_CHECK_LAUNCH("attn_fwd: attributes");
    if (rdev >= 0 && rdev < 64) launch_regs[rdev] = fa.numRegs;
    PBSA_CHECK_ARG(fa.numRegs == kFwdLaunchRegs, PBSA_ERR_CUDA,
                   "attn_fwd: kernel built with " + std::to_string(fa.numRegs) +
                       " registers per thread, the register split needs " +
                       std::to_string(kFwdLaunchRegs));
  } else {
    PBSA_CHECK_ARG(launch_regs[rdev] == kFwdLaunchRegs, PBSA_ERR_CUDA,
                   "attn_fwd: kernel register count does not match the register split");
  }
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
  if (launch(kern, dim3(static_cast<unsigned>(tiles)), dim3(kFwdThreads), smem, s, mq, mk, mv,
             prm) != cudaSuccess)
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
  if (d->D == 128 && d->bs == 128) {
    if (FwdCfg<128, 128, 3, 3>::smem_bytes(Amax) <= 227 * 1024)
      return launch_fwd<128, 128, 3, 3>(mq, mk, mv, prm, s);
    return launch_fwd<128, 128, 3, 2>(mq, mk, mv, prm, s);
  }
  if (d->D == 64 && d->bs == 128) return launch_fwd<64, 128, 4, 3>(mq, mk, mv, prm, s);
  if (d->D == 128 && d->bs == 64) return launch_fwd<128, 64, 4, 3>(mq, mk, mv, prm, s);
  return launch_fwd<64, 64, 4, 4>(mq, mk, mv, prm, s);
}

/*
 * pbsa.h -- C ABI of the PBSA (Persistent Block-Sparse Attention) hot path on
 * NVIDIA B200 (sm_100a).
 *
 * Source of the operations: "Sparse Forcing: Native Trainable Sparse
 * Attention for Real-time Autoregressive Diffusion Video Generation"
 * (arXiv 2604.21221), as summarised on gist.science/es (section 2
 * "Metodología: Sparse Forcing": items "Arquitectura Propuesta" and
 * "Persistente Block-Sparse Attention (PBSA)") and in the paper's abstract
 * (shd-paper.top page).  The pages describe the method in words only; the
 * concrete formulas below are the plainest reading of them.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor arguments are DEVICE pointers owned by the caller; the library
 *    allocates no device memory at run time.  Its device state is static,
 *    created when the library is loaded on a device: one status word per
 *    device (a __device__ variable, see pbsa_get_status) and the 16 MiB
 *    scratch array of pbsa_attn_bwd_noalloc (a __device__ array that every
 *    device which loads the library holds until the process exits).
 *  - `stream` is a cudaStream_t passed as void*.  Every call is asynchronous
 *    on that stream; nothing synchronises except pbsa_get_status.
 *  - Batch-major layouts, all contiguous:
 *      q, o, dO          [B, H, Tq, D]          (query chunk, Tq tokens)
 *      kpool, vpool      [B, H, NB, bs, D]      (block pool, NB physical blocks)
 *      blk_len, blk_pos  [B, H, NB]   int32     (valid rows of a block; global
 *                                               token position of its row 0)
 *      k_bar             [B, H, NB, D] float    (pooled key of each block)
 *      q_bar             [B, H, nQB, D] float   nQB query blocks (see below)
 *      scores            [B, H, nQB, NB] float
 *      mem_score         [B, H, G, NB] float    G query chunks (1 if q_chunk = 0)
 *      slot_src, slot_w  [B, H, P]    int32 / float  (persistent slots are
 *                                               physical ids 0..P-1)
 *      idx               [B, H, nQB, Amax] int32 (attended physical ids,
 *                                               ascending, padded with -1)
 *      cnt               [B, H, nQB]  int32
 *  - Query rows are a sequence of chunks of dims.q_chunk rows (the last chunk
 *    may be shorter; q_chunk = 0 means one chunk of Tq rows).  Each chunk is
 *    tiled into blocks of bs rows on its own, so the last block of every chunk
 *    may be partial: with nb = ceil(q_chunk / bs), query block i covers rows
 *    [c*q_chunk + b*bs, c*q_chunk + min((b+1)*bs, len_c)) for c = i / nb,
 *    b = i % nb, len_c the rows of chunk c.  nQB counts these blocks.  Rows
 *    of a cache block at or past blk_len are padding: never read as tokens.
 *  - Supported shapes: D in {64, 128}; bs in {64, 128}; B*H >= 1.
 *  - bf16 buffers must be 16-byte aligned (128-bit loads and TMA); float and
 *    int buffers 4-byte aligned.
 *
 * Errors
 * ------
 *  Every call validates its arguments on the host first and returns a negative
 *  pbsa_status without launching anything when they are wrong.  A failed launch
 *  returns PBSA_ERR_CUDA.  Faults found on the device (a bounded wait that ran
 *  out) set the device status word, read and cleared by pbsa_get_status.
 *  pbsa_last_error() gives a message for the last failing call of the thread.
 */
#ifndef PBSA_H
#define PBSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PBSA_OK = 0,
  PBSA_ERR_ARG = -1,        /* null pointer, negative size, bad enum        */
  PBSA_ERR_SHAPE = -2,      /* unsupported or inconsistent shape            */
  PBSA_ERR_ALIGN = -3,      /* misaligned buffer                           */
  PBSA_ERR_DTYPE = -4,      /* dtype not supported by this call            */
  PBSA_ERR_CUDA = -5,       /* CUDA runtime error (launch, copy)           */
  PBSA_ERR_TIMEOUT = -6,    /* device: a bounded wait ran out              */
  PBSA_ERR_WORKSPACE = -7   /* workspace missing or too small              */
} pbsa_status;

typedef enum { PBSA_BF16 = 0, PBSA_FP32 = 1 } pbsa_dtype;
typedef enum { PBSA_EVICT = 0, PBSA_MERGE_MEAN = 1 } pbsa_policy;
typedef enum { PBSA_MASK_CHUNK = 0, PBSA_MASK_TOKEN = 1 } pbsa_mask;

/* Problem dimensions shared by all calls.  scale multiplies <q, k> (usually
 * 1/sqrt(D)); dtype is the storage type of q, kpool and vpool; q_chunk is the
 * number of query rows per chunk (0: the whole query is one chunk). */
typedef struct {
  int B, H, D, bs;
  float scale;
  int dtype; /* pbsa_dtype */
  int q_chunk;
} pbsa_dims;

/* ---------------------------------------------------------------------------
 * a1 + a2: block compression by pooling and coarse block scoring.
 * Passage: gist.science/es section 2, PBSA item "Compresión de Bloques" (pooled
 * block representatives for coarse routing) and item "Bloques Dinámicos"
 * (coarse scoring of historical blocks for the current step).
 *
 *   q_bar[b,h,i]     = mean of the rows of query block i
 *   k_bar[b,h,j]     = mean of the first blk_len[b,h,j] rows of block j, for
 *                      j in pool_ids only (other entries are left as they are;
 *                      a block of length 0 pools to zero)
 *   scores[b,h,i,j]  = scale * <q_bar[b,h,i], k_bar[b,h,j]>  for all j < NB
 *   mem_score[b,h,g,j] = mean of scores[b,h,i,j] over the query blocks i of
 *                      query chunk g (one chunk, g = 0, when dims.q_chunk = 0),
 *                      computed as scale * <mean of those q_bar[b,h,i],
 *                      k_bar[b,h,j]>, which equals it up to rounding
 *
 * q, kpool: dtype of dims (bf16 or fp32).  pool_ids: device int32 [n_pool],
 * the same list for every (b,h); n_pool may be 0.  Outputs are overwritten.
 * ------------------------------------------------------------------------- */
int pbsa_score_blocks(const pbsa_dims* dims, const void* q, int Tq,
                      const void* kpool, int NB, const int32_t* blk_len,
                      const int32_t* pool_ids, int n_pool,
                      float* q_bar, float* k_bar, float* scores, float* mem_score,
                      void* stream);

/* ---------------------------------------------------------------------------
 * a0: KV append with block compression fused in.
 * Passage: gist.science/es section 2, PBSA item "Compresión de Bloques" (the
 * pooled representative of each block) and item "Optimización" (selective KV
 * cache updates are part of the kernel's job).
 *
 * The chunk's rows t = 0..Tc-1 fall into blocks c = t / bs (nb = ceil(Tc/bs)
 * of them; the last may be partial).  Chunk block c goes to pool block
 * blk_ids[c], for every (b,h):
 *   kpool[b,h,blk_ids[c], r] = k[b,h,c*bs + r]   for r < n_c = min(bs, Tc - c*bs)
 *   vpool[b,h,blk_ids[c], r] = v[b,h,c*bs + r]   (rows r >= n_c are zeroed)
 *   blk_len[b,h,blk_ids[c]] = n_c,  blk_pos[b,h,blk_ids[c]] = pos0 + c*bs
 *   k_bar[b,h,blk_ids[c]]   = mean of the n_c rows written (fp32), the same
 *                             value pbsa_score_blocks gives for that block
 * so a following pbsa_score_blocks needs no pool_ids for the chunk's blocks.
 *
 * k, v: dtype of dims, [B,H,Tc,D] contiguous.  kpool, vpool: [B,H,NB,bs,D].
 * blk_len, blk_pos: int32 [B,H,NB].  k_bar: fp32 [B,H,NB,D].  blk_ids: device
 * int32 [nb], distinct, each in [0, NB) (an id outside that range sets the
 * device status to PBSA_ERR_ARG and its block is skipped).  k, v, kpool, vpool
 * 16-byte aligned.  Nothing is allocated; the call is asynchronous on stream.
 * ------------------------------------------------------------------------- */
int pbsa_append_chunk(const pbsa_dims* dims, const void* k, const void* v, int Tc, int pos0,
                      void* kpool, void* vpool, int NB, const int32_t* blk_ids,
                      int32_t* blk_len, int32_t* blk_pos, float* k_bar, void* stream);

/* ---------------------------------------------------------------------------
 * a3: persistent-memory update (Top-C retention, sinks, evict or mean-merge).
 * Passage: gist.science/es section 2 "Arquitectura Propuesta", items "Memoria
 * Persistente", "Bloques Sumidero", "Bloques Dinámicos", "Mecanismo de
 * Actualización"; the abstract (the memory compresses as well as keeps its
 * blocks); PBSA item "Optimización" (selective cache updates).
 *
 * Per (b,h): the candidates are the occupied non-sink slots (slot_src >= 0,
 * index >= n_sink) and the blocks leaving the window, cand_ids (physical ids)
 * with global ids cand_src.  A leaving block with cand_src < n_sink fills
 * sink slot cand_src and is not ranked.  Candidates are ranked by
 * mem_score (descending; ties: lower global id first) and the best
 * P - n_sink are kept.  Kept slots stay where they are; newly kept blocks
 * fill the free non-sink slots in ascending order, in ascending global-id
 * order.  Losers are dropped (PBSA_EVICT) or, with PBSA_MERGE_MEAN, merged
 * into the kept slot whose pre-merge pooled key has the largest dot product
 * with theirs (ties: lowest slot).  A merged slot holds the weight-averaged,
 * row-wise mean of its blocks (rows past a block's length count as zero),
 * its weight is the sum of weights, its length the maximum, and its k_bar is
 * the mean of its stored rows.  Slot rows, blk_len, blk_pos, k_bar, slot_src
 * and slot_w of slot ids 0..P-1 are updated IN PLACE; other ids are only read.
 *
 * cand_ids, cand_src: device int32 [n_cand], same for every (b,h).
 * Limits: 1 <= P <= 256, 0 <= n_sink <= P, (P - n_sink) + n_cand <= 256.
 * workspace: device buffer of at least pbsa_update_memory_workspace() bytes,
 * 256-byte aligned; its contents need not be initialised.
 * ------------------------------------------------------------------------- */
size_t pbsa_update_memory_workspace(const pbsa_dims* dims, int P, int n_cand);
int pbsa_update_memory(const pbsa_dims* dims, void* kpool, void* vpool, int NB,
                       int32_t* blk_len, int32_t* blk_pos, float* k_bar,
                       int P, int n_sink, int32_t* slot_src, float* slot_w,
                       const int32_t* cand_ids, const int32_t* cand_src, int n_cand,
                       const float* mem_score, int policy,
                       void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Backward of a3 for the key and value rows: the recurrent trainable path.
 * Passage: gist.science/es section 2 "Entrenamiento" (training with the
 * dynamically updated cache) and the abstract (the memory learns to compress,
 * keep and refresh persistent blocks): the loss reaches a block's keys and
 * values also through the slots it was copied or merged into.
 *
 * After pbsa_update_memory every slot s is a weighted row-wise sum of
 * pre-update blocks: unchanged; emptied; a copy of one block (the whole
 * block); or the merge (bw * base[r < len_base] + sum_m w_m * src_m[r < len_m])
 * / (bw + sum_m w_m) of its kept block and the losers merged into it (a loser
 * that was a slot overwritten in the same update is that slot's content before
 * it).  The selection and merge decisions are constants.  This call applies
 * the transposed sum:
 *   on entry dk, dv = the gradient of a loss w.r.t. the pool after the update;
 *   on return       = the gradient w.r.t. the pool before it: every block keeps
 *                     its own gradient plus weight * d(slot)[r] (r < rows) for
 *                     each slot term it appears in; a slot whose content the
 *                     update replaced or emptied gets only what reaches its
 *                     pre-update content through such terms; an unchanged slot
 *                     keeps its gradient.
 * The rounding of merged rows to the storage type is taken as the identity.
 *
 * plan: the first pbsa_update_plan_bytes(dims, P, n_cand) bytes of the
 * workspace of the pbsa_update_memory call being differentiated, as that call
 * left them (a rollout keeps a copy per step), 16-byte aligned.  dk, dv: float
 * [B,H,NB,bs,D], 16-byte aligned.  Candidate ids must lie outside the slot ids
 * (as in every layout where the window and the slots are apart).
 * workspace: at least pbsa_update_memory_bwd_workspace(dims, P) bytes,
 * 256-byte aligned.  Nothing is allocated; asynchronous on `stream`.
 * ------------------------------------------------------------------------- */
size_t pbsa_update_plan_bytes(const pbsa_dims* dims, int P, int n_cand);
size_t pbsa_update_memory_bwd_workspace(const pbsa_dims* dims, int P);
int pbsa_update_memory_bwd(const pbsa_dims* dims, int NB, int P, int n_cand, const void* plan,
                           float* dk, float* dv, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * a4 + a5: local Top-K selection and the attended-block list.
 * Passage: gist.science/es section 2 "Arquitectura Propuesta", item "Ventana
 * Local" (per-query Top-K of relevant blocks inside the sliding window) and
 * PBSA item "Atención Híbrida" (dense over the persistent memory).
 *
 * For each (b,h) and query block i < nQB of this call (list row
 * r = qb_offset + i of the nQB_total rows of scores, idx and cnt):
 *   candidates = win_ids[0..n_win) with blk_len > 0 (and, with PBSA_MASK_TOKEN,
 *                blk_pos <= q_pos0 + last row of block i);
 *   local      = the best min(k, #candidates) by scores[b,h,r,j] (descending;
 *                ties: lower physical id first);
 *   list       = mem_ids[b,h,0..n_mem) entries >= 0 with blk_len > 0, united
 *                with local, ascending, without duplicates.
 * Written to idx[b,h,r,0..cnt) (rest -1) and cnt[b,h,r].
 *
 * Errors found on the device: a list longer than Amax sets PBSA_ERR_SHAPE and
 * writes an empty row (cnt 0, every entry -1), so a later attention call on
 * the same stream attends nothing for that row rather than stale blocks; a
 * win_ids entry outside [0, NB), or a mem_ids entry outside [-1, NB), sets
 * PBSA_ERR_ARG and is skipped.
 *
 * scores: [B,H,nQB_total,NB] float, indexed by the same physical ids as
 * blk_len and blk_pos [B,H,NB].  win_ids: device int32 [n_win], same for every
 * (b,h).  mem_ids: device int32, row (b,h) at mem_ids + (b*H+h)*mem_ld
 * (mem_ld = 0 means n_mem), or NULL with n_mem = 0.  blk_pos may be NULL with
 * PBSA_MASK_CHUNK.  Tq is this call's query rows (nQB must be their block
 * count under dims.q_chunk; used for the token mask).
 * Limits: n_win <= 512, n_mem + min(k, n_win) <= min(Amax, 512).
 * ------------------------------------------------------------------------- */
int pbsa_select_local(const pbsa_dims* dims, const float* scores, int nQB, int NB,
                      const int32_t* win_ids, int n_win, int k,
                      const int32_t* mem_ids, int n_mem, int mem_ld,
                      const int32_t* blk_len, int mask, int q_pos0, const int32_t* blk_pos,
                      int Tq, int32_t* idx, int32_t* cnt, int Amax,
                      int qb_offset, int nQB_total, void* stream);

/* ---------------------------------------------------------------------------
 * a4 + a5, two-level variant: frame -> block local selection, the alternative
 * router of the "next" rows.
 * Passage: Light Forcing (gist.science/it, section 2.2 "Attenzione Sparsa
 * Gerarchica (HSA)"): keys are mean-pooled per block and per frame; each query
 * block keeps a few relevant frames by their frame-level keys, then the
 * critical blocks inside those frames by their block-level keys.
 *
 * As pbsa_select_local, except that the local set is chosen in two levels.
 * A frame is a group of window entries: win_frame[e] in [0, n_frames) is the
 * frame of entry e (same for every (b,h); n_frames <= 32).  For query block i
 * the frame's score is the length-weighted mean of scores[b,h,r,j] over its
 * candidate blocks j (the mean pooled key of the frame's tokens, scored; the
 * candidates follow the rules of pbsa_select_local), summed in window order;
 * the F frames of highest score are kept (ties: lower frame), and the local
 * set is the best min(k, #their candidates) blocks of the kept frames by score
 * (ties: lower physical id).  The list is its union with the memory ids.  With
 * F >= n_frames it equals pbsa_select_local's list.
 * Limits: n_win <= 512, n_mem <= 512, n_mem + min(k, n_win) <= Amax,
 * NB <= 32768.  win_frame: device int32 [n_win].  Errors as pbsa_select_local
 * (a win_frame label outside [0, n_frames) sets PBSA_ERR_ARG and the entry is
 * skipped).
 * ------------------------------------------------------------------------- */
int pbsa_select_hier(const pbsa_dims* dims, const float* scores, int nQB, int NB,
                     const int32_t* win_ids, const int32_t* win_frame, int n_win, int n_frames,
                     int F, int k, const int32_t* mem_ids, int n_mem, int mem_ld,
                     const int32_t* blk_len, int mask, int q_pos0, const int32_t* blk_pos,
                     int Tq, int32_t* idx, int32_t* cnt, int Amax, int qb_offset,
                     int nQB_total, void* stream);

/* ---------------------------------------------------------------------------
 * a1..a5 in one launch: score -> update memory -> select for one query chunk.
 * Passages: those of pbsa_score_blocks, pbsa_update_memory and
 * pbsa_select_local above; this call has no separate counterpart on the pages.
 * It is the routing half of a decode step as the pages order it.
 *
 * Results are exactly those of the three calls made in order on the same
 * stream:
 *   pbsa_score_blocks(dims, q, Tq, kpool, NB, blk_len, pool_ids, n_pool,
 *                     q_bar, k_bar, scores, mem_score)
 *   pbsa_update_memory(dims, kpool, vpool, NB, blk_len, blk_pos, k_bar, P,
 *                      n_sink, slot_src, slot_w, cand_ids, cand_src, n_cand,
 *                      mem_score, policy, ...)   -- skipped if P == 0 or n_cand == 0
 *   pbsa_select_local(dims, scores, nQB, NB, win_ids, n_win, k, mem_ids, n_mem,
 *                     0, blk_len, mask, q_pos0, blk_pos, Tq, idx, cnt, Amax,
 *                     0, nQB)
 * with the same argument rules and limits.  The work runs as one persistent
 * kernel when the shape has an instantiation (n_win <= 256 and n_mem +
 * min(k, n_win) <= 128); otherwise the call makes the three per-call launches
 * itself.  Inside the kernel every piece of work (a block to pool, a tile of
 * scores, a head's update plan, a slot to write, eight attended lists) is a
 * ticket handed out in order by an atomic counter, and each ticket waits
 * (bounded in time) only for the per-head tickets it reads, so no step waits
 * for every head of the step before it.
 *
 * workspace: device, 256-byte aligned, at least pbsa_route_workspace() bytes.
 * Its first C = 256 * ceil((16 + 20*B*H) / 256) bytes hold the kernel's
 * counters: zero them once before the first call (e.g. cudaMemset); every
 * call leaves them zero again.  The rest is the update's workspace.  Calls
 * that share a workspace must not run concurrently.
 * ------------------------------------------------------------------------- */
typedef struct {
  /* a1 + a2 */
  const void* q;
  int Tq;
  void* kpool;
  void* vpool;
  int NB;
  int32_t* blk_len;
  int32_t* blk_pos;
  const int32_t* pool_ids;
  int n_pool;
  float* q_bar;
  float* k_bar;
  float* scores;
  float* mem_score;
  /* a3 */
  int P;
  int n_sink;
  int32_t* slot_src;
  float* slot_w;
  const int32_t* cand_ids;
  const int32_t* cand_src;
  int n_cand;
  int policy; /* pbsa_policy */
  /* a4 + a5 */
  const int32_t* win_ids;
  int n_win;
  int k;
  const int32_t* mem_ids;
  int n_mem;
  int mask; /* pbsa_mask */
  int q_pos0;
  int32_t* idx;
  int32_t* cnt;
  int Amax;
} pbsa_route_args;

size_t pbsa_route_workspace(const pbsa_dims* dims, int P, int n_cand);
int pbsa_route_step(const pbsa_dims* dims, const pbsa_route_args* args, void* workspace,
                    size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * a6: hybrid block-sparse attention, forward.
 * Passage: gist.science/es section 2 PBSA item "Atención Híbrida" (dense over
 * the persistent memory plus sparse over the local window, one kernel) and
 * item "Optimización" (irregular sparsity); section 4 (speed-up over
 * FlashAttention-2 grows with sparsity).
 *
 * For each row r of query block i: one softmax over the valid rows of the
 * blocks idx[b,h,i,0..cnt):
 *   O[r]   = sum_c softmax_c(scale * <q_r, k_c>) v_c
 *   lse[r] = log sum_c exp(scale * <q_r, k_c>)          (natural log)
 * PBSA_MASK_TOKEN keeps only keys with blk_pos + row <= q_pos0 + r.  A row
 * with no visible key gets O = 0 and lse = -inf.
 * q, kpool, vpool, o: bf16 only (dims.dtype must be PBSA_BF16); lse: float.
 * Every idx entry must be in [0, NB); cnt <= Amax.  Runs on tcgen05 tensor
 * cores (sm_100a).
 * ------------------------------------------------------------------------- */
int pbsa_attn_fwd(const pbsa_dims* dims, const void* q, int Tq, int q_pos0,
                  const void* kpool, const void* vpool, int NB,
                  const int32_t* blk_len, const int32_t* blk_pos,
                  const int32_t* idx, const int32_t* cnt, int Amax, int mask,
                  void* o, float* lse, void* stream);

/* ---------------------------------------------------------------------------
 * a7: backward of pbsa_attn_fwd for the trainable path.
 * Passage: gist.science/es section 2 "Entrenamiento" (training with the
 * dynamically updated cache) and section 3 "Contribuciones Clave", item
 * "Kernel PBSA" (the kernel serves training as well as inference).
 *
 * The attended lists are constants.  With P the forward's softmax:
 *   dV_c += P^T dO,  dP = dO V^T,  Delta_r = <dO_r, O_r>,
 *   dS = P * (dP - Delta),  dQ = scale * dS K,  dK_c += scale * dS^T Q.
 * o, lse are the forward's outputs; dO bf16 [B,H,Tq,D].  dq [B,H,Tq,D],
 * dk/dv [B,H,NB,bs,D] are float and fully overwritten (blocks nobody attends
 * get zero).  workspace: at least pbsa_attn_bwd_workspace() bytes.
 * ------------------------------------------------------------------------- */
size_t pbsa_attn_bwd_workspace(const pbsa_dims* dims, int Tq, int NB, int Amax);
int pbsa_attn_bwd(const pbsa_dims* dims, const void* q, int Tq, int q_pos0,
                  const void* kpool, const void* vpool, int NB,
                  const int32_t* blk_len, const int32_t* blk_pos,
                  const int32_t* idx, const int32_t* cnt, int Amax, int mask,
                  const void* o, const float* lse, const void* dO,
                  float* dq, float* dk, float* dv,
                  void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * pbsa_attn_bwd_noalloc: the backward of pbsa_attn_fwd, as pbsa_attn_bwd, for
 * callers that cannot give the library a device buffer.  The Sparse Forcing
 * pages have no counterpart; this is an interface convenience.
 *
 * Who needs it: a host process that owns all device memory through its own
 * pool and offers no allocator hook, or code that must never enter the CUDA
 * allocator (cudaMalloc may synchronise the device and stall for
 * milliseconds).  Arguments and results are those of pbsa_attn_bwd minus the
 * workspace; the caller still passes every input and output buffer.
 *
 * Scratch: a fixed 16 MiB array of device memory inside the library (see
 * pbsa_attn_bwd_noalloc_max_scratch).  Every GPU that loads the library keeps
 * it allocated until the process exits.  Problems whose scratch
 * (pbsa_attn_bwd_workspace) exceeds it are rejected with PBSA_ERR_WORKSPACE and
 * nothing is launched.  The call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current) and caches it for the life of the
 * process; make that first call before any stream capture.  cudaDeviceReset
 * invalidates the cached address: do not call this entry point on a device
 * after resetting it.  All calls share the one array, which keeps the previous call's
 * contents (each call clears what must start at zero): calls that may overlap
 * on the GPU -- different streams, or different host threads -- race on it
 * and must be ordered by the caller.
 * ------------------------------------------------------------------------- */
int pbsa_attn_bwd_noalloc(const pbsa_dims* dims, const void* q, int Tq, int q_pos0,
                          const void* kpool, const void* vpool, int NB,
                          const int32_t* blk_len, const int32_t* blk_pos,
                          const int32_t* idx, const int32_t* cnt, int Amax, int mask,
                          const void* o, const float* lse, const void* dO,
                          float* dq, float* dk, float* dv, void* stream);

/* Size in bytes of the built-in scratch used by pbsa_attn_bwd_noalloc. */
size_t pbsa_attn_bwd_noalloc_max_scratch(void);

/* ---------------------------------------------------------------------------
 * Status and diagnostics (no counterpart on the pages).
 * ------------------------------------------------------------------------- */

/* Synchronises `stream`, returns the device status word of the current device
 * (PBSA_OK, or PBSA_ERR_TIMEOUT when a kernel's bounded wait ran out) and
 * clears it.  Returns PBSA_ERR_CUDA if the read itself fails. */
int pbsa_get_status(void* stream);

/* Checks the software exponent of the attention softmax.  For i < n:
 * y_poly[i] = 2^x[i] as the softmax computes it on the FMA pipe for one pair of
 * scores in four (a degree-3 polynomial after a Cody-Waite range split, stated
 * relative error 7.6e-5 for x in [-125, 8]), y_hw[i] = 2^x[i] from the
 * special-function unit (ex2.approx).  x, y_poly, y_hw: device float [n].
 * Returns PBSA_ERR_ARG for NULL buffers or n < 1.  No counterpart on the
 * pages: a test hook. */
int pbsa_check_exp2(const float* x, float* y_poly, float* y_hw, int n, void* stream);

/* Message for the last failing call made by this host thread ("" if none). */
const char* pbsa_last_error(void);

/* Library version string. */
const char* pbsa_version(void);

/* Test hook for the failure path.  Sets the time limit of every bounded
 * device wait (nanoseconds; <= 0 restores the default of 2 s) and debug
 * flags: bit 0 makes the next pbsa_attn_fwd launches skip the first V-tile
 * load, so that the tensor-core issuer's wait for it runs out, the kernel
 * sets PBSA_ERR_TIMEOUT and every CTA returns cleanly; bit 1 makes the next
 * pbsa_route_step kernels withhold the completion counts of head 0's pooling,
 * so that head's dependent work times out, the kernel sets PBSA_ERR_TIMEOUT,
 * skips the rest, and still leaves its counters zero. */
void pbsa_set_debug(int flags, int64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* PBSA_H */

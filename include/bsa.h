/*
 * bsa.h -- C ABI of the B200 (sm_100a) block-sparse video self-attention
 * library, libbsa.so.
 *
 * What the library computes.  Tokens of a video latent lie on a T x H x W
 * grid (Prism / Kandinsky 6 speed ablation, oh-my-gpu.com, section
 * "토큰 수의 제곱으로 느는 어텐션 비용": 720p, 121 frames -> 32 x 48 x 80,
 * 122,880 tokens with padding).  They are grouped into 64-token blocks,
 * either fixed 4x4x4 cubes or, per 8x8x8 region, a 64-token box whose
 * short side lies on the axis along which K changes most (same page,
 * section "같은 계산량 안에서 볼 곳을 고르는 Prism").  Q and K are mean-pooled
 * per block; every query block keeps the key blocks with the highest
 * pooled score (sparsity 0.75 keeps 25 %, 480 of 1,920), and attention runs
 * over the kept 64 x 64 tiles only, so empty tiles are skipped outright
 * (Sparse VideoGen on TPU, aibase.it, section "이론적 sparsity와 물리적
 * sparsity의 차이").  An optional conditioning prefix (text, reference
 * image, reference audio) sits in segment-pure blocks that every query
 * keeps and whose queries attend densely (Ref2VA VSA, pulmap.app, section
 * "조건 토큰은 왜 다르게 다루나").
 *
 * The call sequence for one attention layer:
 *   bsa_layout -> bsa_permute (Q, K, V) -> bsa_pool -> bsa_select_topk
 *   -> bsa_sparse_attn_fwd -> bsa_unpermute
 * (bsa_permute_pool does the permutes and the pooling in one pass).
 * bsa_dense_attn_fwd is the same attention kernel over every tile (the
 * speed-up denominator).
 *
 * Conventions (every entry point):
 *   - The caller owns all memory.  The library allocates no device memory
 *     (its one static device array, for bsa_forward_noalloc, comes with the
 *     loaded code); sizes of every buffer come from bsa_query_sizes.
 *   - Device pointers must be 16-byte aligned (index lists and counts: 4
 *     bytes); the innermost (head_dim) dimension of every tensor is
 *     contiguous.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *     void*; NULL = legacy default stream).  Arguments are validated on the
 *     host before anything is launched: on any error nothing is launched and
 *     a bsa_status other than BSA_OK is returned; bsa_last_error() then
 *     gives a message (per calling thread).
 *   - Errors found on the device (a bounded wait that ran out) are written
 *     to the optional `dev_status` int32 device word as a bsa_status value;
 *     the word is never cleared by the library.  With dev_status == NULL
 *     they go to one library-owned word per device instead, shared by every
 *     such call; nothing reports it unless the caller reads it with
 *     bsa_take_default_status.
 *   - Token order "raster": prefix segment s occupies
 *     [off_s, off_s + pad64(prefix_len[s])) with its pad tokens at the end,
 *     then video token (t, y, x) sits at P + (t*H + y)*W + x, where
 *     P = sum of padded segment lengths and N = P + T*H*W.
 *     Token order "perm" (block order): slot s of block j = j*64 + s; the
 *     prefix keeps raster order; video blocks follow the layout.
 *   - Raster tensors are [B, N, heads, head_dim] bf16 addressed with element
 *     strides (stride_b, stride_n, stride_h); permuted tensors are
 *     contiguous [B, heads, N, head_dim] bf16.
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BSA_MAX_PREFIX_SEGMENTS 8

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad scalar */
  BSA_ERR_SHAPE = 2,       /* grid, block or prefix geometry not allowed */
  BSA_ERR_UNSUPPORTED = 3, /* head_dim other than 64 or 128, more than 6,144
                              64-token blocks per sequence (the attention
                              kernel's on-chip step table), more video blocks
                              than on-chip selection holds, no sm_100 GPU */
  BSA_ERR_WORKSPACE = 4,   /* a caller buffer is too small */
  BSA_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed */
  BSA_ERR_TIMEOUT = 6,     /* device-side bounded wait ran out */
  BSA_ERR_HOST_MEMORY = 7  /* a host-side allocation failed */
} bsa_status;

typedef enum {
  BSA_BLOCK_FIXED_444 = 0,  /* 4x4x4 token cubes, blocks in (bt,bh,bw) raster order */
  BSA_BLOCK_DYNAMIC_888 = 1 /* one of 7 64-token shapes per 8x8x8 region */
} bsa_block_mode;

/* One attention call.  Every field must be set; there are no defaults. */
typedef struct {
  int32_t B, heads, head_dim;    /* head_dim in {64, 128} */
  int32_t T, H, W;               /* padded grid; multiples of 4 (8 in dynamic mode) */
  int32_t T_valid, H_valid, W_valid; /* valid extents; trailing indices are pad.
                                        T-T_valid etc. < 4 (fixed) / < 2 (dynamic)
                                        so that no block is all pad */
  int32_t n_prefix_segments;     /* 0..BSA_MAX_PREFIX_SEGMENTS */
  int32_t prefix_len[BSA_MAX_PREFIX_SEGMENTS]; /* valid tokens per segment (>= 1) */
  int32_t keep_blocks;           /* video key blocks kept per video query block,
                                    1..n_video_blocks (see bsa_keep_count) */
  int32_t block_mode;            /* bsa_block_mode */
  float dyn_tau;                 /* dynamic mode: a region keeps 4x4x4 when
                                    max(v) < dyn_tau*min(v); finite, >= 1 */
  float softmax_scale;           /* logit scale, finite and > 0 (1/sqrt(head_dim)
                                    for standard attention) */
} bsa_problem;

/* Sizes derived from a problem (all byte counts are for the whole batch). */
typedef struct {
  int64_t n_tokens;          /* N = P + T*H*W */
  int64_t n_prefix_tokens;   /* P */
  int64_t n_blocks;          /* nb = N / 64 */
  int64_t n_prefix_blocks;   /* nbp = P / 64 */
  int64_t n_video_blocks;    /* nbv = T*H*W / 64 */
  int64_t n_regions;         /* dynamic mode: (T/8)(H/8)(W/8); else 0 */
  int64_t list_capacity;     /* kcap = nbp + keep_blocks: ints per index-list row */
  size_t layout_bytes;       /* layout buffer (bsa_layout output) */
  size_t perm_tensor_bytes;  /* one permuted tensor [B, heads, N, head_dim] bf16 */
  size_t raster_tensor_bytes;/* one dense raster tensor [B, N, heads, head_dim] bf16 */
  size_t pool_bytes;         /* one pooled tensor [B, heads, nb, head_dim] fp32 */
  size_t idx_bytes;          /* index lists [B, heads, nb, kcap] int32 */
  size_t cnt_bytes;          /* list lengths [B, heads, nb] int32 */
} bsa_sizes;

/* Kept video key blocks per video query block for a keep ratio r = 1 - sparsity:
 * max(1, ceil(r*n - 1e-9)), at most n (Prism speed ablation, section
 * "같은 계산량 안에서 볼 곳을 고르는 Prism": sparsity 0.75 -> 480 of 1,920).
 * Returns -1 for n < 1 or r outside [0, 1] or not finite.  Host only. */
int32_t bsa_keep_count(int32_t n_blocks, double keep_ratio);

/* Validate `prob` and fill `out`.  Host only; no CUDA call. */
bsa_status bsa_query_sizes(const bsa_problem* prob, bsa_sizes* out);

/* Build the block layout into `layout_buf` (layout_bytes, caller-owned).
 * Fixed mode: a closed-form permutation; k_raster may be NULL.
 * Dynamic mode (the Prism section on 8x8x8 regions): per (batch, region)
 *   v_a = mean |K(p+e_a) - K(p)| over heads, channels and adjacent valid
 *   in-region token pairs along axis a (fp32 sums); the region keeps 4x4x4
 *   when max(v) < dyn_tau*min(v) or max(v) == 0, otherwise the axes ranked
 *   by (v descending, t<h<w) get block sides 2, 4, 8.  The shape is shared
 *   by all heads.  k_raster is K in raster order with element strides
 *   (stride_b, stride_n, stride_h).
 * layout_buf holds: slot->raster and raster->slot maps (int32 [B, N], bit 31
 * set for pad tokens), per-block valid-slot masks (uint64 [B, nb]) and
 * counts (int32 [B, nb]), and shape codes (uint8 [B, n_regions]). */
bsa_status bsa_layout(const bsa_problem* prob, const void* k_raster, int64_t stride_b,
                      int64_t stride_n, int64_t stride_h, void* layout_buf, void* stream);

/* Gather one raster tensor into block order: x_perm[b, h, s, :] =
 * x_raster[b, perm[b][s], h, :], pad slots written as 0 (token permutation,
 * Sparse VideoGen on TPU, section "실무에서 배울 최적화 기준"). */
bsa_status bsa_permute(const bsa_problem* prob, const void* layout_buf, const void* x_raster,
                       int64_t stride_b, int64_t stride_n, int64_t stride_h, void* x_perm,
                       void* stream);

/* Block means of Q and K over each block's valid tokens, fp32
 * [B, heads, nb, head_dim] (Prism section: a block is judged by the mean of
 * its 64 tokens). */
bsa_status bsa_pool(const bsa_problem* prob, const void* layout_buf, const void* q_perm,
                    const void* k_perm, float* q_pool, float* k_pool, void* stream);

/* bsa_permute of Q, K and V and bsa_pool in one pass: the block means are
 * summed from the rows as they are moved, so the permuted Q and K are not
 * read back (the Prism section's block means; Sparse VideoGen on TPU,
 * aibase.it, section "실무에서 배울 최적화 기준": the permutation is part of
 * the cost to be measured).  Outputs equal those of the separate calls bit
 * for bit.  q_raster, k_raster and v_raster share the element strides
 * (stride_b, stride_n, stride_h); q_perm, k_perm, v_perm, q_pool and k_pool
 * are laid out as for bsa_permute and bsa_pool. */
bsa_status bsa_permute_pool(const bsa_problem* prob, const void* layout_buf, const void* q_raster,
                            const void* k_raster, const void* v_raster, int64_t stride_b,
                            int64_t stride_n, int64_t stride_h, void* q_perm, void* k_perm,
                            void* v_perm, float* q_pool, float* k_pool, void* stream);

/* Per (batch, head) and video query block i: scores S[i, j] = q_pool[i] .
 * k_pool[j] (fp32) over video key blocks j; keep the keep_blocks best by
 * (score descending, index ascending).  Row i of idx [B, heads, nb, kcap]
 * receives every prefix block then the kept video blocks, ascending;
 * cnt[i] = nbp + keep_blocks.  Prefix query blocks attend densely:
 * cnt = -1 and their idx row is left untouched (Ref2VA VSA, section
 * "조건 토큰은 왜 다르게 다루나").  Up to 2,048 video blocks the scores come
 * from the tensor cores (tf32 with every operand split into two tf32 parts:
 * each channel's product within 3 * 2^-20 |q_c||k_c| of the exact one; lists can
 * differ from an fp32 FMA evaluation only between blocks whose scores are
 * that close); above that, from fp32 FMA chains.  A bounded internal wait
 * that runs out reports BSA_ERR_TIMEOUT through bsa_take_default_status. */
bsa_status bsa_select_topk(const bsa_problem* prob, const float* q_pool, const float* k_pool,
                           int32_t* idx, int32_t* cnt, void* stream);

/* bsa_select_topk with a learned-gate score (Ref2VA VSA, pulmap.app, section
 * "토큰 75%를 건너뛰는 VSA": a trained predictor, to_gate_compress, picks the
 * tiles that matter instead of a fixed rule).  Each pooled query row is
 * mapped through its head's gate matrix before scoring:
 *   S[i, j] = sum_c (sum_e G[h][c][e] q_pool[i][e]) k_pool[j][c]   (fp32)
 * gate: device fp32 [heads][head_dim][head_dim], row-major, caller-owned.
 * G = identity gives exactly the bsa_select_topk lists.  Everything else
 * (prefix handling, ties, output format) as bsa_select_topk. */
bsa_status bsa_select_topk_gated(const bsa_problem* prob, const float* q_pool,
                                 const float* k_pool, const float* gate, int32_t* idx,
                                 int32_t* cnt, void* stream);

/* Block-sparse attention over the kept tiles: for each query block i and
 * each key block j in idx row i (all blocks when cnt[i] == -1), logits
 * softmax_scale * q.k over the valid keys of j, online softmax, O = P V,
 * normalised; pad query rows are written as 0.  Inputs and output are in
 * block order [B, heads, N, head_dim] bf16; accumulation is fp32.
 * Index rows must be strictly ascending with entries in [0, nb). */
bsa_status bsa_sparse_attn_fwd(const bsa_problem* prob, const void* layout_buf,
                               const void* q_perm, const void* k_perm, const void* v_perm,
                               const int32_t* idx, const int32_t* cnt, void* o_perm,
                               int32_t* dev_status, void* stream);

/* ---- training: the same sparse attention, forward with statistics and
 * backward (Prism / Kandinsky 6 speed ablation, section "같은 계산량 안에서
 * 볼 곳을 고르는 Prism": the sparse attention also trains, a 2K training step
 * from 26.5 to 10.6 minutes). */

/* bsa_sparse_attn_fwd that also writes each query row's log-sum-exp in the
 * exp2 domain, lse[b, h, slot] = m + log2(l) with P = exp2(s * softmax_scale
 * * log2(e) - lse) (fp32 [B, heads, N], block order, 16-byte aligned; +inf
 * for pad rows), which the backward reuses. */
bsa_status bsa_sparse_attn_fwd_lse(const bsa_problem* prob, const void* layout_buf,
                                   const void* q_perm, const void* k_perm, const void* v_perm,
                                   const int32_t* idx, const int32_t* cnt, void* o_perm,
                                   float* lse, int32_t* dev_status, void* stream);

/* Bytes of the backward's workspace (rowsum(dO * O) per row and the
 * transposed key-block -> query-block bitmaps).  Host only. */
bsa_status bsa_query_bwd_workspace(const bsa_problem* prob, size_t* bytes);

/* Gradients of the block-sparse attention over the same kept tiles, all in
 * block order [B, heads, N, head_dim] bf16 (use bsa_permute on dO and
 * bsa_unpermute on the gradients for raster order):
 *   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
 *   dQ = softmax_scale * dS K,  dK = softmax_scale * dS^T Q,
 * with P recomputed from lse (bsa_sparse_attn_fwd_lse) over the kept tiles
 * of idx/cnt (the forward's lists).  Pad tokens get zero gradients.
 * workspace: caller-owned, ws_bytes >= bsa_query_bwd_workspace (16-byte
 * aligned), else BSA_ERR_WORKSPACE.  Accumulation is fp32 in tensor memory;
 * each gradient element is written once (no atomics), so results are
 * deterministic. */
bsa_status bsa_sparse_attn_bwd(const bsa_problem* prob, const void* layout_buf,
                               const void* q_perm, const void* k_perm, const void* v_perm,
                               const void* o_perm, const void* do_perm, const float* lse,
                               const int32_t* idx, const int32_t* cnt, void* dq_perm,
                               void* dk_perm, void* dv_perm, void* workspace, size_t ws_bytes,
                               int32_t* dev_status, void* stream);

/* The same attention over every tile (pad keys masked): the dense comparator. */
bsa_status bsa_dense_attn_fwd(const bsa_problem* prob, const void* layout_buf,
                              const void* q_perm, const void* k_perm, const void* v_perm,
                              void* o_perm, int32_t* dev_status, void* stream);

/* Scatter block-ordered rows back to raster order: o_raster[b, n, h, :] =
 * o_perm[b, h, iperm[b][n], :]; pad tokens written as 0. */
bsa_status bsa_unpermute(const bsa_problem* prob, const void* layout_buf, const void* o_perm,
                         void* o_raster, int64_t stride_b, int64_t stride_n, int64_t stride_h,
                         void* stream);

/* ---- raster order: the same call without permuted copies -----------------
 * The permutation exists only so that every kept block is one contiguous
 * tile (Sparse VideoGen on TPU, section "실무에서 배울 최적화 기준": token
 * order decides whether a sparse pattern pays).  With these two calls the
 * kernels read the tiles straight out of the raster tensors instead, so
 * bsa_permute and bsa_unpermute, and the four permuted buffers, drop out:
 *   bsa_layout -> bsa_pool_raster -> bsa_select_topk
 *   -> bsa_sparse_attn_fwd_raster
 * Results equal the permuted sequence's (pooled means bit for bit; the
 * attention output up to the order of fp32 accumulation, which is the same). */

/* Block means of raster Q and K (the bsa_pool definition), read through the
 * layout's slot -> raster map.  q_raster and k_raster share the element
 * strides (stride_b, stride_n, stride_h). */
bsa_status bsa_pool_raster(const bsa_problem* prob, const void* layout_buf, const void* q_raster,
                           const void* k_raster, int64_t stride_b, int64_t stride_n,
                           int64_t stride_h, float* q_pool, float* k_pool, void* stream);

/* bsa_sparse_attn_fwd on raster tensors.  Each kept K or V block is loaded
 * as one TMA box of the [B, T, H, W, heads*head_dim] grid (video blocks;
 * one box shape per block shape) or as 64 consecutive tokens (prefix
 * blocks); query rows are read and output rows written through the
 * layout's slot -> raster map.
 *   q_raster, k_raster, v_raster  [B, N, heads, head_dim] bf16 sharing the
 *                                 strides (stride_b, stride_n, stride_h);
 *                                 stride_h must equal head_dim (heads
 *                                 contiguous in a token row, as a fused QKV
 *                                 projection leaves them), else
 *                                 BSA_ERR_UNSUPPORTED
 *   o_raster                      output [B, N, heads, head_dim] with its own
 *                                 strides; pad tokens are written as 0
 * Pad tokens of the raster K and V are read (and masked out of the
 * softmax), so they must hold finite values; a pad row of V multiplies a
 * probability of exactly 0. */
bsa_status bsa_sparse_attn_fwd_raster(const bsa_problem* prob, const void* layout_buf,
                                      const void* q_raster, const void* k_raster,
                                      const void* v_raster, int64_t stride_b, int64_t stride_n,
                                      int64_t stride_h, const int32_t* idx, const int32_t* cnt,
                                      void* o_raster, int64_t o_stride_b, int64_t o_stride_n,
                                      int64_t o_stride_h, int32_t* dev_status, void* stream);

/* Window heads: attention under a per-head spatio-temporal window instead of
 * top-k lists, with tiles classed full / boundary / empty (Sparse VideoGen on
 * TPU, sections "Sparse VideoGen의 핵심 아이디어": spatial heads look within
 * nearby frames, temporal heads at the same place across frames; and
 * "이론적 sparsity와 물리적 sparsity의 차이": empty tiles are skipped, only
 * boundary tiles need an element mask).
 *   windows  device int32 [heads][3] = (w_t, w_y, w_x); a negative entry
 *            leaves that axis unbounded.  Query token (t, y, x) attends to
 *            video key (t', y', x') when |t'-t| <= w_t, |y'-y| <= w_y and
 *            |x'-x| <= w_x; every query attends to every prefix key and
 *            prefix queries attend to every key; pad keys are excluded and
 *            pad query rows are 0.  A spatial head is (w, -1, -1), a
 *            temporal head (-1, r, r).
 * A query block walks only the key blocks whose box its box can reach
 * through the window (non-empty tiles); inside a tile each query row masks
 * the keys outside its window (boundary tiles), while full tiles need no
 * mask.  Other arguments as in bsa_sparse_attn_fwd_raster (prob.keep_blocks
 * is validated but unused). */
bsa_status bsa_window_attn_fwd_raster(const bsa_problem* prob, const void* layout_buf,
                                      const void* q_raster, const void* k_raster,
                                      const void* v_raster, int64_t stride_b, int64_t stride_n,
                                      int64_t stride_h, const int32_t* windows, void* o_raster,
                                      int64_t o_stride_b, int64_t o_stride_n, int64_t o_stride_h,
                                      int32_t* dev_status, void* stream);

/* Histogram of video blocks by shape code over the whole batch (hist7[0]
 * counts 4x4x4 blocks; each dynamic region adds 8 blocks of its code), the
 * block-shape log of the Prism speed ablation (section "동적 블록을 켜도
 * 그대로였던 속도").  Dynamic mode synchronises `stream` and copies the codes
 * to the host.  Fixed mode: hist7[0] = B * n_video_blocks, no CUDA call. */
bsa_status bsa_layout_stats(const bsa_problem* prob, const void* layout_buf, int64_t hist7[7],
                            void* stream);

/* Device buffers of one whole call (caller-owned, sizes from
 * bsa_query_sizes): raster Q, K, V, O (raster_tensor_bytes each, contiguous
 * [B, N, heads, head_dim]), permuted Q, K, V, O (perm_tensor_bytes each),
 * the layout (layout_bytes), pooled Q and K (pool_bytes each), index lists
 * (idx_bytes) and counts (cnt_bytes).  16-byte aligned (idx and cnt: 4).
 * The four permuted buffers may all be NULL: bsa_forward_host then runs the
 * permute-free sequence (bsa_pool_raster, bsa_sparse_attn_fwd_raster) on the
 * raster buffers and needs no permuted copies. */
typedef struct bsa_device_buffers {
  void* q_raster;
  void* k_raster;
  void* v_raster;
  void* o_raster;
  void* q_perm;
  void* k_perm;
  void* v_perm;
  void* o_perm;
  void* layout_buf;
  float* q_pool;
  float* k_pool;
  int32_t* idx;
  int32_t* cnt;
} bsa_device_buffers;

/* The whole call (layout, permute, pool, top-k selection, sparse attention,
 * unpermute: the sequence above) for Q, K, V and O in HOST memory, with the
 * transfers overlapped with the computation.  Heads are processed in groups
 * of `heads_per_group`.  Group g+1 is copied to the device while group g is
 * computed and group g-1's output is copied back, on two library-owned
 * copy streams tied to `stream` by events.  Even groups compute on `stream`,
 * odd ones on a third library-owned stream, so that one group's first
 * kernels run on the SMs that the previous group's last kernels leave idle.
 * The dynamic layout needs every head of K, so in dynamic mode K is copied
 * whole first.
 *   q_host, k_host, v_host  [B, N, heads, head_dim] bf16, contiguous, host
 *                           memory (page-locked memory lets copies overlap)
 *   o_host                  same layout, written; pad tokens are 0
 *   buf                     device buffers as described above
 *   heads_per_group         1..heads, must divide heads
 *   dev_status, stream      as in bsa_sparse_attn_fwd; the call is complete
 *                           when the work queued on `stream` is complete.
 * Results equal the step-by-step sequence up to the order of the attention
 * kernel's fp32 accumulation (a group's CTAs start their key walks at
 * different blocks).  Buffer slices: group g uses the g-th 1/groups of the
 * permuted, pooled, idx and cnt buffers, each laid out as for a problem
 * with heads = heads_per_group.  Every argument is validated before
 * anything is queued; a CUDA error while queueing (rare) returns
 * BSA_ERR_CUDA and may leave part of the work queued.  The library creates
 * its two copy streams per device on first use and keeps them; it
 * allocates no memory. */
bsa_status bsa_forward_host(const bsa_problem* prob, const void* q_host, const void* k_host,
                            const void* v_host, void* o_host, const bsa_device_buffers* buf,
                            int32_t heads_per_group, int32_t* dev_status, void* stream);

/* Test hook for the device-side timeout path.  While enabled (nonzero),
 * attention launches issue no PV product (forward) and no accumulation
 * (backward: dQ += dS K, dV += P^T dO, dK += dS^T Q), so a bounded wait on
 * the first of them runs out after 2 s.  The kernel then writes
 * BSA_ERR_TIMEOUT to the status word, drains its copies and MMAs, frees
 * tensor memory and returns, and the CUDA context stays usable.  Output is
 * undefined for launches made while enabled.  The switch belongs to the
 * calling thread: only attention launches queued by that thread are
 * affected, never another thread's.  Off by default. */
bsa_status bsa_debug_stall_pv(int32_t enable);

/* The library-owned status word of the current device, which receives the
 * device-side errors of every call made with dev_status == NULL: waits for
 * the work queued on `stream` (which should include those calls), writes
 * the word to *out (BSA_OK when nothing went wrong) and clears it.  The word
 * is shared by all such calls on the device, so a caller that needs
 * per-call status passes its own dev_status instead. */
bsa_status bsa_take_default_status(int32_t* out, void* stream);

/* Size of the library's static scratch array used by bsa_forward_noalloc
 * (64 MiB per device that loads the library, held until the process exits). */
#define BSA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* The whole device-side call (layout, permute, pool, top-k selection, sparse
 * attention, unpermute) without any caller-provided intermediate buffer and
 * without allocating device memory.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate, such as a plugin or
 * FFI binding that receives only the tensors it is handed and cannot reach
 * its host application's allocator, a runtime whose device memory is fixed
 * at start-up, or a latency-bound loop that must not call cudaMalloc (which
 * can synchronise the device).
 *   q_raster, k_raster, v_raster  [B, N, heads, head_dim] bf16 on the device,
 *                                 sharing the element strides (stride_b,
 *                                 stride_n, stride_h)
 *   o_raster                      output, same layout with strides
 *                                 (o_stride_b, o_stride_n, o_stride_h); pad
 *                                 tokens are written as 0
 *   dev_status, stream            as in bsa_sparse_attn_fwd
 * The intermediates (layout, permuted Q/K/V/O, pooled means, index lists)
 * live in one static device array of BSA_NOALLOC_SCRATCH_BYTES owned by the
 * library.  A problem that needs more returns BSA_ERR_WORKSPACE with the
 * byte counts in bsa_last_error(), before anything is launched.  The first
 * call on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current); make that first call before any stream capture.
 * Every call on a device shares the one array and leaves its contents
 * behind; no part of it needs to start at zero, because each step writes
 * what later steps read.  Calls whose work overlaps on the GPU (other
 * streams, other threads) race on the array: serialise them.  The library
 * calls no cudaMalloc, cudaFree or allocating routine here. */
bsa_status bsa_forward_noalloc(const bsa_problem* prob, const void* q_raster,
                               const void* k_raster, const void* v_raster, int64_t stride_b,
                               int64_t stride_n, int64_t stride_h, void* o_raster,
                               int64_t o_stride_b, int64_t o_stride_n, int64_t o_stride_h,
                               int32_t* dev_status, void* stream);

/* Name of a status code. */
const char* bsa_status_string(bsa_status status);
/* Message of the last failed call on this thread ("" if none). */
const char* bsa_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H */

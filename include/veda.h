/*
 * veda.h -- C ABI of the Veda block-sparse attention hot path for NVIDIA B200 (sm_100a).
 *
 * The path (per attention call), as described on the "Miowtion" README (bullet
 * "Sparse acceleration (Veda)"; Key Features / Veda sparse attention) and on
 * "Deploying this checkpoint" (preamble; section 2, SM90 and SM100 paragraphs):
 *
 *   1. veda_permute_tiles          raster tokens -> 3D tiles of 128 tokens
 *   2. veda_tile_pool              mean / max / min of every Q and K tile
 *   3. veda_block_scores           per-head residual projection, (q tile, k tile) scores
 *   4. veda_select_blocks          Bresenham budgets, forced diagonal, full/partial lists
 *   5. veda_block_sparse_attn_fwd  attention over the listed key tiles only
 *   6. veda_unpermute              tiles -> raster order
 *
 * and, for training and for the predictor's teacher signal and its check ("Miowtion" README,
 * Key Features; "Deploying this checkpoint", sections 4 and 6):
 *
 *   veda_transpose_lists           query tiles of every key tile (the backward's lists)
 *   veda_block_sparse_attn_bwd     dQ, dK, dV over the same block lists
 *   veda_block_heat                per-block attention mass of dense attention
 *   veda_mask_quality              attention mass a mask keeps, recall against the oracle mask
 *   veda_rel_error                 relative output error per head (tile-plan search)
 *   veda_tile_plan_vote            the search's vote: kept tile shapes, one per head (host)
 *
 * and an FP8 variant of step 5 (the pages ship their predictor in FP8, "Deploying this
 * checkpoint", preamble and section 3; the attention variant is this library's):
 *
 *   veda_quantize_fp8              tiled bf16 -> e4m3 codes with one scale per (batch, head)
 *   veda_block_sparse_attn_fwd_fp8 step 5 with e4m3 Q / K / V and e4m3 P on the tensor cores
 *
 * Conventions shared by every call:
 *  - Ownership: the caller allocates and owns every buffer. Pointers named *_dev or
 *    documented as "device" must be device memory of the current CUDA device; the
 *    library allocates no device memory of its own (its status word is a static
 *    __device__ variable) and keeps no pointer after a call returns.
 *  - Synchrony: device calls only enqueue work on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) and return. Argument errors are detected on the host
 *    before anything is launched. Errors found by a kernel (bad index, NaN score,
 *    bounded wait that ran out) are recorded in a per-device status word and are
 *    reported by veda_check_device_status().
 *  - Architecture: every device call returns VEDA_ERR_UNSUPPORTED on a device other
 *    than compute capability 10.0 (B200) and for head_dim != 128. There is no dense,
 *    CPU or other fallback.
 *  - Types: Q/K/V/O are bf16 (uint16 storage); pooled features, projection weights,
 *    scores and LSE are fp32; indices and counts are int32. All arrays are dense
 *    row-major with the shapes given below.
 *  - Shapes: B batch, H heads, D = 128 head_dim, N raster tokens, nT tiles per head
 *    (the maximum over heads), Npad = nT * 128 tile slots per head.
 */
#ifndef VEDA_H_
#define VEDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VEDA_API __attribute__((visibility("default")))
#else
#define VEDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define VEDA_ABI_VERSION 1
#define VEDA_TILE 128          /* tokens per tile and rows per query tile */
#define VEDA_MAX_SEGMENTS 4    /* key segments with their own budget */
#define VEDA_MAX_TILES 2048    /* tiles per head accepted by veda_select_blocks */

typedef struct CUstream_st* veda_stream_t;   /* same type as cudaStream_t */

typedef enum veda_status {
  VEDA_OK = 0,
  VEDA_ERR_INVALID_ARG = 1,   /* a pointer, size or geometry argument is invalid */
  VEDA_ERR_UNSUPPORTED = 2,   /* not a compute-capability 10.0 device, or head_dim != 128 */
  VEDA_ERR_CUDA = 3,          /* a CUDA runtime call failed (see veda_last_error()) */
  VEDA_ERR_TIMEOUT = 4,       /* a kernel's bounded wait ran out; it stopped early */
  VEDA_ERR_DEVICE_CHECK = 5,  /* a kernel found a bad index, count or NaN score */
} veda_status;

/* One 3D tile shape; t*h*w must equal 128 ("3D tiles of 128 tokens"). */
typedef struct veda_tile_shape {
  int32_t t, h, w;
} veda_tile_shape;

/*
 * Token geometry of one attention call (host memory, read during the call only).
 * "Miowtion" README, Key Features / Veda sparse attention: up to two (t, h, w) tile
 * shapes per layer (per head), padded grids with valid-prefix tiles, segmented
 * reference/target budgets; NEWS 2026/09/23: per-head dynamic tile permutations.
 *   H            heads
 *   T, Hg, Wg    video grid (raster index of token (t,h,w) = (t*Hg + h)*Wg + w)
 *   n_tail       appended 1D tokens (e.g. audio), raster indices T*Hg*Wg + j
 *   head_shape   [H] tile shape of each head
 *   tile_order   NULL, or [H][order_stride]: head h's position p holds its video tile
 *                tile_order[h*order_stride + p] of the raster tile enumeration (the
 *                first n_video_tiles(h) entries must be a permutation)
 */
typedef struct veda_geometry {
  int32_t H;
  int32_t T, Hg, Wg;
  int32_t n_tail;
  const veda_tile_shape* head_shape;
  const int32_t* tile_order;
  int32_t order_stride;
} veda_geometry;

/* Library ABI version (VEDA_ABI_VERSION). */
VEDA_API int32_t veda_abi_version(void);

/* Static description of a status code. Never NULL. */
VEDA_API const char* veda_status_string(veda_status s);

/* Message of the last failing call on this host thread ("" if none). Never NULL. */
VEDA_API const char* veda_last_error(void);

/*
 * Sizes implied by a geometry (host only, no CUDA). Outputs (any may be NULL):
 *   N        raster tokens T*Hg*Wg + n_tail
 *   nT_max   tiles per head, maximum over heads (video tiles of the padded grid
 *            plus ceil(n_tail/128) tail tiles)
 *   Npad_max nT_max * 128
 * Returns VEDA_ERR_INVALID_ARG for a NULL geometry, negative sizes or a tile shape
 * whose volume is not 128.
 */
VEDA_API veda_status veda_geometry_sizes(const veda_geometry* g, int32_t* N, int32_t* nT_max,
                                int32_t* Npad_max);

/*
 * Step 1 plan: slot -> raster-token map of every head (host only, no CUDA).
 * "Miowtion" README, bullet "Sparse acceleration (Veda)" (tokens permuted into 3D
 * tiles of 128) and Key Features (padded grids with valid-prefix tiles). Each head's
 * grid is padded to a multiple of its tile shape; tiles are enumerated in raster
 * order of their tile coordinates (then reordered by tile_order); inside a tile the
 * valid tokens come first, in local (t,h,w) raster order; tail tokens follow as 1D
 * tiles of 128. Video tiles are key segment 0, tail tiles segment 1.
 * Outputs (host memory, caller-allocated):
 *   tile_map     [H][Npad_max] raster token of each slot, -1 for a pad slot
 *   tile_valid   [H][nT_max]   valid tokens of each tile (0 past the head's tiles)
 *   tile_segment [H][nT_max]   key segment of each tile
 *   nT_per_head  [H]           tiles of each head
 */
VEDA_API veda_status veda_build_tile_map(const veda_geometry* g, int32_t* tile_map, int32_t* tile_valid,
                                int32_t* tile_segment, int32_t* nT_per_head);

/*
 * Step 1: gather raster tokens into tile order (device).
 *   x        [B][N][H][D] bf16, raster order
 *   x_tiled  [B][H][Npad][D] bf16; slot s of head h receives x[b][tile_map[h][s]][h],
 *            or zeros when tile_map[h][s] < 0
 *   tile_map [H][Npad] int32 (device), values in [-1, N)
 * Out-of-range map entries are skipped (the slot is zeroed) and flagged as
 * VEDA_ERR_DEVICE_CHECK in the status word. x and x_tiled must not overlap.
 */
VEDA_API veda_status veda_permute_tiles(const void* x, void* x_tiled, const int32_t* tile_map,
                               int32_t B, int32_t N, int32_t H, int32_t D, int32_t Npad,
                               veda_stream_t stream);

/*
 * Step 2: mean, max and min of every tile over its valid slots, per channel (device).
 * "Miowtion" README, Key Features / Veda sparse attention: mean/max/min pooling.
 *   x_tiled    [B][H][nT*128][D] bf16 (output of step 1)
 *   tile_valid [H][nT] int32 (device), each in [0, 128]; a tile with 0 pools to zeros
 *   pooled     [B][H][nT][3][D] fp32: [..][0][:] mean, [1] max, [2] min
 * Sums are accumulated in fp32.
 */
VEDA_API veda_status veda_tile_pool(const void* x_tiled, const int32_t* tile_valid, float* pooled,
                           int32_t B, int32_t H, int32_t nT, int32_t D, veda_stream_t stream);

/* Workspace bytes veda_block_scores needs (the projected features of Q and K tiles). */
VEDA_API size_t veda_block_scores_workspace_bytes(int32_t B, int32_t H, int32_t nT, int32_t D);

/*
 * Step 3: score every (query tile, key tile) pair (device).
 * "Miowtion" README, bullet "Sparse acceleration (Veda)": a small per-head predictor
 * scores (query tile, key tile) pairs; Key Features: "mean/max/min pooling + per-head
 * residual projection". For head h with f = [mean; max; min] (3D values):
 *   qhat_i = mean_q,i + Wq[h] f_q,i      khat_j = mean_k,j + Wk[h] f_k,j
 *   scores[b][h][i][j] = qhat_i . khat_j
 *   pooled_q, pooled_k  [B][H][nT][3][D] fp32 (output of step 2)
 *   Wq, Wk              [H][D][3D] fp32
 *   scores              [B][H][nT][nT] fp32
 *   workspace           device scratch of >= veda_block_scores_workspace_bytes(...)
 *                       bytes, 256-byte aligned; clobbered
 * Products are accumulated in fp32.
 */
VEDA_API veda_status veda_block_scores(const float* pooled_q, const float* pooled_k, const float* Wq,
                              const float* Wk, float* scores, void* workspace,
                              size_t workspace_bytes, int32_t B, int32_t H, int32_t nT, int32_t D,
                              veda_stream_t stream);

/*
 * Allocation-free variant of veda_block_scores (no counterpart on the pages: it only
 * changes where the scratch memory comes from).
 *
 * Some callers cannot hand the library a workspace: a plugin inside a runtime that owns
 * every device allocation and gives the plugin no allocator, or latency-critical code
 * that must not call cudaMalloc (it can synchronise the whole device). This entry point
 * takes the same inputs and outputs as veda_block_scores but uses a scratch array that
 * is part of the library itself: a static __device__ array of
 * VEDA_NOALLOC_SCORES_BYTES (32 MiB) that every GPU holds from the moment it loads the
 * library until the process exits. It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *   - Limit: 2 * B * H * nT * D * 4 bytes must not exceed VEDA_NOALLOC_SCORES_BYTES
 *     (B * H * nT <= 32768 at D = 128); larger calls return VEDA_ERR_INVALID_ARG
 *     without launching anything.
 *   - Set-up: the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before
 *     any stream capture. The address is cached with the context it was looked up in;
 *     a call made in a different context (after cudaDeviceReset, say) looks it up again.
 *   - Sharing: every call on a device uses the same array and leaves its contents
 *     behind. Nothing in it needs to start at zero (each call overwrites all it reads),
 *     but calls whose executions overlap on the GPU (different streams without
 *     ordering, or concurrent host threads) race on it: order them.
 * Results equal veda_block_scores' for the same inputs.
 */
#define VEDA_NOALLOC_SCORES_BYTES (32u * 1024u * 1024u)
VEDA_API veda_status veda_block_scores_noalloc(const float* pooled_q, const float* pooled_k,
                                               const float* Wq, const float* Wk, float* scores,
                                               int32_t B, int32_t H, int32_t nT, int32_t D,
                                               veda_stream_t stream);

/*
 * Step 4: block lists of every query tile (device).
 * "Miowtion" README, Key Features / Veda sparse attention: equal-kernel-cost budgets
 * with Bresenham rounding, forced diagonal tiles, segmented budgets, full/partial
 * block lists; "Deploying this checkpoint", section 2 (SM90): the block mask is
 * packed into full/partial index lists.
 * For head h with n = nT_per_head[h] tiles and segment s holding nK_s of them, row
 * r < n takes k_rs = floor((r+1) nK_s p_s/q_s) - floor(r nK_s p_s/q_s) key tiles of
 * segment s (exact integer arithmetic; rho_s = rho_num[s]/rho_den[s]). In the row's
 * own segment k is raised to at least 1 and the diagonal tile r is taken first; the
 * other tiles are taken by score, highest first, equal scores (-0 == +0) to the lower
 * index. The chosen set is sorted ascending and split into full tiles
 * (tile_valid == 128) and partial tiles. Rows r >= n get empty lists.
 *   scores        [B][H][nT][nT] fp32 (device); a NaN among a row's candidates is
 *                 flagged VEDA_ERR_DEVICE_CHECK and ranked last
 *   tile_valid, tile_segment  [H][nT] int32 (device); segments in [0, n_segments)
 *   nT_per_head   [H] int32 (device), each in [0, nT]
 *   rho_num, rho_den  [n_segments] int32 (HOST), 0 <= num <= den, den >= 1
 *   full_cnt, part_cnt  [B][H][nT] int32 (device, out)
 *   full_idx, part_idx  [B][H][nT][list_stride] int32 (device, out); the first cnt
 *                 entries of a row are valid, the rest are left untouched
 *   list_stride   entries per row; must be >= min(nT, sum_s ceil(nT*rho_s) + 1)
 * Limits: nT <= VEDA_MAX_TILES, 1 <= n_segments <= VEDA_MAX_SEGMENTS.
 */
VEDA_API veda_status veda_select_blocks(const float* scores, const int32_t* tile_valid,
                               const int32_t* tile_segment, const int32_t* nT_per_head,
                               int32_t n_segments, const int32_t* rho_num, const int32_t* rho_den,
                               int32_t* full_cnt, int32_t* full_idx, int32_t* part_cnt,
                               int32_t* part_idx, int32_t list_stride, int32_t B, int32_t H,
                               int32_t nT, veda_stream_t stream);

/*
 * Step 5: block-sparse attention forward (device).
 * "Deploying this checkpoint", preamble (attention only visits the selected key
 * tiles) and section 2 (128 x 128 tiles at head_dim 128, one 128-row query tile per
 * block row); "Miowtion" README, Key Features (full/partial block lists, a single
 * mask function on partial blocks). For every (b, h, query tile r), with rows
 * i in [r*128, r*128+128) (pad rows included):
 *   o[i] = sum_j softmax_j(scale * q_i . k_j) v_j
 * over the valid slots (slot < tile_valid) of the key tiles listed in full_idx and
 * part_idx for that row; online softmax, fp32 scores/accumulators, bf16 output.
 *   q, k, v       [B][H][nT*128][128] bf16 (device, output of step 1), 16-byte aligned
 *   tile_valid    [H][nT] int32 (device)
 *   full_cnt/idx, part_cnt/idx  as produced by step 4 (device); key indices in [0, nT)
 *   o             [B][H][nT*128][128] bf16 (device, out); rows with no key tile get 0
 *   lse           NULL or [B][H][nT*128] fp32 (device, out): natural-log sum of
 *                 exp(scale * q.k) over the visited keys; -inf for rows with none
 * Out-of-range key indices or counts are flagged VEDA_ERR_DEVICE_CHECK and that
 * query tile's output is zeroed.
 */
VEDA_API veda_status veda_block_sparse_attn_fwd(const void* q, const void* k, const void* v,
                                       const int32_t* tile_valid, const int32_t* full_cnt,
                                       const int32_t* full_idx, const int32_t* part_cnt,
                                       const int32_t* part_idx, int32_t list_stride,
                                       float softmax_scale, void* o, float* lse, int32_t B,
                                       int32_t H, int32_t nT, int32_t D, veda_stream_t stream);

/*
 * Steps 1 and 2 fused (device; a variant of the two calls, which stay available): the tile
 * gather of veda_permute_tiles and, on the way, the mean / max / min of veda_tile_pool over
 * each tile's valid slots, so that the tiled tensor is not read a second time. Outputs are
 * those of the two calls: x_tiled bit-identical, pooled max / min identical, pooled mean
 * equal up to fp32 summation order.
 *   x, x_tiled, tile_map, B, N, H, D, Npad  as veda_permute_tiles
 *   tile_valid    [H][Npad/128] int32 (device)
 *   pooled        [B][H][Npad/128][3][128] fp32 (device, out)
 */
VEDA_API veda_status veda_permute_pool(const void* x, void* x_tiled, const int32_t* tile_map,
                              const int32_t* tile_valid, float* pooled, int32_t B, int32_t N, int32_t H,
                              int32_t D, int32_t Npad, veda_stream_t stream);

/*
 * Step 6: scatter tile-order rows back to raster order (device).
 *   o_tiled  [B][H][Npad][D] bf16
 *   o        [B][N][H][D] bf16; o[b][tile_map[h][s]][h] = o_tiled[b][h][s] for every
 *            slot with tile_map[h][s] >= 0; pad slots are dropped. Raster rows that no
 *            slot maps to are left untouched.
 *   tile_map [H][Npad] int32 (device)
 */
VEDA_API veda_status veda_unpermute(const void* o_tiled, void* o, const int32_t* tile_map, int32_t B,
                           int32_t N, int32_t H, int32_t D, int32_t Npad, veda_stream_t stream);

/*
 * Transposed block lists for the backward (device). "Miowtion" README, Key Features / Veda
 * sparse attention ("transposed backward lists"): for every (b, h, key tile j), the query
 * tiles i < nT_per_head[h] whose full or partial list (as produced by step 4) holds j, in
 * ascending order.
 *   full_cnt/idx, part_cnt/idx  forward lists (device), ascending per row, stride list_stride
 *   nT_per_head   [H] int32 (device)
 *   t_cnt         [B][H][nT] int32 (device, out); key tiles j >= nT_per_head[h] get 0
 *   t_idx         [B][H][nT][t_stride] int32 (device, out); t_stride >= nT
 * Bad counts are flagged VEDA_ERR_DEVICE_CHECK.
 */
VEDA_API veda_status veda_transpose_lists(const int32_t* full_cnt, const int32_t* full_idx,
                                 const int32_t* part_cnt, const int32_t* part_idx,
                                 int32_t list_stride, const int32_t* nT_per_head, int32_t* t_cnt,
                                 int32_t* t_idx, int32_t t_stride, int32_t B, int32_t H, int32_t nT,
                                 veda_stream_t stream);

/*
 * Backward of step 5 over the same block lists (device). For an output gradient dO, over
 * exactly the keys the forward visited, per query row q: P = exp(scale q.k - LSE_q),
 * D_q = dO_q . O_q, dS = P (dO_q . v - D_q); then
 *   dQ_q = scale * sum_k dS k,   dK_k = scale * sum_q dS q,   dV_k = sum_q P dO_q.
 * Pad query slots are treated as the forward treats them; pad key slots (slot >=
 * tile_valid) receive 0; query tiles with no listed key tile get dQ = 0 and key tiles
 * listed by no query tile get dK = dV = 0.
 *   q, k, v, o    [B][H][nT*128][128] bf16 (device): the forward's inputs and output
 *   dout          [B][H][nT*128][128] bf16 (device): dO in tile order (step 1 applied to
 *                 the raster gradient: pad slots 0)
 *   lse           [B][H][nT*128] fp32 (device): the forward's LSE
 *   tile_valid    [H][nT] int32 (device)
 *   full_cnt/idx, part_cnt/idx  the forward's lists; t_cnt/t_idx from veda_transpose_lists
 *   dq, dk, dv    [B][H][nT*128][128] bf16 (device, out)
 *   delta         B*H*nT*128 + 4 fp32 values (device): scratch; receives D, then the
 *                 kernels' work-queue counters (the library zeroes them)
 * All tensors 16-byte aligned. Out-of-range indices or counts are flagged
 * VEDA_ERR_DEVICE_CHECK.
 * Streams: D and dK/dV run on `stream`; dQ, which is independent of dK/dV, runs on a second
 * stream the library keeps for the device (created on the first call, kept until exit),
 * forked from and joined back into `stream` with events, so that the call is ordered on
 * `stream` like a single kernel. Calls from several host threads enqueue one at a time.
 */
VEDA_API veda_status veda_block_sparse_attn_bwd(const void* q, const void* k, const void* v,
                                       const void* o, const void* dout, const float* lse,
                                       const int32_t* tile_valid, const int32_t* full_cnt,
                                       const int32_t* full_idx, const int32_t* part_cnt,
                                       const int32_t* part_idx, int32_t list_stride,
                                       const int32_t* t_cnt, const int32_t* t_idx, int32_t t_stride,
                                       float softmax_scale, void* dq, void* dk, void* dv, float* delta,
                                       int32_t B, int32_t H, int32_t nT, int32_t D, veda_stream_t stream);

/*
 * FP8 variant, quantisation (device). "Deploying this checkpoint", preamble and section 3:
 * the predictor ships in FP8; the pages give no FP8 attention, so this variant quantises the
 * tiled Q, K, V per tensor and follows step 5 (the plainest reading). Tiled bf16 tensors ->
 * e4m3 codes (OCP FP8 E4M3, no infinities) with one scale per (batch, head): scale = max |x| / 448 and
 * code = e4m3(x * (448 / max |x|)), both in fp32, rounding to nearest even and saturating at
 * +-448; an all-zero (batch, head) gets scale 1. With transpose_tiles = 1 every 128 x 128
 * tile of the codes is stored transposed ([channel][key position]), the layout the FP8
 * attention takes for V: within every group of 16 positions, position 16m + 4c + e
 * (c, e in 0..3) holds key slot 16m + 2c + (e & 1) + 8 (e >> 1), the order in which the
 * attention's softmax packs P into tensor memory.
 *   x_tiled          [B][H][nT*128][D] bf16 (device)
 *   codes            [B][H][nT*128][D] uint8 e4m3 (device, out)
 *   scale            [B][H] fp32 (device, out; also used as scratch during the call)
 *   transpose_tiles  0 or 1
 * Three launches and one memset on `stream`. Errors: VEDA_ERR_INVALID_ARG (null pointer,
 * size <= 0, transpose_tiles not 0/1, x_tiled / codes not 16-byte aligned),
 * VEDA_ERR_UNSUPPORTED (D != 128, device other than sm_100).
 */
VEDA_API veda_status veda_quantize_fp8(const void* x_tiled, void* codes, float* scale, int32_t B, int32_t H,
                                       int32_t nT, int32_t D, int32_t transpose_tiles, veda_stream_t stream);

/*
 * FP8 variant of step 5 (device; same passages as veda_block_sparse_attn_fwd, FP8 as in
 * veda_quantize_fp8): the attention of veda_block_sparse_attn_fwd over the same lists, from
 * e4m3 operands. Each query tile visits its own key tile first when its list holds it, then
 * the rest in list order (the result depends on the order only through fp32 rounding). S = (Q codes)(K codes)^T on the tensor cores, times
 * q_scale * k_scale * softmax_scale; P = 2^(s - m + 7) enters P V as e4m3 (the row reference
 * m moves when a row maximum grows by more than 1.75 in log2 units, so that 2^7 P stays
 * below 448); O = (P V) * v_scale / l in bf16, LSE as in the bf16 call.
 *   q8, k8        [B][H][nT*128][D] uint8 e4m3 codes (veda_quantize_fp8, transpose_tiles 0)
 *   vt8           [B][H][nT*128][D] uint8 e4m3 codes of V with transposed tiles
 *                 (veda_quantize_fp8, transpose_tiles 1)
 *   q_scale, k_scale, v_scale   [B][H] fp32 (device) scales of the three tensors
 *   tile_valid, full_cnt, full_idx, part_cnt, part_idx, list_stride, softmax_scale, o, lse,
 *   B, H, nT, D   as veda_block_sparse_attn_fwd
 * Errors as veda_block_sparse_attn_fwd (codes and O 16-byte aligned).
 */
VEDA_API veda_status veda_block_sparse_attn_fwd_fp8(const void* q8, const void* k8, const void* vt8,
                                                    const float* q_scale, const float* k_scale,
                                                    const float* v_scale, const int32_t* tile_valid,
                                                    const int32_t* full_cnt, const int32_t* full_idx,
                                                    const int32_t* part_cnt, const int32_t* part_idx,
                                                    int32_t list_stride, float softmax_scale, void* o, float* lse,
                                                    int32_t B, int32_t H, int32_t nT, int32_t D,
                                                    veda_stream_t stream);

/*
 * Teacher block heat (device). "Miowtion" README, Key Features / Veda sparse attention:
 * the predictor is trained against teacher block heat from the dense LSE. For every
 * (b, h, query tile i) and every key tile j listed for it:
 *   heat[b][h][i][j] = (1 / n_i) * sum over valid query slots q of tile i
 *                      of sum over valid key slots k of tile j of exp(scale * q.k - lse[q])
 * with n_i = tile_valid[h][i]. With the lists of every key tile (step 4 at density 1/1)
 * and the LSE of step 5 run on those lists (dense attention), each valid row of heat sums
 * to 1.
 *   q, k          [B][H][nT*128][128] bf16 (device, output of step 1), 16-byte aligned
 *   tile_valid    [H][nT] int32 (device)
 *   full_cnt/idx, part_cnt/idx  block lists as produced by step 4 (device)
 *   lse           [B][H][nT*128] fp32 (device): natural-log LSE of the query rows
 *   heat          [B][H][nT][nT] fp32 (device, out): overwritten; entries of blocks not
 *                 listed are 0
 * Out-of-range key indices or counts are flagged VEDA_ERR_DEVICE_CHECK.
 */
VEDA_API veda_status veda_block_heat(const void* q, const void* k, const int32_t* tile_valid,
                            const int32_t* full_cnt, const int32_t* full_idx, const int32_t* part_cnt,
                            const int32_t* part_idx, int32_t list_stride, const float* lse,
                            float softmax_scale, float* heat, int32_t B, int32_t H, int32_t nT,
                            int32_t D, veda_stream_t stream);

/*
 * Quality of a block mask against the oracle mask (device). "Deploying this checkpoint",
 * section 4 (recall of the predictor against the oracle mask) and section 6 (the attention
 * mass an oracle mask keeps at a 10% keep ratio). The oracle mask is step 4 run on heat as
 * the score. For every row (b, h, i < nT_per_head[h]):
 *   mass_rows[b][h][i]   = sum of heat[b][h][i][j] over the predicted tiles j
 *   recall_rows[b][h][i] = |predicted & oracle| / |oracle| (0 when the oracle list is empty)
 * and totals[0..3] receive sum(tile_valid * mass), sum(tile_valid), sum(recall) and the
 * number of rows with a non-empty oracle list, so that the kept attention mass is
 * totals[0] / totals[1] and the mean recall totals[2] / totals[3]. Rows i >= nT_per_head[h]
 * get 0 and do not count.
 *   heat          [B][H][nT][nT] fp32 (device)
 *   tile_valid    [H][nT], nT_per_head [H] int32 (device)
 *   pred_*, orc_* block lists (device) with strides pred_stride, orc_stride
 *   mass_rows, recall_rows  [B][H][nT] fp32 (device, out); totals [4] fp32 (device, out,
 *                 overwritten)
 * Limits: nT <= VEDA_MAX_TILES. Bad counts or indices are flagged VEDA_ERR_DEVICE_CHECK.
 */
VEDA_API veda_status veda_mask_quality(const float* heat, const int32_t* tile_valid,
                              const int32_t* nT_per_head, const int32_t* pred_full_cnt,
                              const int32_t* pred_full_idx, const int32_t* pred_part_cnt,
                              const int32_t* pred_part_idx, int32_t pred_stride,
                              const int32_t* orc_full_cnt, const int32_t* orc_full_idx,
                              const int32_t* orc_part_cnt, const int32_t* orc_part_idx,
                              int32_t orc_stride, float* mass_rows, float* recall_rows, float* totals,
                              int32_t B, int32_t H, int32_t nT, veda_stream_t stream);

/*
 * Relative output error per head (device), the criterion of the oracle tile-plan search
 * ("Miowtion" README, Key Features: "relative output MSE under the best mask"):
 *   sums[2h]     = sum over b, tokens, channels of (o - o_ref)^2 for head h
 *   sums[2h + 1] = sum of o_ref^2 for head h
 * so that the relative error of head h is sums[2h] / sums[2h + 1].
 *   o, o_ref      [B][N][H][128] bf16 (device), raster order
 *   sums          [H][2] fp32 (device, out, overwritten); H <= 256
 */
VEDA_API veda_status veda_rel_error(const void* o, const void* o_ref, float* sums, int32_t B, int32_t N,
                           int32_t H, int32_t D, veda_stream_t stream);

/*
 * Vote of the oracle tile-plan search (host). "Miowtion" README, Key Features / Veda sparse
 * attention: tile shapes per layer by oracle search over the relative output MSE under the
 * best mask, majority vote, at most two shapes per layer.
 *   errors     [H][C] fp64 (host): relative output error of candidate c for head h
 *              (veda_rel_error's sums[2h] / sums[2h + 1] under that candidate's tiling)
 *   max_shapes shapes the layer may keep (the pages: 2)
 *   kept       [min(max_shapes, C)] int32 (host, out): kept candidates, ascending
 *   n_kept     (host, out): how many entries of kept are set (>= 1)
 *   assign     [H] int32 (host, out): the candidate each head takes
 * A head votes for its candidate of least error (the earliest of equal errors); the layer
 * keeps the most voted candidates, at most max_shapes and only voted ones (the earliest of
 * equal counts first); each head takes its least-error kept candidate (the earliest of
 * equal errors). NaN errors return VEDA_ERR_INVALID_ARG. No device work.
 */
VEDA_API veda_status veda_tile_plan_vote(const double* errors, int32_t H, int32_t C, int32_t max_shapes,
                                         int32_t* kept, int32_t* n_kept, int32_t* assign);

/*
 * Self-test of the library's failure detection (no counterpart on the pages). Launches
 * one thread that waits on an mbarrier nothing will ever arrive on, through the same
 * bounded-wait routine every kernel of the library uses, with a limit of `limit_us`
 * microseconds (1 .. 1,000,000). The wait gives up, records a timeout in the status word
 * and the kernel returns normally: the next veda_check_device_status() returns
 * VEDA_ERR_TIMEOUT (site 0xEE in the detail bits) and the context stays usable.
 */
VEDA_API veda_status veda_selftest_wait_timeout(uint32_t limit_us, veda_stream_t stream);

/*
 * Synchronise `stream`, then read and clear the current device's status word.
 * Returns VEDA_OK, VEDA_ERR_TIMEOUT, VEDA_ERR_DEVICE_CHECK or VEDA_ERR_CUDA.
 * detail (may be NULL) receives the raw status bits (see VEDA_STATUS_* in the
 * library source) -- 0 when clean.
 */
VEDA_API veda_status veda_check_device_status(veda_stream_t stream, uint32_t* detail);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* VEDA_H_ */

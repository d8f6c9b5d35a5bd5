/*
 * vdit.h -- C ABI of libvdit: spatio-temporal self-attention over the latent tokens of a
 * video diffusion transformer (frames x grid_h x grid_w patches), on one NVIDIA B200 (sm_100a).
 *
 * The library computes, for each head,
 *     o_i = sum_j softmax_j( (R(p_i) q_i) . (R(p_j) k_j) * scale  restricted to mask_ij ) v_j
 * where R(p) is a 3-D rotary embedding at token position p = (t, h, w) and mask is dense,
 * block-causal over chunks of latent frames, radial (distance-decayed), or block-causal AND
 * radial. Passages each call follows:
 *
 *   [CRoPE] "Accelerating Video Generation Inference with Sequential-Parallel 3D Positional
 *           Encoding Using a Global Time Index": section 2.B (global time index
 *           t_global = t_local + s, s = the chunk's start frame, so no rank or chunk asks another
 *           for its positions), section 2.A (KV cache of past chunks), section 2.C (RoPE
 *           frequencies precomputed into contiguous tables; QKV projection and RoPE fused).
 *   [TR]    "Timeripple: Accelerating vDiTs by Understanding the Spatio-Temporal Correlations
 *           in Latent Space", Metodologia 1 (RoPE channels form a temporal and two spatial groups).
 *   [DR]    "DynamicRad: Content-Adaptive Sparse Attention for Long Video Diffusion", section 2
 *           (radial window whose width decays with temporal distance by a factor gamma;
 *           long-range factor lambda; static-ratio mode: a fixed, content-free mask).
 *   [WF]    Wave Forcing / WaveRT news item (block-causal attention over chunks of latent frames,
 *           frame count divisible by 3; per-layer K/V cache refreshed chunk by chunk).
 *
 * Conventions shared by every call
 *   - Tensors are bf16, contiguous, in device memory, 16-byte aligned.
 *   - Token order inside a clip or chunk: frame-major, then patch row h, then column w; token n
 *     of a chunk starting at global frame s has t = s + n / (grid_h*grid_w), h and w local.
 *   - Q, K, V, O: [tokens, heads, head_dim].
 *   - KV cache: two buffers [heads, capacity_frames * grid_h * grid_w, head_dim]; global frame f
 *     lives in frame slot f mod capacity_frames (a ring holding the newest capacity_frames).
 *     The caller owns the buffers; zero them once before first use so that never-written slots
 *     hold finite values (they are masked out, but 0 * NaN would still poison O).
 *   - RoPE: head_dim splits into bands band_t, band_h, band_w (channels in that order from 0);
 *     each band is a 1-D rotary embedding over adjacent channel pairs (2j, 2j+1) turned by
 *     pos * theta^(-2j / band). Wan2.1 shapes: 44/42/42 at head_dim 128, 24/20/20 at 64.
 *   - Every call is asynchronous on the caller's CUDA stream (a cudaStream_t passed as void*;
 *     NULL = legacy default stream) except vdit_attn_plan, vdit_plan_info and vdit_plan_export,
 *     which are host-only, and vdit_get_status, which synchronises the device.
 *   - CUDA graphs: the first call of a launching entry point on a device may set up state there
 *     (the RoPE tables of a band set, kernel attributes); after one such call has run outside a
 *     capture, the launching calls (vdit_rope3d_apply, vdit_kv_append, vdit_kv_write,
 *     vdit_attn_forward and its variants on an uploaded plan, vdit_qkv_rope, the pack and push
 *     calls) neither allocate nor synchronise, so they may be captured into a CUDA graph on the
 *     caller's stream. A replay reads the captured pointers' current contents.
 *   - Errors: each call returns VDIT_OK (0) or a negative VDIT_ERR_* code and never throws;
 *     vdit_last_error() gives a thread-local message for the last failure on this thread.
 *     Argument checks happen before any launch, so a rejected call has no effect.
 */
#ifndef VDIT_H
#define VDIT_H

#if defined(__GNUC__)
#define VDIT_API __attribute__((visibility("default")))
#else
#define VDIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
    VDIT_OK = 0,
    VDIT_ERR_INVALID_ARG = -1,  /* null pointer, size out of range, inconsistent geometry     */
    VDIT_ERR_UNSUPPORTED = -2,  /* valid request the library does not implement (head_dim,...) */
    VDIT_ERR_MISALIGNED = -3,   /* a tensor pointer is not 16-byte aligned                    */
    VDIT_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed (message has the reason)  */
    VDIT_ERR_TIMEOUT = -5,      /* a bounded wait inside a kernel gave up (vdit_get_status)    */
    VDIT_ERR_NOT_UPLOADED = -6  /* vdit_attn_forward on a plan without vdit_plan_upload        */
};

/* Mask kinds (bit set). */
#define VDIT_MASK_DENSE 0
#define VDIT_MASK_BLOCK_CAUSAL 1
#define VDIT_MASK_RADIAL 2
#define VDIT_MASK_DYNAMIC 4

#define VDIT_TILE 128         /* query and key tile edge of the schedule and of the kernel   */
#define VDIT_MAX_FRAME 16383  /* largest global frame index the RoPE tables cover           */
#define VDIT_MAX_GRID 1024    /* largest grid_h and grid_w                                  */
#define VDIT_MAX_DT 1023      /* largest |t_q - t_k| a plan may contain                     */
#define VDIT_MAX_PEERS 16     /* most ranks of the peer-memory exchange (vdit_seq_*_peers)  */

/* Token grid, head layout and RoPE bands. heads >= 1; head_dim 64 or 128; bands even, > 0,
 * band_t + band_h + band_w == head_dim; theta > 1. */
typedef struct vdit_geom {
    int grid_h;   /* patch rows per latent frame (Wan2.1 480p: 30) */
    int grid_w;   /* patch columns per latent frame (Wan2.1 480p: 52) */
    int heads;
    int head_dim;
    int band_t, band_h, band_w;
    double theta; /* RoPE base, 10000 */
} vdit_geom;

/* Mask predicate for a query at (t_q, h_q, w_q) and a key at (t_k, h_k, w_k), global frames:
 *   BLOCK_CAUSAL ([WF]): kept iff floor(t_k / chunk_frames) <= floor(t_q / chunk_frames).
 *   RADIAL ([DR] sec. 2, static-ratio mode): with dt = |t_q - t_k| and
 *     d = max(|h_q - h_k|, |w_q - w_k|) (Chebyshev patch distance), kept iff
 *     (lambda > 0 and dt mod lambda == 0) or d <= w0 * 2^(-gamma_shift * dt).
 *   Both bits: AND of the two. 0: dense. Keys in never-written cache slots are never kept.
 *   DYNAMIC ([DR] sec. 2, dynamic-threshold mode; combined with any of the above, which then
 *     form the candidate set): the pre-softmax logits are the importance proxies. With
 *     z = scale * q . k over a query row's candidates and z_max their maximum, a candidate is
 *     kept iff z >= z_max - tau (tau > 0): the threshold adapts to each row. The attention
 *     kernel then makes two passes over the candidate tiles (logit maxima, then the softmax). */
typedef struct vdit_mask {
    int kind;          /* VDIT_MASK_* bits */
    int chunk_frames;  /* >= 1 when BLOCK_CAUSAL (Wan2.1 causal decode: 3) */
    long long w0;      /* >= 0 when RADIAL (52 on a 30 x 52 grid) */
    int gamma_shift;   /* >= 0; gamma = 2^-gamma_shift (1 -> gamma = 1/2) */
    int lambda;        /* >= 0; 0 disables the long-range frames (8) */
    double tau;        /* > 0 when DYNAMIC: logit margin below the row maximum (natural log) */
} vdit_mask;

/* Opaque attention schedule: the non-empty 128 x 128 (query x key) tiles of the mask. */
typedef struct vdit_plan vdit_plan;

typedef struct vdit_plan_info_t {
    int q_tokens;        /* query tokens = q_frames * grid_h * grid_w */
    int kv_tokens;       /* key slots = capacity_frames * grid_h * grid_w */
    int q_tiles, kv_tiles;
    int tiles;           /* listed (non-empty) tiles */
    int full_tiles;      /* listed tiles that are complete and wholly kept */
    long long kept_pairs;/* kept (query, key) pairs per head */
    int uploaded;        /* 1 after vdit_plan_upload */
    int kv_splits;       /* most key-range pieces of one (query block, head) unit in the CTA
                            schedule (1: no unit is cut), set by vdit_plan_upload */
    long long workspace_bytes; /* device scratch the plan holds for the pieces' partial results */
    long long mask_bytes;      /* keep masks of the partial tiles: 2 KiB per distinct block
                                  (identical blocks of several tiles are stored once; see
                                  vdit_plan_export_masks) */
    int work_entries;          /* entries of the kernel's work list (vdit_plan_export_work) */
    int single_patch_entries;  /* of which single-patch entries at unaligned key rows */
    long long work_mask_bytes; /* keep-mask blocks of the work list (2 KiB per distinct block) */
    int ctas;                  /* CTAs of the attention launch (set by vdit_plan_upload) */
    int cut_units;             /* (query block, head) units cut into key pieces (merged by a
                                  second kernel; set by vdit_plan_upload) */
} vdit_plan_info_t;

/* 3-D RoPE ([CRoPE] 2.B, [TR] Metodologia 1) of n_tokens consecutive tokens of one chunk whose
 * first token is at global frame start_frame, local patch (0, 0):
 *   y[n, head, :] = R(start_frame + n / (grid_h*grid_w), (n / grid_w) mod grid_h, n mod grid_w)
 *                   x[n, head, :].
 * x, y: device bf16 [n_tokens, heads, head_dim]; y == x (in place) is allowed, other overlap is
 * not. Math in fp32 with cos/sin from fp64-built tables, result rounded to bf16 (nearest-even).
 * n_tokens == 0 is a no-op. The first call per device and band set builds the tables
 * (allocates, synchronous); later calls only launch. start_frame + frames <= VDIT_MAX_FRAME + 1. */
VDIT_API int vdit_rope3d_apply(const vdit_geom* g, const void* x, void* y, int start_frame,
                      long long n_tokens, void* stream);

/* KV-cache append ([CRoPE] 2.A; [WF] cache refresh): for frames start_frame .. start_frame +
 * n_frames - 1 of one chunk, rotates K at its global positions (as vdit_rope3d_apply) and writes
 * K' and V (unchanged, bit-exact) into frame slot f mod capacity_frames of the caches.
 * k, v: device bf16 [n_frames * grid_h * grid_w, heads, head_dim]; k_cache, v_cache: device bf16
 * [heads, capacity_frames * grid_h * grid_w, head_dim], must not overlap k or v.
 * 1 <= n_frames <= capacity_frames. Window bookkeeping (which frames the cache holds) is the
 * caller's: it passes that window to vdit_attn_plan. */
VDIT_API int vdit_kv_append(const vdit_geom* g, void* k_cache, void* v_cache, int capacity_frames,
                   const void* k, const void* v, int start_frame, int n_frames, void* stream);

/* Ring write of an already rotated chunk ([CRoPE] 2.A cache of past chunks; 2.C, when the RoPE
 * ran in the producer, e.g. vdit_seq_pack with rotate): as vdit_kv_append, but K' is k_rotated
 * copied unchanged (bit-exact) instead of RoPE(k). Same arguments, layout and checks. */
VDIT_API int vdit_kv_write(const vdit_geom* g, void* k_cache, void* v_cache, int capacity_frames,
                           const void* k_rotated, const void* v, int start_frame, int n_frames,
                           void* stream);

/* Tile schedule (host only; [DR] sec. 2 and [WF] masks): queries are q_frames frames starting at
 * global frame q_start_frame; keys are the capacity_frames-frame ring cache holding global frames
 * kv_first_frame .. kv_last_frame (at most capacity_frames of them; other slots empty).
 * Lists, per 128-query tile in ascending order, the 128-key tiles (ascending) that contain a kept
 * pair, each flagged full iff it is complete and wholly kept. Built exactly from the rectangle
 * geometry of the tiles (integer arithmetic only), so it is identical to the tile list of the
 * explicit per-pair mask. *out receives a new plan owned by the caller (vdit_plan_destroy).
 * The query tiles are computed on up to 16 host threads (environment variable VDIT_PLAN_THREADS
 * overrides the count, 1 .. 64) and merged in tile order: the plan does not depend on it. */
VDIT_API int vdit_attn_plan(vdit_plan** out, const vdit_geom* g, const vdit_mask* m,
                   int q_start_frame, int q_frames,
                   int capacity_frames, int kv_first_frame, int kv_last_frame);

/* Copies the plan's schedule and tables to the current device (allocates; the copy is ordered on
 * stream). Idempotent. Required before vdit_attn_forward. It also fixes the CTA schedule of the
 * forward pass from the device's SM count (one CTA per SM at a time, launched in order, each
 * running one query block of two 128-query tiles of one head, a "unit", over its key list):
 * units run whole in head-major order, longest list first, except where the SMs would otherwise
 * idle at the end of the launch; there units are cut into key pieces that fill the SMs up to one
 * common level, found by bisection on a list-scheduling model of the launch. Each piece writes
 * its normalised fp32 partial output and log-sum-exp into a workspace slot held by the plan, and
 * a second kernel merges the pieces of every cut unit. The cut schedule is kept only when its
 * estimated time (makespan plus the partial results and the extra launch) is shorter; it never
 * uses more than 32768 / (head_dim + 1) slots (the no-allocation buffer's capacity), and the
 * dynamic-threshold mode, whose threshold needs each row's maximum over all its candidates, is
 * never cut. Forward calls that share one plan must therefore not run concurrently on different
 * streams. */
VDIT_API int vdit_plan_upload(vdit_plan* p, void* stream);

/* Host only: the CTA schedule vdit_plan_upload would fix for this plan on a device with
 * sm_count SMs (the rule above), without touching any device. *n_ctas and *n_cut_units receive
 * the counts; when cta (or merge) is not NULL it receives, per CTA in launch order, 5 ints
 * (query block, head, first entry of the piece within the unit's key list, entries, partial slot
 * or -1 for a unit that runs whole), and per cut unit 4 ints (query block, head, first slot,
 * pieces). Call once with NULL arrays for the sizes. */
VDIT_API int vdit_plan_export_schedule(const vdit_plan* p, int sm_count, int* n_ctas, int* n_cut_units,
                                       int* cta, int* merge);

VDIT_API int vdit_plan_info(const vdit_plan* p, vdit_plan_info_t* info);

/* Host copy of the schedule: row_ptr [q_tiles + 1], col_idx [tiles], full [tiles] (0/1). */
VDIT_API int vdit_plan_export(const vdit_plan* p, int* row_ptr, int* col_idx, unsigned char* full);

/* Host copy of the per-row keep masks the kernel applies to partial tiles (listed, not full),
 * computed on the host from the mask predicate above. For schedule entry i (the col_idx order of
 * vdit_plan_export), mask_index[i] is its block number, or -1 for a full tile; entries whose
 * masks are identical share one block. Block b is
 * words[512 b .. 512 b + 511]: for row r (query q_tile * 128 + r) and key kt * 128 + k, the pair
 * is kept iff bit (k mod 32) of words[512 b + 4 r + k / 32] is set. Rows and keys past the token
 * counts are 0. mask_index: [tiles]; words: [mask_bytes / 4] (may be NULL when mask_bytes is 0). */
VDIT_API int vdit_plan_export_masks(const vdit_plan* p, int* mask_index, unsigned int* words);

/* Host copy of the attention kernel's work list. It covers the same kept pairs as the schedule
 * above, each exactly once, but for radial masks on frames of at least 128 tokens the "same
 * patch" pairs of frame offsets whose radial window is a single patch (radius 0; [DR] sec. 2:
 * the window narrows with temporal distance) leave the aligned tiles: per query tile and such
 * offset one entry at an unaligned key row k holds them, query row r meeting key row k + r (the
 * same patch dt frames away), when that shortens the tile's list. For query tile qt, entries
 * row_ptr[qt] .. row_ptr[qt + 1] - 1 give key_row (first of 128 consecutive key rows) and
 * mask_index (a block of words, laid out as in vdit_plan_export_masks, or -1 for a complete,
 * wholly kept tile). row_ptr: [q_tiles + 1]; key_row, mask_index: [work_entries]; words:
 * [work_mask_bytes / 4] (may be NULL when that is 0). */
VDIT_API int vdit_plan_export_work(const vdit_plan* p, int* row_ptr, int* key_row, int* mask_index,
                                   unsigned int* words);

/* Frees the plan and its device copy (cudaFree). A forward launched on the plan reads that copy
 * until it completes: synchronise its stream before destroying the plan. NULL is a no-op. */
VDIT_API void vdit_plan_destroy(vdit_plan* p);

/* Attention forward over an uploaded plan. q: UNROTATED queries, device bf16
 * [q_tokens, heads, head_dim] (RoPE at the plan's query positions is applied while the Q tile is
 * staged into shared memory, [CRoPE] 2.C fusion). k_cache: rotated keys, v_cache: values, in the
 * ring layout above. o: device bf16 [q_tokens, heads, head_dim]. lse: optional device fp32
 * [heads, q_tokens] (natural-log sum of exp of the kept scaled scores) or NULL. scale > 0
 * (1/sqrt(head_dim) for the Wan2.1 shapes). Rows with no kept key get o = 0, lse = -inf.
 * head_dim 64 or 128 (the plan accepts no other). With VDIT_MASK_DYNAMIC the output is the
 * softmax over the kept candidates only, and lse their log-sum-exp. When vdit_get_status reports
 * VDIT_ERR_TIMEOUT for a call, its o and lse are unspecified. */
VDIT_API int vdit_attn_forward(const vdit_plan* p, const void* q, const void* k_cache, const void* v_cache,
                      void* o, float* lse, float scale, void* stream);

/* vdit_attn_forward with queries that are already rotated at the plan's query positions
 * ([CRoPE] 2.C: the RoPE runs in the producer of Q, e.g. vdit_seq_pack with rotate or
 * vdit_qkv_rope): the Q tile is loaded as given. Same arguments, results and error codes. */
VDIT_API int vdit_attn_forward_rotated(const vdit_plan* p, const void* q_rotated, const void* k_cache,
                                       const void* v_cache, void* o, float* lse, float scale,
                                       void* stream);

/* Attention forward that allocates nothing. No passage of the source pages has a counterpart:
 * this is a service for callers that cannot allocate device memory when they run attention,
 * for instance code running while another framework owns the GPU's memory through its own
 * pool (a cudaMalloc would fail or fragment it), or latency-critical loops that must not enter
 * the allocator or synchronise the device. Same arguments, results and error codes as
 * vdit_attn_forward; the difference is where the key-piece scratch lives: instead of the
 * workspace that vdit_plan_upload gives the plan, the partial results go to one fixed 32 MiB
 * device buffer that is part of the library (every GPU that loads the library holds it until
 * the process exits). The CTA schedule never uses more partial slots than the buffer holds
 * (256 x (head_dim + 1) x 4 bytes each), so every uploaded plan runs here.
 * The call itself makes no cudaMalloc / cudaFree or other allocating call: the plan must already
 * be uploaded, and the RoPE tables for its bands must already exist on the device (any earlier
 * vdit_kv_append, vdit_rope3d_apply or vdit_attn_forward builds them; otherwise
 * VDIT_ERR_INVALID_ARG). The buffer lives in the library's attention module: under CUDA's lazy
 * module loading that module, buffer included, is loaded on a device at its first use there, and
 * vdit_plan_upload makes that first use (it also resolves the buffer's device address with
 * cudaGetSymbolAddress), so this call, which needs a plan uploaded to the current device, only
 * launches kernels. All calls share the buffer and it keeps the last call's contents (nothing in it
 * needs to start at zero): calls whose kernels may overlap on the GPU, e.g. on two streams of one
 * device, race on it. After a call whose kernel timed out (VDIT_ERR_TIMEOUT) o and lse are
 * unspecified (the merge may have read an earlier call's partial results). */
VDIT_API int vdit_attn_forward_noalloc(const vdit_plan* p, const void* q, const void* k_cache,
                                       const void* v_cache, void* o, float* lse, float scale,
                                       void* stream);

/* Fused QKV projection + 3-D RoPE + KV-cache append ([CRoPE] 2.C: the QKV projections and the
 * causal RoPE in one kernel; 2.B global time index; 2.A cache of past chunks). For the tokens of
 * frames start_frame .. start_frame + n_frames - 1 of one chunk (local patch (0, 0) first):
 *   [Q | K | V] = X W^T in fp32 (tcgen05 tensor cores),
 *   q_out[n, head, :] = R(pos(n)) Q[n, head, :] (as vdit_rope3d_apply), bf16;
 *   K' = R(pos(n)) K and V go, bf16, to frame slot (frame mod capacity_frames) of k_cache /
 *   v_cache in the ring layout of vdit_kv_append.
 * x: device bf16 [n_frames * grid_h * grid_w, d_model] (row-major); w: device bf16
 * [3 * heads * head_dim, d_model] (the rows of W_q, then W_k, then W_v: the weight layout of a
 * linear layer); q_out: device bf16 [tokens, heads, head_dim]. No bias, no normalisation.
 * Requires heads * head_dim a multiple of 256, d_model a positive multiple of 8, 16-byte aligned
 * pointers and 1 <= n_frames <= capacity_frames. Builds the RoPE tables on first use per device
 * and band set (as vdit_rope3d_apply). */
VDIT_API int vdit_qkv_rope(const vdit_geom* g, const void* x, const void* w, int d_model,
                           int start_frame, int n_frames, void* q_out, void* k_cache, void* v_cache,
                           int capacity_frames, void* stream);

/* Sequence-to-head pack of the Ulysses-style exchange ([CRoPE] 2.A: the sequence is split over
 * the ranks; 2.B: the global time index, so each rank rotates its own tokens without asking
 * another for positions; 2.C: one fused all-to-all that gathers the sequence and splits the
 * heads, for Q, K and V together). Rank `rank` of n_ranks holds the chunk-local tokens
 * rank * n_tokens .. (rank + 1) * n_tokens - 1 of a chunk whose first frame is start_frame:
 * q, k, v: device bf16 [n_tokens, heads, head_dim] (g->heads = all heads; n_ranks divides it).
 * Writes, in one launch:
 *   send: device bf16 [n_ranks][3][n_tokens][heads / n_ranks][head_dim]; block r (r != rank) holds
 *     Q, K, V of the heads rank r owns (heads r * heads / n_ranks ..), ready to be sent to rank r
 *     as three contiguous messages; block `rank` is not written (may be NULL when n_ranks == 1);
 *   q_full, k_full, v_full: device bf16 [n_ranks * n_tokens][heads / n_ranks][head_dim], the
 *     head-sharded buffers of this rank: rows rank * n_tokens .. get this rank's own block; the
 *     exchange fills the other rows with the blocks the other ranks send.
 * With rotate != 0, Q and K are rotated at their global positions (as vdit_rope3d_apply); V is
 * always a bit-exact copy. The consumers of rotated data are vdit_kv_write (K', V into the ring)
 * and vdit_attn_forward_rotated. No output may overlap an input or another output. */
VDIT_API int vdit_seq_pack(const vdit_geom* g, const void* q, const void* k, const void* v, void* send,
                           void* q_full, void* k_full, void* v_full, int rank, int n_ranks,
                           int start_frame, long long n_tokens, int rotate, void* stream);

/* Head-to-sequence unpack of the return exchange after attention ([CRoPE] 2.A-2.C, the second
 * all-to-all of the sequence-parallel step). Rank `rank` computed attention for heads
 * rank * heads / n_ranks .. of all n_ranks * n_tokens tokens; rank r sent it the output rows of
 * the rank's own tokens for r's heads. recv: device bf16 [n_ranks][n_tokens][heads / n_ranks]
 * [head_dim] (block r from rank r; block `rank` unused, recv may be NULL when n_ranks == 1);
 * own: device bf16 [n_tokens][heads / n_ranks][head_dim], this rank's own output rows for its
 * tokens; out: device bf16 [n_tokens, heads, head_dim], out[n, r * heads / n_ranks + j, :] =
 * block r row n head j. A copy (bit-exact); out must not overlap recv or own. */
VDIT_API int vdit_seq_unpack(const vdit_geom* g, const void* recv, const void* own, void* out, int rank,
                             int n_ranks, long long n_tokens, void* stream);

/* The sequence-to-head exchange with the transfer fused into the pack ([CRoPE] 2.C "Comunicacao
 * Fundida": the causal RoPE and the all-to-all of Q, K and V in one operation): instead of filling
 * a send buffer for a library all-to-all, this rank's kernel writes the rows of its tokens
 * straight into every rank's head-sharded buffers. q_dst, k_dst, v_dst: HOST arrays of n_ranks
 * device addresses, valid in this process (rank r's q_full / k_full / v_full
 * [n_ranks * n_tokens][heads / n_ranks][head_dim]: this rank's own buffers for r == rank, peer
 * memory mapped over NVLink otherwise); this rank writes their rows rank * n_tokens ..
 * (rank + 1) * n_tokens - 1, rotating Q and K at their global positions when `rotate` (as
 * vdit_seq_pack). Every CTA ends with a system-scope memory fence, so once the kernels of all
 * ranks have completed (the caller's barrier between the ranks, ordered after this call on
 * `stream`), every rank's buffers hold the whole exchange. 1 <= n_ranks <= VDIT_MAX_PEERS,
 * n_ranks divides heads; this rank's own destinations must not overlap the inputs or each other
 * (peer ranges are not checked). */
VDIT_API int vdit_seq_pack_peers(const vdit_geom* g, const void* q, const void* k, const void* v,
                                 void* const* q_dst, void* const* k_dst, void* const* v_dst, int rank,
                                 int n_ranks, int start_frame, long long n_tokens, int rotate,
                                 void* stream);

/* The return exchange after attention in push form: o_full [n_ranks * n_tokens][heads / n_ranks]
 * [head_dim] holds this rank's heads' attention output for every rank's tokens; the rows of rank
 * s's tokens go to out_dst[s] (rank s's out [n_tokens][heads][head_dim], a HOST array of n_ranks
 * device addresses valid in this process) at this rank's head columns. A bit-exact copy; the same
 * fence and barrier rule as vdit_seq_pack_peers. */
VDIT_API int vdit_seq_push_peers(const vdit_geom* g, const void* o_full, void* const* out_dst, int rank,
                                 int n_ranks, long long n_tokens, void* stream);

/* Reads and clears the current device's kernel status word: *status = VDIT_OK, or
 * VDIT_ERR_TIMEOUT when a bounded wait in a kernel gave up since the last read. Synchronises the
 * device. */
VDIT_API int vdit_get_status(int* status);

/* Test hook for failure detection (no counterpart in the pages): while on != 0, the K/V producer
 * of every vdit_attn_forward launch issues no load, so the kernel's bounded waits expire (after
 * about 2 s), each CTA raises VDIT_ERR_TIMEOUT in the status word, drains and frees its tensor
 * memory and exits; the output is left unwritten and the CUDA context stays usable. Not for use
 * outside tests. */
VDIT_API void vdit_debug_skip_loads(int on);

/* Message of the last failed call on this thread ("" if none). Valid until the next call. */
VDIT_API const char* vdit_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* VDIT_H */

/*
 * vsa -- block-sparse attention over a flattened 3D video token grid, for B200
 * (sm_100a).  C ABI: plain pointers, sizes and status codes; no C++ types, no
 * exceptions cross it.
 *
 * Call order for one attention layer:
 *
 *   vsa_plan_create   mask specs + grid + 3D unit + tile shape
 *                     -> int8 tile map, per-query-block kv-tile lists,
 *                        tile-major token order (built on the GPU)
 *   vsa_permute       q, k, v  natural [B,Hh,N,D] -> tile-major [B,Hh,n_slots,D]
 *   vsa_sparse_attn_fwd       tile-major q,k,v -> tile-major o, lse
 *   vsa_unpermute     o  tile-major -> natural [B,Hh,N,D]
 *   vsa_svg_route     sampled-query profiling -> per-head spatial / temporal
 *                     flags; vsa_plan_apply_route switches the heads' specs
 *   vsa_ulysses_permute / _unpermute  sequence-sharded <-> head-sharded
 *                     exchange fused with the token order, across GPUs
 *
 * Sources (web pages on block-sparse video attention):
 *  [SVG-TPU] "Sparse VideoGen: accelerating video diffusion attention on TPU"
 *  [PSA]     "Parameterized Stripe Attention for Efficient Video Generation"
 *  [STA]     "Fast Video Generation with Sliding Tile Attention" (explainer)
 *  [VDS]     "Video diffusion long-sequence attention and sparsity", section 7
 *
 * Token order.  The natural order flattens (t,h,w) with t slowest:
 * n = (t*H + h)*W + w ([VDS] section 7.2).  The tile-major order pads each
 * axis to a multiple of the 3D unit (bt,bh,bw) (T' = ceil(T/bt)*bt, [PSA] key
 * design 2), lists units in (t,h,w) row-major order and, inside a unit, tokens
 * in (t,h,w) row-major order, so the tokens of a unit are contiguous ([STA]
 * section 3).  The slot count n_slots is the padded token count rounded up to
 * a multiple of max(128, q_tile, kv_tile); every slot that holds no real token
 * is padding.  Padding keys never receive attention weight ([SVG-TPU],
 * "aligning the sparse mask with execution").
 *
 * Memory.  The caller owns q, k, v, o and lse (device memory, contiguous,
 * 16-byte aligned).  A plan owns its device buffers; their shapes never
 * change after creation.  vsa_plan_build rewrites the maps in place, and
 * vsa_plan_apply_route rewrites the head specs on the device and then the
 * maps.  vsa_permute, vsa_permute_qkv, vsa_unpermute, vsa_sparse_attn_fwd,
 * vsa_svg_route (caller's workspace), vsa_plan_apply_route and the
 * vsa_ulysses_* exchange allocate nothing.
 *
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream).  Every launch is asynchronous on that stream; host-visible results
 * (tile maps, counts, status) are read by the calls documented as synchronous.
 *
 * Errors.  Every call returns VSA_OK (0) or a negative code.  Argument errors
 * are detected on the host before any launch.  A device-side watchdog turns a
 * wait that cannot complete into VSA_ERR_TIMEOUT, reported by
 * vsa_check_status; no kernel traps or spins without bound.
 */
#ifndef VSA_H
#define VSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VSA_VERSION 1

enum {
    VSA_OK = 0,
    VSA_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, bad enum      */
    VSA_ERR_UNSUPPORTED = -2, /* valid but not implemented: D, tile/unit shape  */
    VSA_ERR_ALIGNMENT = -3,   /* a tensor pointer is not 16-byte aligned        */
    VSA_ERR_CUDA = -4,        /* a CUDA runtime / driver call failed            */
    VSA_ERR_OOM = -5,         /* device allocation failed (vsa_plan_create)     */
    VSA_ERR_TIMEOUT = -6,     /* a kernel's bounded wait expired (watchdog)     */
    VSA_ERR_DEVICE = -7       /* a kernel flagged an inconsistent state         */
};

/* Mask families.
 *  FULL          keep every real key.
 *  SVG_SPATIAL   keep iff |t_k - t_q| <= rt                     ([SVG-TPU] SVG heads)
 *  SVG_TEMPORAL  keep iff |h_k - h_q| <= rh and |w_k - w_q| <= rw ([SVG-TPU] SVG heads)
 *  STA           keep iff the key's 3D unit lies in the query unit's window of
 *                kt x kh x kw units; the window is centred on the query's unit
 *                and shifted inward at the grid edge so that it always holds
 *                min(k, units on that axis) units ([STA] section 3, Eq. 4)
 *  STRIPE        keep iff (|t_k - t_q - To| mod Ts) <= Tw - 1 and
 *                (|s_k - s_q - So| mod Ss) <= Sw - 1, s = h*W + w ([PSA] key design 1)
 * With sink = 1 every query also keeps every real key of frame 0 (t_k = 0),
 * the attention sink both SVG masks keep ([SVG-TPU] figure 3).  All
 * coordinates are real (unpadded) grid coordinates. */
typedef enum {
    VSA_MASK_FULL = 0,
    VSA_MASK_SVG_SPATIAL = 1,
    VSA_MASK_SVG_TEMPORAL = 2,
    VSA_MASK_STA = 3,
    VSA_MASK_STRIPE = 4
} vsa_mask_kind;

typedef struct {
    int32_t kind;            /* vsa_mask_kind                                    */
    int32_t sink;            /* 0 or 1                                           */
    int32_t rt, rh, rw;      /* SVG radii (>= 0)                                 */
    int32_t kt, kh, kw;      /* STA window in units (>= 1)                       */
    int32_t Tw, To, Ts;      /* stripe, inter-frame: width >= 1, offset, stride >= 1 */
    int32_t Sw, So, Ss;      /* stripe, intra-frame: width >= 1, offset, stride >= 1 */
    int32_t layout;          /* vsa_layout: token order of this head (see below)   */
    int32_t tile_round;      /* 0 exact mask; 1 tile-aligned rounding (see below)  */
} vsa_mask_spec;

/* tile_round = 1 replaces the head's mask by its tile-aligned rounding, a
   lossy opt-in mode ("Sparse VideoGen: accelerating video diffusion attention
   on TPU", "aligning the sparse mask with execution", B3): a tile pair with
   some kept (real query, real key) pairs is kept whole when at least half of
   its real pairs are kept and dropped otherwise, so boundary work remains
   only where a kv tile holds padding slots.  The tile map, the kv-tile lists
   and the attention follow the rounded mask; vsa_plan_kept_pairs still counts
   the exact mask.  Allowed for full and SVG spatial / temporal heads
   (VSA_ERR_UNSUPPORTED otherwise). */

/* Token order of a head inside the [B, heads, n_slots, D] tensors.
   VSA_LAYOUT_TILE_MAJOR: tile-major over the 3D units (bt,bh,bw), padded per
     axis ("Parameterized Stripe Attention", key design 2).
   VSA_LAYOUT_FRAME0_FIRST: frame 0 in (h,w) row-major order, then every
     spatial position (h,w) in row-major order with its frames 1..T-1 in
     order; no padding inside, slots past T*H*W are padding.  This is the
     temporal-head permutation of "Sparse VideoGen: accelerating video
     diffusion attention on TPU" ("arranging tokens for efficient temporal
     access"), with the frame-0 sink kept in front so that it does not put a
     kept key in every tile.  Allowed for temporal and full heads only
     (VSA_ERR_UNSUPPORTED otherwise).  vsa_permute / vsa_unpermute and the
     tile map follow each head's layout; the attention output is the same
     set of rows in another order. */
typedef enum { VSA_LAYOUT_TILE_MAJOR = 0, VSA_LAYOUT_FRAME0_FIRST = 1 } vsa_layout;

typedef struct vsa_plan_s* vsa_plan_t;

typedef struct {
    int32_t T, H, W;          /* real latent grid                                */
    int32_t bt, bh, bw;       /* 3D unit                                         */
    int32_t num_heads;
    int32_t q_tile, kv_tile;  /* tile-map granularity (rows of q / k per tile)   */
    int32_t n_q_tiles, n_kv_tiles;
    int64_t n_tokens;         /* T*H*W                                           */
    int64_t n_padded;         /* T'H'W'                                          */
    int64_t n_slots;          /* rows of every tile-major tensor                 */
    int64_t map_bytes;        /* num_heads * n_q_tiles * n_kv_tiles              */
} vsa_plan_info_t;

/* Tile classes stored in the map ([SVG-TPU], "logical sparsity is not
 * physical sparsity"): a (q tile, kv tile) pair is EMPTY when no (real query,
 * key slot) pair is kept, FULL when every such pair is kept (so a kv tile that
 * holds padding is never full), BOUNDARY otherwise. */
enum { VSA_TILE_EMPTY = 0, VSA_TILE_BOUNDARY = 1, VSA_TILE_FULL = 2 };

/* Build a plan for `num_heads` heads (specs[h] for head h) on the T x H x W
 * grid with 3D unit (bt,bh,bw) and tile shape q_tile x kv_tile.
 * Supported: q_tile in {64,128,256}, kv_tile in {64,128}; bw in
 * {1,2,4,8,16,32} dividing kv_tile; each tile either a whole number of units
 * or one box inside a unit (its size a multiple of bh*bw, or of bw and
 * dividing bh*bw, or dividing bw); T, H, W < 32768; H*W <= 65536 for stripe heads.
 * Allocates the plan's device buffers on the current device and launches the
 * build kernels on `stream` (asynchronous).  On error *out is left NULL. */
int vsa_plan_create(const vsa_mask_spec* specs, int num_heads,
                    int T, int H, int W, int bt, int bh, int bw,
                    int q_tile, int kv_tile, void* stream, vsa_plan_t* out);

/* Host-only: the shapes a plan with these arguments would have (n_slots,
 * tile counts, map size), for sizing buffers before vsa_plan_create.  Same
 * argument checks as vsa_plan_create (stripe heads are not considered). */
int vsa_layout_info(int num_heads, int T, int H, int W, int bt, int bh, int bw,
                    int q_tile, int kv_tile, vsa_plan_info_t* out);

/* Re-run the build kernels (tile map, kv-tile lists, tables) into the plan's
 * own buffers.  Asynchronous, allocates nothing. */
int vsa_plan_build(vsa_plan_t plan, void* stream);

/* Host-side shape information; no device work. */
int vsa_plan_info(vsa_plan_t plan, vsa_plan_info_t* out);

/* Synchronous: copies the int8 map [num_heads][n_q_tiles][n_kv_tiles] to host
 * memory `host_dst` of `bytes` >= map_bytes. */
int vsa_plan_tile_map(vsa_plan_t plan, int8_t* host_dst, size_t bytes, void* stream);

/* Synchronous: per-head tile totals, host_counts[3*h + c] for class c. */
int vsa_plan_tile_counts(vsa_plan_t plan, int64_t* host_counts, size_t n, void* stream);

/* Synchronous: perm[slot] = natural token index or -1 (padding), n >= n_slots. */
int vsa_plan_perm(vsa_plan_t plan, int32_t* host_dst, size_t n, void* stream);

/* The same for either layout (vsa_layout): perm[slot] = natural token index
   (t*H + h)*W + w or -1 for padding, n >= n_slots.  VSA_ERR_INVALID_ARG for an
   unknown layout.  Synchronous on `stream`; allocates and frees a device
   buffer of n_slots int32. */
int vsa_plan_layout_perm(vsa_plan_t plan, int layout, int32_t* host_dst, size_t n, void* stream);

/* Synchronous: number of executed (kv tile, 128-row query block) steps per
 * head, host_dst[h]; the attention kernel runs one tensor-core tile per step. */
int vsa_plan_exec_steps(vsa_plan_t plan, int64_t* host_dst, size_t n, void* stream);

/* Synchronous: how the attention kernel groups the 128-row execution blocks,
 * host_dst[h * n_blocks + e] (n_blocks = n_slots / 128, n >= num_heads *
 * n_blocks): the partner block of a pair's leader, -1 for a block that runs
 * alone, -2 for a block that runs in its leader's CTA.  Two blocks pair when
 * their kv-tile lists hold the same kv tiles in the same order, so one CTA
 * loads each K and V tile once for both ([SVG-TPU], "tile-size tuning can
 * introduce trade-offs"): always the two halves of a 256-row q tile; for
 * 128-row q tiles, per head, block 2i with 2i + 1 or a block with the one a
 * t-slab of units later, whichever pairs more; never for 64-row q tiles.
 * The tile map and the tile counts do not change. */
int vsa_plan_exec_pairs(vsa_plan_t plan, int32_t* host_dst, size_t n, void* stream);

/* Synchronous: kept (real query, real key) pairs per head, host_dst[h]
 * (the logical density the tile map approximates; [SVG-TPU], "logical
 * sparsity is not physical sparsity").  Evaluates the element predicate on
 * the GPU for every pair; allocates a small scratch buffer. */
int vsa_plan_kept_pairs(vsa_plan_t plan, int64_t* host_dst, size_t n, void* stream);

/* No-allocation tile map.  None of the pages has a counterpart to this call;
 * it serves callers that cannot call cudaMalloc: a host framework that owns
 * all device memory through its own pool (a direct allocation would bypass
 * its accounting and can fail once the pool holds the memory), or a serving
 * loop that cannot afford cudaMalloc's implicit device synchronisation.
 *
 * Writes the same int8 map [num_heads][n_q_tiles][n_kv_tiles] that
 * vsa_plan_create builds (arguments and supported shapes as there) into
 * `map_out`, caller-owned device memory of `map_bytes` >= the map size
 * (vsa_layout_info gives it).  Asynchronous on `stream`.  `map_out` must be
 * device or managed memory of the current device (checked with
 * cudaPointerGetAttributes, which allocates nothing; VSA_ERR_INVALID_ARG
 * otherwise), and `map_bytes` must not exceed what the caller really owns
 * from `map_out` on: the kernel writes the whole map.
 *
 * Working memory is one file-scope device array of VSA_NOALLOC_SCRATCH_BYTES
 * that every GPU loading the library holds until the process exits; it keeps
 * the mask specs (at most VSA_NOALLOC_MAX_HEADS heads) and the stripe offset
 * tables (4 * ceil((2*H*W - 1) / 32 + 1) bytes per head).  Larger requests
 * fail with VSA_ERR_UNSUPPORTED before any device work.  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 * The first call on a device looks up the array's device address with
 * cudaGetSymbolAddress (once per device, with that device current); make that
 * first call before any stream capture.  The address is cached for the life
 * of the process: after cudaDeviceReset (or anything else that destroys the
 * device's primary context) it is stale, so do not call this entry point on
 * that device again in the same process.  All calls share the array and it
 * keeps the last call's contents (each call rewrites what it reads), so calls
 * that overlap on the GPU race: serialise them, e.g. on one stream. */
#define VSA_NOALLOC_SCRATCH_BYTES (1u << 20)
#define VSA_NOALLOC_MAX_HEADS 64
int vsa_tile_map_noalloc(const vsa_mask_spec* specs, int num_heads,
                         int T, int H, int W, int bt, int bh, int bw,
                         int q_tile, int kv_tile, int8_t* map_out, size_t map_bytes,
                         void* stream);

/* Frees the plan's device buffers (synchronises the device first). */
int vsa_plan_destroy(vsa_plan_t plan);

/* Gather into tile-major order ([VDS] section 7.2: a [N,d] gather per head;
 * [PSA] key design 2).  in: bf16 [B][num_heads][N][D] natural order;
 * out: bf16 [B][num_heads][n_slots][D]; padding rows are written as zeros.
 * D in {64,128}.  in and out must not overlap.  Asynchronous. */
int vsa_permute(vsa_plan_t plan, const void* in, void* out, int B, int D, void* stream);

/* Restore natural order ([SVG-TPU], "supporting dynamic masks and token
 * layouts": the order is restored after attention).  in: bf16
 * [B][num_heads][n_slots][D]; out: bf16 [B][num_heads][N][D]; padding rows
 * are dropped.  Asynchronous. */
int vsa_unpermute(vsa_plan_t plan, const void* in, void* out, int B, int D, void* stream);

/* q, k and v through the same permutation in one launch (the slot -> token
 * arithmetic done once per row for the three tensors); same layouts,
 * ownership and errors as vsa_permute, and no output may overlap an input or
 * another output (VSA_ERR_INVALID_ARG). */
int vsa_permute_qkv(vsa_plan_t plan, const void* q, const void* k, const void* v,
                    void* q_out, void* k_out, void* v_out, int B, int D, void* stream);

/* Block-sparse attention forward on tile-major tensors.
 * q, k, v: bf16 [B][num_heads][n_slots][D]; o: bf16 same shape;
 * lse: fp32 [B][num_heads][n_slots] (natural log of the sum over kept keys of
 * exp(scale * q.k)).  For each real query row:
 *   o_q = sum_{k kept} softmax_k(scale * q.k) v_k       ([STA] section 2, Eq. 1)
 * Empty kv tiles are skipped, full tiles run with no per-element masking,
 * boundary tiles evaluate the exact predicate, and partial results merge by
 * online softmax ([SVG-TPU], "avoid in-tile masking when nothing needs
 * masking").  A row with no kept key gets o = 0 and lse = -inf.  Padding rows
 * of o and lse are unspecified.  D in {64,128}.  Asynchronous; device-side
 * failures surface in vsa_check_status. */
int vsa_sparse_attn_fwd(const void* q, const void* k, const void* v,
                        void* o, float* lse, vsa_plan_t plan,
                        int B, int D, float scale, void* stream);

/* ---- SVG routing: spatial or temporal mask per head ----------------------
 * [SVG-TPU] section on SVG heads: a few query rows are sampled, their outputs
 * are computed under full attention and under each head's spatial and
 * temporal masks, and the head takes the mask whose outputs deviate least
 * from the full ones ([VDS]: the sample is 1-2% of the tokens).  [SVG-TPU]
 * "supporting dynamic routing with fixed tensor shapes": the per-head flags
 * select the candidate spec, and with it the head's token order, without
 * changing any tensor shape, so the steps after routing run unchanged.
 *
 * vsa_plan_set_route_candidates: the two candidates of every head (host
 * arrays of num_heads specs, copied before return; spatial[h].kind must be
 * VSA_MASK_SVG_SPATIAL and temporal[h].kind VSA_MASK_SVG_TEMPORAL, each
 * valid for vsa_plan_create, else VSA_ERR_INVALID_ARG / _UNSUPPORTED).  Their
 * layout and tile_round fields only take effect once applied; routing
 * compares the exact predicates.  Synchronises `stream`. */
int vsa_plan_set_route_candidates(vsa_plan_t plan, const vsa_mask_spec* spatial,
                                  const vsa_mask_spec* temporal, void* stream);

/* Bytes of device workspace vsa_svg_route needs for B batches, head dim D
 * and n_rows sampled rows on the current device. */
int vsa_svg_route_workspace_size(vsa_plan_t plan, int B, int D, int n_rows, size_t* bytes);

/* Deviation of each candidate from full attention over sampled rows.
 * q, k, v: bf16 [B][num_heads][N][D] in natural (t, h, w) order (device,
 * 16-byte aligned); rows: device int32 [n_rows] natural token indices shared
 * by every (batch, head) (an index outside [0, N) is read as 0 and flags
 * VSA_ERR_DEVICE in vsa_check_status).  Outputs (device): err fp32
 * [num_heads][2] = mean over batch, rows and D of (o_spatial - o_full)^2 and
 * (o_temporal - o_full)^2; flags int32 [num_heads] = 1 iff the temporal
 * deviation is strictly smaller.  workspace: device, 16-byte aligned, at
 * least vsa_svg_route_workspace_size bytes, owned by the caller.  Needs
 * candidates (VSA_ERR_INVALID_ARG otherwise).  D in {64,128}.  Asynchronous;
 * no host synchronisation, capturable in a CUDA graph. */
int vsa_svg_route(vsa_plan_t plan, const void* q, const void* k, const void* v,
                  int B, int D, const int32_t* rows, int n_rows, float scale,
                  float* err, int32_t* flags, void* workspace, size_t workspace_bytes,
                  void* stream);

/* Applies device flags [num_heads] (nonzero = temporal): each head's spec
 * becomes its temporal or spatial candidate, then the tile map, the
 * per-query-block lists and the counts are rebuilt on the device.  Shapes
 * (n_slots, list capacity) are unchanged; vsa_permute / vsa_unpermute pick
 * each head's token order from the new specs.  Asynchronous, capturable. */
int vsa_plan_apply_route(vsa_plan_t plan, const int32_t* flags, void* stream);

/* ---- Head-sharded attention across GPUs ---------------------------------
 * [SVG-TPU] "performing layout transformation on local heads": inputs
 * arrive sequence-sharded, an all-to-all gives every rank all tokens of its
 * heads ([B,S/N,H,D] -> [B,S,H/N,D]), each rank permutes its heads' tokens
 * after that exchange, runs attention, restores the order and exchanges
 * back.  Here exchange and permutation are one pass each way, through the
 * other ranks' memory (peer stores over NVLink).
 *
 * world ranks (1..8), rank r holds the natural tokens [off_r, off_{r+1}),
 * off_r = floor(r * N / world), of all world*num_heads heads; rank g owns
 * global heads [g*num_heads, (g+1)*num_heads) and `plan` is its plan (its
 * heads' specs, the full grid).  head_layout: device int32 [world*num_heads],
 * the token order (vsa_layout) of every global head, equal to each owner's
 * plan spec.  dst: host array of `world` device pointers (16-byte aligned),
 * entry g addressable from this GPU (rank g's buffer, or a local one when
 * every rank lives on this GPU).
 *
 * vsa_ulysses_permute: x = this rank's shard bf16 [B][n_rank][world*heads][D]
 * -> dst[g] = rank g's tile-major q/k/v [B][num_heads][n_slots][D]: every
 * (token, head) row goes to its owner at the token's slot; this rank also
 * zeroes the padding slots of its own buffer dst[rank].
 * vsa_ulysses_unpermute: o = this rank's tile-major output
 * [B][num_heads][n_slots][D] -> dst[r] = rank r's output shard
 * [B][n_r][world*heads][D], each token to its owner.
 *
 * The kernels wait on no other rank.  The caller orders them: every rank's
 * exchange must be complete before any rank reads the buffers it wrote (a
 * collective on the stream after each exchange), and a rank's buffers must
 * not be rewritten while it still reads them.  Asynchronous. */
int vsa_ulysses_permute(vsa_plan_t plan, const void* x, int B, int D, int rank, int world,
                        const int32_t* head_layout, void* const* dst, void* stream);
int vsa_ulysses_unpermute(vsa_plan_t plan, const void* o, int B, int D, int rank, int world,
                          const int32_t* head_layout, void* const* dst, void* stream);

/* ---- Host buffers, copies overlapped with compute ------------------------
 * The (batch, head) pairs are cut into chunks of chunk_heads heads, each with
 * its own plan (the specs of those heads).  Per chunk, on three internal
 * streams: host -> device copies of q, k, v; plan rebuild (first batch) +
 * vsa_permute_qkv + vsa_sparse_attn_fwd + vsa_unpermute; device -> host
 * copies of o and lse.  Two sets of device staging buffers alternate, so
 * chunk c computes while chunk c+1's inputs and chunk c-1's outputs cross
 * PCIe.  Chunks are issued in decreasing order of their plan's executed tile
 * steps (ties in head order), so the compute left after the last copy in is
 * the lightest; outputs land at each head's own offset whatever the order.
 *
 * vsa_pipeline_create: same spec / grid / tile arguments and errors as
 * vsa_plan_create, plus B >= 1, D in {64,128}, chunk_heads >= 1; allocates
 * the plans and 2 x chunk_heads x (4 natural + 4 tile-major) rows of
 * staging on the current device.  Synchronous.
 * vsa_pipeline_run: q, k, v, o host bf16 [B][num_heads][N][D] natural order,
 * lse host fp32 [B][num_heads][n_slots] (tile-major, as vsa_sparse_attn_fwd);
 * pinned (page-locked) memory for the copies to overlap.  Work starts after
 * everything already on `stream` and `stream` resumes after the last copy
 * back; nothing is synchronised on the host.  The host buffers must stay
 * valid until then.
 * vsa_pipeline_check_status: vsa_check_status over every chunk's plan.
 * vsa_pipeline_destroy: synchronises the device, frees everything. */
typedef struct vsa_pipeline_s* vsa_pipeline_t;
int vsa_pipeline_create(const vsa_mask_spec* specs, int num_heads, int T, int H, int W,
                        int bt, int bh, int bw, int q_tile, int kv_tile, int B, int D,
                        int chunk_heads, vsa_pipeline_t* out);
int vsa_pipeline_run(vsa_pipeline_t p, const void* q_host, const void* k_host,
                     const void* v_host, void* o_host, float* lse_host, float scale,
                     void* stream);
int vsa_pipeline_check_status(vsa_pipeline_t p, void* stream);
int vsa_pipeline_destroy(vsa_pipeline_t p);

/* Synchronises `stream`, then reports and clears the plan's device status
 * word: VSA_OK, VSA_ERR_TIMEOUT or VSA_ERR_DEVICE; VSA_ERR_CUDA if the
 * stream itself failed. */
int vsa_check_status(vsa_plan_t plan, void* stream);

/* Test hook for the device watchdog: launches one warp that waits, with the
 * same bounded wait the attention kernel uses, on an mbarrier that nothing
 * arrives at; after `cycles` SM clock cycles (1 .. 2^31) the wait gives up
 * and records a timeout in the plan's status word, so the next
 * vsa_check_status returns VSA_ERR_TIMEOUT and clears it.  Nothing faults,
 * traps or hangs; the context stays usable.  Asynchronous. */
int vsa_selftest_watchdog(vsa_plan_t plan, long long cycles, void* stream);

/* Static description of a status code. */
const char* vsa_status_string(int code);

/* VSA_VERSION of the built library. */
int vsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H */

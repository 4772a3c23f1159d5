// Internal declarations shared by the vsa CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "vsa.h"

// Device status bits (plan->d_status).
#define VSA_DEV_TIMEOUT 1u
#define VSA_DEV_BADSTATE 2u

// Execution block: the attention kernel always runs 128 query rows per CTA
// (one M = 128 tensor-core tile); q tiles of 64 rows are executed in pairs.
#define VSA_EXEC_ROWS 128

// A kv-tile list entry: kv tile index in bits [0,24), class of the lower 64
// query rows of the execution block in [24,26), of the upper 64 rows in [26,28).
#define VSA_ENTRY_KV(e) ((e) & 0xFFFFFF)
#define VSA_ENTRY_CLS(e, half) (((e) >> (24 + 2 * (half))) & 3)

struct vsa_dims {
    int T, H, W;          // real grid
    int bt, bh, bw;       // unit
    int Tp, Hp, Wp;       // padded grid
    int nTt, nTh, nTw;    // units per axis
    int U;                // tokens per unit
    int heads;
    int Bq, Bk;           // tile-map granularity
    int nQ, nK;           // q tiles, kv tiles
    int nE;               // 128-row execution blocks
    int nseg;             // kv tile segments (Bk / bw)
    int box_nh;           // when a kv tile is one box inside a unit: latent rows per t-slice
                          // of the tile (its runs go h fastest, then t); 0 otherwise
    int sbits_words;      // words per head of the stripe offset table (0 if none)
    long long N, Npad, Nslots;
};

struct vsa_plan_s {
    int device;
    vsa_dims d;
    vsa_mask_spec* d_specs;     // [heads]
    int8_t* d_map;              // [heads][nQ][nK]
    int32_t* d_list_cnt;        // [heads][nE]
    int32_t* d_list;            // [heads][nE][nK]
    int32_t* d_pair;            // [heads][nE]: partner block of a pair's leader, -1 alone, -2 in its leader's CTA
    int8_t* d_pair_flag;        // [heads][2 strides][ceil(nE/2)] candidate pairs with the same kv tiles
    int* d_pair_votes;          // [heads][2 strides] matching candidates
    int32_t* d_order;           // [heads] attention launch order: heads by decreasing executed steps
    int2* d_seg;                // [nK][nseg]: x = t | h << 16, y = w0 | nvalid << 16
    uint32_t* d_sbits;          // [heads][sbits_words] stripe intra-frame offset bits
    unsigned long long* d_counts;  // [heads][3] tile totals
    unsigned long long* d_steps;   // [heads] executed steps
    unsigned int* d_status;     // watchdog / state flags
    int has_stripe;
    vsa_mask_spec* d_cand;      // [2][heads] SVG routing candidates: spatial, temporal
    int has_cand;
    int32_t* d_slot2tok;        // [2 layouts][Nslots] natural token of a slot, -1 for padding
    int32_t* d_tok2slot;        // [2 layouts][N] slot of a natural token
};

// Host helpers ------------------------------------------------------------

#define VSA_CUDA_TRY(expr)                                 \
    do {                                                   \
        cudaError_t _e = (expr);                           \
        if (_e != cudaSuccess) return VSA_ERR_CUDA;        \
    } while (0)

int vsa_build_plan_kernels(vsa_plan_s* p, cudaStream_t s);
int vsa_dims_for(int num_heads, int T, int H, int W, int bt, int bh, int bw, int q_tile, int kv_tile,
                 int has_stripe, vsa_dims* out);
int vsa_check_spec(const vsa_mask_spec* m);
int vsa_launch_stripe_bits(const vsa_dims& d, const vsa_mask_spec* specs, uint32_t* sbits, cudaStream_t s);
int vsa_launch_tile_map(const vsa_dims& d, const vsa_mask_spec* specs, const uint32_t* sbits, int8_t* map,
                        cudaStream_t s);

static inline bool vsa_aligned16(const void* p) { return (((uintptr_t)p) & 15u) == 0; }

// Device helpers ----------------------------------------------------------

#ifdef __CUDACC__

// Natural coordinates of tile-major slot p (within one head); returns false
// for padding slots.
__device__ __forceinline__ bool vsa_slot_coords(const vsa_dims& d, long long p,
                                                int& t, int& h, int& w)
{
    if (p >= d.Npad) return false;
    const int u = (int)(p / d.U);
    const int o = (int)(p - (long long)u * d.U);
    const int per_t = d.nTh * d.nTw;
    const int tt = u / per_t;
    const int th = (u - tt * per_t) / d.nTw;
    const int tw = u - tt * per_t - th * d.nTw;
    const int hw = d.bh * d.bw;
    const int ot = o / hw;
    const int oh = (o - ot * hw) / d.bw;
    const int ow = o - ot * hw - oh * d.bw;
    t = tt * d.bt + ot;
    h = th * d.bh + oh;
    w = tw * d.bw + ow;
    return t < d.T && h < d.H && w < d.W;
}

// Tile-major slot of the real token (t,h,w).
__device__ __forceinline__ long long vsa_token_slot(const vsa_dims& d, int t, int h, int w)
{
    const int tt = t / d.bt, th = h / d.bh, tw = w / d.bw;
    const int ot = t - tt * d.bt, oh = h - th * d.bh, ow = w - tw * d.bw;
    const long long u = ((long long)tt * d.nTh + th) * d.nTw + tw;
    return u * d.U + (ot * d.bh + oh) * d.bw + ow;
}

// Natural coordinates of slot p of a frame-0-first head (VSA_LAYOUT_FRAME0_FIRST):
// slots [0, HW) are frame 0 in (h,w) order, then position (h,w) in row-major
// order with its frames 1..T-1; false for padding slots (p >= T*H*W).
__device__ __forceinline__ bool vsa_slot_coords_f0(const vsa_dims& d, long long p, int& t, int& h, int& w)
{
    const long long HW = (long long)d.H * d.W;
    if (p < HW) {
        t = 0;
        h = (int)(p / d.W);
        w = (int)(p - (long long)h * d.W);
        return true;
    }
    const long long r = p - HW;
    if (d.T <= 1 || r >= HW * (d.T - 1)) return false;
    const long long pos = r / (d.T - 1);
    t = 1 + (int)(r - pos * (d.T - 1));
    h = (int)(pos / d.W);
    w = (int)(pos - (long long)h * d.W);
    return true;
}

// Slot of the real token (t,h,w) in a frame-0-first head.
__device__ __forceinline__ long long vsa_token_slot_f0(const vsa_dims& d, int t, int h, int w)
{
    const long long pos = (long long)h * d.W + w;
    return t == 0 ? pos : (long long)d.H * d.W + pos * (d.T - 1) + (t - 1);
}

// Either layout.
__device__ __forceinline__ bool vsa_slot_coords_any(const vsa_dims& d, int layout, long long p, int& t, int& h,
                                                    int& w)
{
    return layout == VSA_LAYOUT_FRAME0_FIRST ? vsa_slot_coords_f0(d, p, t, h, w) : vsa_slot_coords(d, p, t, h, w);
}

__device__ __forceinline__ int vsa_iabs(int x) { return x < 0 ? -x : x; }

// STA along one axis: first unit of the window of query unit uq.
__device__ __forceinline__ int vsa_sta_start(int uq, int n, int k)
{
    const int kk = k < n ? k : n;
    int s = uq - kk / 2;
    s = s < 0 ? 0 : s;
    return s > n - kk ? n - kk : s;
}

__device__ __forceinline__ uint32_t vsa_low_bits(int n) { return n >= 32 ? 0xFFFFFFFFu : ((1u << n) - 1u); }

// Query-row context for the boundary predicate.
struct vsa_row_ctx {
    int tq, hq, wq, sq;
    bool real;
    int sta_t, sta_h, sta_w;   // first unit of the STA window per axis
    int kk_t, kk_h, kk_w;      // window length per axis (clamped)
};

// Kept-key bits of one run of `nv` real keys at (t, h, w0 .. w0+nv-1).
__device__ __forceinline__ uint32_t vsa_run_bits(const vsa_mask_spec& m, const vsa_dims& d, const vsa_row_ctx& q,
                                             const uint32_t* stab, const uint32_t* ttab, int t, int h,
                                             int w0, int nv)
{
    if (nv == 0 || !q.real) return 0u;
    const uint32_t vm = vsa_low_bits(nv);
    if (m.sink && t == 0) return vm;
    switch (m.kind) {
    case VSA_MASK_FULL:
        return vm;
    case VSA_MASK_SVG_SPATIAL:
        return vsa_iabs(t - q.tq) <= m.rt ? vm : 0u;
    case VSA_MASK_SVG_TEMPORAL: {
        if (vsa_iabs(h - q.hq) > m.rh) return 0u;
        const int lo = max(q.wq - m.rw, w0) - w0;
        const int hi = min(q.wq + m.rw, w0 + nv - 1) - w0;
        if (lo > hi) return 0u;
        return vsa_low_bits(hi - lo + 1) << lo;
    }
    case VSA_MASK_STA: {
        const int ut = t / d.bt, uh = h / d.bh, uw = w0 / d.bw;
        const bool in = ut >= q.sta_t && ut < q.sta_t + q.kk_t && uh >= q.sta_h &&
                        uh < q.sta_h + q.kk_h && uw >= q.sta_w && uw < q.sta_w + q.kk_w;
        return in ? vm : 0u;
    }
    case VSA_MASK_STRIPE: {
        const int it = t - q.tq + d.T - 1;
        if (!((ttab[it >> 5] >> (it & 31)) & 1u)) return 0u;
        const int x = h * d.W + w0 - q.sq + d.H * d.W - 1;
        const uint32_t v = __funnelshift_r(stab[x >> 5], stab[(x >> 5) + 1], x & 31);
        return v & vm;
    }
    default:
        return 0u;
    }
}

// Query-row context of slot `slot` (in the head's layout) for the predicate above.
__device__ __forceinline__ vsa_row_ctx vsa_row_init(const vsa_dims& d, const vsa_mask_spec& m,
                                                    long long slot)
{
    vsa_row_ctx q;
    q.tq = q.hq = q.wq = 0;
    q.real = vsa_slot_coords_any(d, m.layout, slot, q.tq, q.hq, q.wq);
    q.sq = q.hq * d.W + q.wq;
    q.kk_t = min(m.kt, d.nTt);
    q.kk_h = min(m.kh, d.nTh);
    q.kk_w = min(m.kw, d.nTw);
    q.sta_t = vsa_sta_start(q.tq / d.bt, d.nTt, m.kt);
    q.sta_h = vsa_sta_start(q.hq / d.bh, d.nTh, m.kh);
    q.sta_w = vsa_sta_start(q.wq / d.bw, d.nTw, m.kw);
    return q;
}

// Word i of the stripe inter-frame table: bit b <-> dt = 32 i + b - (T - 1),
// set when (|dt - To| mod Ts) <= Tw - 1 (dt = t_k - t_q).
__device__ __forceinline__ uint32_t vsa_stripe_tword(const vsa_mask_spec& m, int T, int i)
{
    uint32_t v = 0;
    for (int b = 0; b < 32; ++b) {
        const int dt = i * 32 + b - (T - 1);
        if (dt > T - 1) break;
        if ((vsa_iabs(dt - m.To) % m.Ts) <= m.Tw - 1) v |= 1u << b;
    }
    return v;
}

// Words of the two stripe tables a kernel keeps in shared memory.
static inline __host__ __device__ int vsa_ttab_words(int T) { return (2 * T - 1 + 31) / 32 + 1; }

#endif  // __CUDACC__

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
    int2* d_seg;                // [nK][nseg]: x = t | h << 16, y = w0 | nvalid << 16
    uint32_t* d_sbits;          // [heads][sbits_words] stripe intra-frame offset bits
    unsigned long long* d_counts;  // [heads][3] tile totals
    unsigned long long* d_steps;   // [heads] executed steps
    unsigned int* d_status;     // watchdog / state flags
    int has_stripe;
};

// Host helpers ------------------------------------------------------------

#define VSA_CUDA_TRY(expr)                                 \
    do {                                                   \
        cudaError_t _e = (expr);                           \
        if (_e != cudaSuccess) return VSA_ERR_CUDA;        \
    } while (0)

int vsa_build_plan_kernels(vsa_plan_s* p, cudaStream_t s);

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

__device__ __forceinline__ int vsa_iabs(int x) { return x < 0 ? -x : x; }

// STA along one axis: first unit of the window of query unit uq.
__device__ __forceinline__ int vsa_sta_start(int uq, int n, int k)
{
    const int kk = k < n ? k : n;
    int s = uq - kk / 2;
    s = s < 0 ? 0 : s;
    return s > n - kk ? n - kk : s;
}

#endif  // __CUDACC__

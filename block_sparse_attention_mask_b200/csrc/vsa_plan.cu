// Plan construction: mask specs -> tile map, per-query-block kv-tile lists,
// kv-tile segment table and stripe offset tables, all built by GPU kernels.
//
// Tile classes follow the three kinds of "Sparse VideoGen: accelerating video
// diffusion attention on TPU" (section "logical sparsity is not physical
// sparsity"); the per-query-block list of kv tiles is the block-sparse
// interface of "Video diffusion long-sequence attention and sparsity",
// section 7.3.
//
// Classification is exact without visiting element pairs: the real tokens of
// a tile form one or a few 3D boxes (a tile is a box inside one unit or a run
// of whole units), and every mask is (relation on t) AND (relation on the
// in-frame position), OR the frame-0 sink.  For a pair of boxes the kept set
// is therefore the product of a t-pair set and an (h,w)-pair set, so "some
// pair kept" and "every pair kept" follow from per-axis any/all tests.  The
// in-frame stripe relation depends on s_k - s_q only, so for each pair of
// latent rows the kept pairs are the offsets of a contiguous range, read
// from a per-head bit table over all offsets.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <new>

#include "vsa_internal.h"

namespace {

struct Box {
    int t0, t1, h0, h1, w0, w1;  // half-open real ranges
};

// Box i of tile `tile` (size B slots).  Returns false when that box holds no
// real token.  Sets *pad when the tile holds any padding slot.
__device__ bool tile_box(const vsa_dims& d, int tile, int B, int i, Box& bx, bool& pad)
{
    const int p0 = tile * B;                 // < 2^24 + B: n_slots is capped at 2^24
    int u, t0, t1, h0, h1, w0, w1;
    if (B <= d.U) {
        if (p0 >= d.Npad) { pad = true; return false; }
        u = p0 / d.U;
        const int o0 = p0 - u * d.U;
        const int per_t = d.nTh * d.nTw;
        const int tt = u / per_t, th = (u - tt * per_t) / d.nTw, tw = u - tt * per_t - th * d.nTw;
        const int hw = d.bh * d.bw;
        const int ot = o0 / hw, oh = (o0 - ot * hw) / d.bw, ow = o0 - ot * hw - oh * d.bw;
        if (B % hw == 0) {
            t0 = tt * d.bt + ot; t1 = t0 + B / hw;
            h0 = th * d.bh; h1 = h0 + d.bh;
            w0 = tw * d.bw; w1 = w0 + d.bw;
        } else if (B % d.bw == 0) {
            t0 = tt * d.bt + ot; t1 = t0 + 1;
            h0 = th * d.bh + oh; h1 = h0 + B / d.bw;
            w0 = tw * d.bw; w1 = w0 + d.bw;
        } else {
            t0 = tt * d.bt + ot; t1 = t0 + 1;
            h0 = th * d.bh + oh; h1 = h0 + 1;
            w0 = tw * d.bw + ow; w1 = w0 + B;
        }
    } else {
        u = (int)(p0 / d.U) + i;
        if ((long long)u * d.U >= d.Npad) { pad = true; return false; }
        const int per_t = d.nTh * d.nTw;
        const int tt = u / per_t, th = (u - tt * per_t) / d.nTw, tw = u - tt * per_t - th * d.nTw;
        t0 = tt * d.bt; t1 = t0 + d.bt;
        h0 = th * d.bh; h1 = h0 + d.bh;
        w0 = tw * d.bw; w1 = w0 + d.bw;
    }
    if (t1 > d.T || h1 > d.H || w1 > d.W) pad = true;
    bx.t0 = t0; bx.t1 = min(t1, d.T);
    bx.h0 = h0; bx.h1 = min(h1, d.H);
    bx.w0 = w0; bx.w1 = min(w1, d.W);
    return bx.t0 < bx.t1 && bx.h0 < bx.h1 && bx.w0 < bx.w1;
}

// Boxes of slots [p0, p0 + B) of a frame-0-first head (VSA_LAYOUT_FRAME0_FIRST):
// the frame-0 part is a run of (h,w) positions in row-major order (part of a
// row, whole rows, part of a row); the rest is a run of (position, frame)
// pairs with frames fastest (part of one position's frames, whole positions
// with frames 1..T-1, part of one position's frames).  At most 8 boxes; sets
// pad when the range reaches past the T*H*W real tokens.
__device__ int f0_tile_boxes(const vsa_dims& d, long long p0, int B, Box* bx, bool& pad)
{
    const long long HW = (long long)d.H * d.W, N = HW * d.T, p1 = p0 + B;
    int n = 0;
    if (p1 > N) pad = true;
    // positions [a, b) of the row-major (h,w) order, with frames [t0, t1)
    auto add_positions = [&](long long a, long long b, int t0, int t1) {
        while (a < b) {
            const int h = (int)(a / d.W), w = (int)(a - (long long)h * d.W);
            if (w == 0 && b - a >= d.W) {
                const int rows = (int)((b - a) / d.W);
                bx[n++] = Box{t0, t1, h, h + rows, 0, d.W};
                a += (long long)rows * d.W;
            } else {
                const int len = (int)min((long long)(d.W - w), b - a);
                bx[n++] = Box{t0, t1, h, h + 1, w, w + len};
                a += len;
            }
        }
    };
    if (p0 < HW) add_positions(p0, min(p1, HW), 0, 1);
    if (d.T > 1 && p1 > HW && p0 < N) {
        const long long F = d.T - 1;
        long long r0 = max(p0, HW) - HW;
        const long long r1 = min(p1, N) - HW;
        if (r0 % F) {                              // the tail of one position's frames
            const long long pos = r0 / F;
            const long long end = min(r1, (pos + 1) * F);
            add_positions(pos, pos + 1, 1 + (int)(r0 - pos * F), 1 + (int)(end - pos * F));
            r0 = end;
        }
        const long long pa = r0 / F, pb = r1 / F;
        if (pb > pa) add_positions(pa, pb, 1, d.T);  // whole positions
        if (r1 > pb * F && pb * F >= r0)           // the head of one position's frames
            add_positions(pb, pb + 1, 1, 1 + (int)(r1 - pb * F));
    }
    return n;
}

__device__ __forceinline__ bool rel_t(const vsa_mask_spec& m, const vsa_dims& d, int tq, int tk)
{
    switch (m.kind) {
    case VSA_MASK_SVG_SPATIAL: return vsa_iabs(tk - tq) <= m.rt;
    case VSA_MASK_STRIPE: return (vsa_iabs(tk - tq - m.To) % m.Ts) <= m.Tw - 1;
    case VSA_MASK_STA: {
        const int s = vsa_sta_start(tq / d.bt, d.nTt, m.kt);
        const int uk = tk / d.bt;
        return uk >= s && uk < s + min(m.kt, d.nTt);
    }
    default: return true;
    }
}

// Interval helpers for |a - b| over a in [a0,a1), b in [b0,b1).
__device__ __forceinline__ int min_absdiff(int a0, int a1, int b0, int b1)
{
    if (b0 > a1 - 1) return b0 - (a1 - 1);
    if (a0 > b1 - 1) return a0 - (b1 - 1);
    return 0;
}
__device__ __forceinline__ int max_absdiff(int a0, int a1, int b0, int b1)
{
    return max(b1 - 1 - a0, a1 - 1 - b0);
}

// Number of set bits of `tab` in bit positions [i0, i1] (inclusive).
__device__ __forceinline__ int count_bits(const uint32_t* tab, int i0, int i1)
{
    int c = 0;
    const int wa = i0 >> 5, wb = i1 >> 5;
    for (int wd = wa; wd <= wb; ++wd) {
        uint32_t m = tab[wd];
        const int lo = (wd == wa) ? (i0 & 31) : 0;
        const int hi = (wd == wb) ? (i1 & 31) : 31;
        m &= (0xFFFFFFFFu >> (31 - hi)) & (0xFFFFFFFFu << lo);
        c += __popc(m);
    }
    return c;
}

// any / all of the in-frame relation over (A.h x A.w) x (B.h x B.w).
__device__ void rel_s(const vsa_mask_spec& m, const vsa_dims& d, const uint32_t* sbits,
                      const Box& A, const Box& B, bool& any, bool& all)
{
    switch (m.kind) {
    case VSA_MASK_SVG_TEMPORAL: {
        const bool anyh = min_absdiff(A.h0, A.h1, B.h0, B.h1) <= m.rh;
        const bool allh = max_absdiff(A.h0, A.h1, B.h0, B.h1) <= m.rh;
        const bool anyw = min_absdiff(A.w0, A.w1, B.w0, B.w1) <= m.rw;
        const bool allw = max_absdiff(A.w0, A.w1, B.w0, B.w1) <= m.rw;
        any = anyh && anyw;
        all = allh && allw;
        return;
    }
    case VSA_MASK_STA: {
        const int sh = vsa_sta_start(A.h0 / d.bh, d.nTh, m.kh), uh = B.h0 / d.bh;
        const int sw = vsa_sta_start(A.w0 / d.bw, d.nTw, m.kw), uw = B.w0 / d.bw;
        const bool in = uh >= sh && uh < sh + min(m.kh, d.nTh) && uw >= sw && uw < sw + min(m.kw, d.nTw);
        any = in;
        all = in;
        return;
    }
    case VSA_MASK_STRIPE: {
        const int HW1 = d.H * d.W - 1;
        const int dlo = B.w0 - (A.w1 - 1), dhi = (B.w1 - 1) - A.w0;
        any = false;
        all = true;
        for (int hq = A.h0; hq < A.h1; ++hq) {
            for (int hk = B.h0; hk < B.h1; ++hk) {
                const int x0 = (hk - hq) * d.W + dlo + HW1, x1 = (hk - hq) * d.W + dhi + HW1;
                const int ones = count_bits(sbits, x0, x1);
                any = any || ones > 0;
                all = all && ones == x1 - x0 + 1;
                if (any && !all) return;
            }
        }
        return;
    }
    default:
        any = true;
        all = true;
        return;
    }
}

// #{(a, b) : a in [a0,a1), b in [b0,b1), |a - b| <= r}
__device__ long long pairs_within(int a0, int a1, int b0, int b1, int r)
{
    long long n = 0;
    for (int a = a0; a < a1; ++a) n += max(0, min(b1 - 1, a + r) - max(b0, a - r) + 1);
    return n;
}

// Kept pairs over real (A x B), for the masks tile rounding accepts (full,
// SVG spatial and temporal, with the frame-0 sink): the frame-0 keys of a
// sink head are all kept, the rest is a product of per-axis pair counts.
__device__ long long count_kept(const vsa_mask_spec& m, const Box& A, const Box& B)
{
    const long long ahw = (long long)(A.h1 - A.h0) * (A.w1 - A.w0);
    const long long bhw = (long long)(B.h1 - B.h0) * (B.w1 - B.w0);
    const int at = A.t1 - A.t0;
    long long kept = 0;
    int tk0 = B.t0;
    if (m.sink && B.t0 == 0) {
        kept += (long long)at * ahw * bhw;
        tk0 = 1;
    }
    if (tk0 >= B.t1) return kept;
    const int bt = B.t1 - tk0;
    switch (m.kind) {
    case VSA_MASK_SVG_SPATIAL:
        return kept + pairs_within(A.t0, A.t1, tk0, B.t1, m.rt) * ahw * bhw;
    case VSA_MASK_SVG_TEMPORAL:
        return kept + (long long)at * bt * pairs_within(A.h0, A.h1, B.h0, B.h1, m.rh) *
                          pairs_within(A.w0, A.w1, B.w0, B.w1, m.rw);
    default:
        return kept + (long long)at * bt * ahw * bhw;
    }
}

__device__ __forceinline__ long long box_size(const Box& b)
{
    return (long long)(b.t1 - b.t0) * (b.h1 - b.h0) * (b.w1 - b.w0);
}

// Class of a tile pair under tile-aligned rounding: kept whole when at least
// half of its real pairs are kept (class 1 if the kv tile holds padding).
__device__ int8_t rounded_class(long long kept, long long pairs, bool kpad)
{
    if (kept == 0 || 2 * kept < pairs) return VSA_TILE_EMPTY;
    return kpad ? VSA_TILE_BOUNDARY : VSA_TILE_FULL;
}

// any / all kept over real (A x B).
__device__ void classify_boxes(const vsa_mask_spec& m, const vsa_dims& d, const uint32_t* sbits,
                               const Box& A, const Box& B, bool& any, bool& all)
{
    const bool sinkk = m.sink && B.t0 == 0;
    const int tk0 = sinkk ? 1 : B.t0;
    if (tk0 >= B.t1) {  // the key box is frame 0 only and every pair is kept by the sink
        any = true;
        all = true;
        return;
    }
    bool anyt = false, allt = true;
    if (m.kind == VSA_MASK_SVG_TEMPORAL || m.kind == VSA_MASK_FULL) {
        anyt = true;                     // no relation on t
    } else {
        for (int tq = A.t0; tq < A.t1; ++tq)
            for (int tk = tk0; tk < B.t1; ++tk) {
                const bool r = rel_t(m, d, tq, tk);
                anyt = anyt || r;
                allt = allt && r;
            }
    }
    bool anys = false, alls = false;
    if (anyt || allt) rel_s(m, d, sbits, A, B, anys, alls);
    any = sinkk || (anyt && anys);
    all = allt && alls;
}

__global__ void tile_map_kernel(vsa_dims d, const vsa_mask_spec* __restrict__ specs,
                                const uint32_t* __restrict__ sbits, int8_t* __restrict__ map)
{
    const long long per_head = (long long)d.nQ * d.nK;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= per_head * d.heads) return;
    int head, a, b;
    if (per_head * d.heads <= 0x7FFFFFFFLL) {          // 32-bit division (the usual case)
        const int i32 = (int)idx, ph = (int)per_head;
        head = i32 / ph;
        const int r = i32 - head * ph;
        a = r / d.nK;
        b = r - a * d.nK;
    } else {
        head = (int)(idx / per_head);
        const long long rem = idx - (long long)head * per_head;
        a = (int)(rem / d.nK);
        b = (int)(rem - (long long)a * d.nK);
    }
    const vsa_mask_spec m = specs[head];
    const uint32_t* sb = sbits ? sbits + (size_t)head * d.sbits_words : nullptr;
    if (m.layout == VSA_LAYOUT_FRAME0_FIRST) {
        Box qb[8], kb[8];
        bool qpad = false, kpad = false;
        const int nq = f0_tile_boxes(d, (long long)a * d.Bq, d.Bq, qb, qpad);
        const int nk = f0_tile_boxes(d, (long long)b * d.Bk, d.Bk, kb, kpad);
        if (m.tile_round) {
            long long kept = 0, nqr = 0, nkr = 0;
            for (int i = 0; i < nq; ++i) nqr += box_size(qb[i]);
            for (int j = 0; j < nk; ++j) nkr += box_size(kb[j]);
            for (int i = 0; i < nq; ++i)
                for (int j = 0; j < nk; ++j) kept += count_kept(m, qb[i], kb[j]);
            map[idx] = rounded_class(kept, nqr * nkr, kpad);
            return;
        }
        bool any = false, all = true;
        for (int i = 0; i < nq && !(any && !all); ++i)
            for (int j = 0; j < nk; ++j) {
                bool ba, bl;
                classify_boxes(m, d, sb, qb[i], kb[j], ba, bl);
                any = any || ba;
                all = all && bl;
                if (any && !all) break;
            }
        map[idx] = (nq > 0 && any) ? ((all && !kpad && nk > 0) ? VSA_TILE_FULL : VSA_TILE_BOUNDARY) : VSA_TILE_EMPTY;
        return;
    }
    const int nqb = d.Bq <= d.U ? 1 : d.Bq / d.U;
    const int nkb = d.Bk <= d.U ? 1 : d.Bk / d.U;
    if (m.tile_round) {
        bool qpad = false, kpad = false;
        long long kept = 0, nqr = 0, nkr = 0;
        for (int j = 0; j < nkb; ++j) {
            Box B;
            if (tile_box(d, b, d.Bk, j, B, kpad)) nkr += box_size(B);
            else kpad = true;
        }
        for (int i = 0; i < nqb; ++i) {
            Box A;
            if (!tile_box(d, a, d.Bq, i, A, qpad)) continue;
            nqr += box_size(A);
            for (int j = 0; j < nkb; ++j) {
                Box B;
                bool kp = false;
                if (tile_box(d, b, d.Bk, j, B, kp)) kept += count_kept(m, A, B);
            }
        }
        map[idx] = rounded_class(kept, nqr * nkr, kpad);
        return;
    }

    bool qpad = false, kpad = false, anyq = false;
    bool any = false, all = true;
    for (int i = 0; i < nqb && !(any && !all); ++i) {
        Box A;
        if (!tile_box(d, a, d.Bq, i, A, qpad)) continue;
        anyq = true;
        for (int j = 0; j < nkb; ++j) {
            Box B;
            if (!tile_box(d, b, d.Bk, j, B, kpad)) continue;
            bool ba, bl;
            classify_boxes(m, d, sb, A, B, ba, bl);
            any = any || ba;
            all = all && bl;
            if (any && !all) break;
        }
    }
    // padding anywhere in the kv tile rules out "full"
    if (!kpad) {
        for (int j = 0; j < nkb; ++j) {
            Box B;
            if (!tile_box(d, b, d.Bk, j, B, kpad)) kpad = true;
        }
    }
    int8_t cls = VSA_TILE_EMPTY;
    if (anyq && any) cls = (all && !kpad) ? VSA_TILE_FULL : VSA_TILE_BOUNDARY;
    map[idx] = cls;
}

// The real boxes of one tile under one token order and its padding flag (any
// slot of the tile that holds no real token).  Returns the number of boxes;
// callers only use this where a tile has at most kMaxTileBoxes of them (a
// frame-0-first tile always does; a tile-major tile when it spans at most
// eight units).
constexpr int kMaxTileBoxes = 8;

__device__ int tile_boxes(const vsa_dims& d, int layout, int tile, int B, Box* bx, bool& pad)
{
    pad = false;
    if (layout == VSA_LAYOUT_FRAME0_FIRST) return f0_tile_boxes(d, (long long)tile * B, B, bx, pad);
    const int nb = B <= d.U ? 1 : B / d.U;
    int n = 0;
    for (int i = 0; i < nb && i < kMaxTileBoxes; ++i) {
        Box b;
        if (tile_box(d, tile, B, i, b, pad)) bx[n++] = b;
    }
    return n;
}

// Tile boxes kept in shared memory as int16 coordinates (T, H, W < 2^15),
// field-major so that thread c reads column c without bank conflicts.
template <int N>
struct BoxCols {
    short v[kMaxTileBoxes][6][N];
    __device__ __forceinline__ void put(int j, int c, const Box& b)
    {
        v[j][0][c] = (short)b.t0; v[j][1][c] = (short)b.t1;
        v[j][2][c] = (short)b.h0; v[j][3][c] = (short)b.h1;
        v[j][4][c] = (short)b.w0; v[j][5][c] = (short)b.w1;
    }
    __device__ __forceinline__ Box get(int j, int c) const
    {
        return Box{v[j][0][c], v[j][1][c], v[j][2][c], v[j][3][c], v[j][4][c], v[j][5][c]};
    }
};

constexpr int kMapKB = 128;  // kv tiles per block, one per thread
constexpr int kMapQB = 32;   // q tiles per block

// The tile map for tiles of at most kMaxTileBoxes boxes: one block per
// (head, 32 q tiles, 128 kv tiles).  Each tile's boxes are derived once per
// block into shared memory; a thread then classifies its kv tile against the
// block's 32 q tiles (coalesced byte stores along kv).  Same classes as
// tile_map_kernel: any / all kept over the real (A x B) box pairs, or the
// kept fraction under tile-aligned rounding.
__global__ void __launch_bounds__(kMapKB) tile_map_blocked_kernel(vsa_dims d,
                                                                  const vsa_mask_spec* __restrict__ specs,
                                                                  const uint32_t* __restrict__ sbits,
                                                                  int8_t* __restrict__ map)
{
    __shared__ BoxCols<kMapQB> qbx;
    __shared__ BoxCols<kMapKB> kbx;
    __shared__ unsigned char qn[kMapQB];
    const int head = blockIdx.z;
    const vsa_mask_spec m = specs[head];
    const uint32_t* sb = sbits ? sbits + (size_t)head * d.sbits_words : nullptr;
    const int c = threadIdx.x;
    const int a0 = blockIdx.y * kMapQB;
    const int b = blockIdx.x * kMapKB + c;
    Box tmp[kMaxTileBoxes];
    if (c < kMapQB) {
        bool qpad;
        const int n = (a0 + c < d.nQ) ? tile_boxes(d, m.layout, a0 + c, d.Bq, tmp, qpad) : 0;
        for (int i = 0; i < n; ++i) qbx.put(i, c, tmp[i]);
        qn[c] = (unsigned char)n;
    }
    bool kpad = false;
    int nk = 0;
    long long nkr = 0;
    if (b < d.nK) {
        nk = tile_boxes(d, m.layout, b, d.Bk, tmp, kpad);
        for (int j = 0; j < nk; ++j) {
            kbx.put(j, c, tmp[j]);
            nkr += box_size(tmp[j]);
        }
    }
    __syncthreads();
    if (b >= d.nK) return;
    const int na = min(kMapQB, d.nQ - a0);
    int8_t* out = map + ((long long)head * d.nQ + a0) * d.nK + b;
    for (int qi = 0; qi < na; ++qi, out += d.nK) {
        const int nq = qn[qi];
        int8_t cls;
        if (m.tile_round) {
            long long kept = 0, nqr = 0;
            for (int i = 0; i < nq; ++i) {
                const Box A = qbx.get(i, qi);
                nqr += box_size(A);
                for (int j = 0; j < nk; ++j) kept += count_kept(m, A, kbx.get(j, c));
            }
            cls = rounded_class(kept, nqr * nkr, kpad);
        } else {
            bool any = false, all = true;
            for (int i = 0; i < nq && !(any && !all); ++i) {
                const Box A = qbx.get(i, qi);
                for (int j = 0; j < nk; ++j) {
                    bool ba, bl;
                    classify_boxes(m, d, sb, A, kbx.get(j, c), ba, bl);
                    any = any || ba;
                    all = all && bl;
                    if (any && !all) break;
                }
            }
            cls = any ? ((all && !kpad) ? VSA_TILE_FULL : VSA_TILE_BOUNDARY) : VSA_TILE_EMPTY;
        }
        *out = cls;
    }
}

// Per kv tile, one entry per run of bw slots sharing (t, h): the run's t, h,
// first w and number of real tokens.
__global__ void seg_table_kernel(vsa_dims d, int2* __restrict__ seg)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)d.nK * d.nseg) return;
    const long long p = idx * d.bw;  // first slot of the run
    int t = 0, h = 0, w0 = 0, nv = 0;
    if (p < d.Npad) {
        int w;
        vsa_slot_coords(d, p, t, h, w);
        w0 = w;
        if (t < d.T && h < d.H) nv = max(0, min(d.bw, d.W - w0));
    }
    seg[idx] = make_int2((t & 0xFFFF) | (h << 16), (w0 & 0xFFFF) | (nv << 16));
}

// Stripe in-frame relation over every offset x = s_k - s_q in [-(HW-1), HW-1]:
// bit (x + HW - 1) = ((|x - So| mod Ss) <= Sw - 1).
__global__ void stripe_bits_kernel(vsa_dims d, const vsa_mask_spec* __restrict__ specs,
                                   uint32_t* __restrict__ sbits)
{
    const int head = blockIdx.y;
    const int wd = blockIdx.x * blockDim.x + threadIdx.x;
    if (wd >= d.sbits_words) return;
    const vsa_mask_spec m = specs[head];
    uint32_t v = 0;
    if (m.kind == VSA_MASK_STRIPE) {
        const int HW = d.H * d.W;
        for (int i = 0; i < 32; ++i) {
            const int x = wd * 32 + i - (HW - 1);
            if (x > HW - 1) break;
            if ((vsa_iabs(x - m.So) % m.Ss) <= m.Sw - 1) v |= 1u << i;
        }
    }
    sbits[(size_t)head * d.sbits_words + wd] = v;
}

// Position of the idx-th kv tile in a list of a tile-major head whose kv
// tiles lie inside units: units spatial-position-major (all t-slabs of one
// (h, w) unit position, then the next position), tiles of a unit in order.
// Consecutive boundary tiles then mostly share their keep bits (a temporal
// window does not depend on the key's frame), which the attention kernel
// reuses.  Slots past the padded grid keep their place at the end.
__device__ __forceinline__ int spatial_major_tile(const vsa_dims& d, int idx)
{
    const int tpu = d.U / d.Bk;                      // kv tiles per unit
    const int nsu = d.nTh * d.nTw;                   // unit positions per t-slab
    if (idx >= d.nTt * nsu * tpu) return idx;
    const int q = idx / tpu;                         // su * nTt + slab
    const int su = q / d.nTt, slab = q - su * d.nTt;
    return (slab * nsu + su) * tpu + (idx - q * tpu);
}

// One warp per (head, execution block): the ordered list of kv tiles with a
// kept pair for either 64-row half, with both halves' classes, plus tile and
// step totals.  Tile-major heads with kv tiles inside units list them
// spatial-position-major (spatial_major_tile), the others in index order.
__global__ void kv_list_kernel(vsa_dims d, const vsa_mask_spec* __restrict__ specs, const int8_t* __restrict__ map,
                               int32_t* __restrict__ list_cnt, int32_t* __restrict__ list,
                               unsigned long long* __restrict__ counts,
                               unsigned long long* __restrict__ steps)
{
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= (long long)d.heads * d.nE) return;
    const int head = (int)(gw / d.nE), e = (int)(gw - (long long)head * d.nE);
    int r0, r1;
    bool own0, own1;
    if (d.Bq == 64) { r0 = 2 * e; r1 = 2 * e + 1; own0 = true; own1 = true; }
    else if (d.Bq == 128) { r0 = e; r1 = e; own0 = true; own1 = false; }
    else { r0 = e >> 1; r1 = r0; own0 = (e & 1) == 0; own1 = false; }
    const int8_t* m0 = map + ((size_t)head * d.nQ + r0) * d.nK;
    const int8_t* m1 = map + ((size_t)head * d.nQ + r1) * d.nK;
    int32_t* out = list + ((size_t)head * d.nE + e) * d.nK;
    const bool spatial_major = specs[head].layout == VSA_LAYOUT_TILE_MAJOR && d.Bk <= d.U;
    int cnt = 0;
    unsigned c[3] = {0, 0, 0};
    for (int jb = 0; jb < d.nK; jb += 32) {
        const int j = (spatial_major && jb + lane < d.nK) ? spatial_major_tile(d, jb + lane) : jb + lane;
        int c0 = 0, c1 = 0;
        if (j < d.nK) {
            c0 = m0[j];
            c1 = m1[j];
            if (own0) c[c0] += 1;
            if (own1) c[c1] += 1;
        }
        const bool nz = (c0 | c1) != 0;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, nz);
        if (nz) {
            const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
            out[pos] = j | (c0 << 24) | (c1 << 26);
        }
        cnt += __popc(bal);
    }
    for (int k = 0; k < 3; ++k)
        for (int off = 16; off > 0; off >>= 1) c[k] += __shfl_xor_sync(0xFFFFFFFFu, c[k], off);
    if (lane == 0) {
        list_cnt[(size_t)head * d.nE + e] = cnt;
        atomicAdd(&steps[head], (unsigned long long)cnt);
        for (int k = 0; k < 3; ++k)
            if (c[k]) atomicAdd(&counts[head * 3 + k], (unsigned long long)c[k]);
    }
}

// Kept (real query, real key) pairs per head: every real query row against
// every run of keys of every kv tile, with the element predicate of the
// boundary path.  One thread per query slot.
__global__ void __launch_bounds__(256) kept_pairs_kernel(vsa_dims d, const vsa_mask_spec* __restrict__ specs,
                                                         const uint32_t* __restrict__ sbits,
                                                         const int2* __restrict__ seg,
                                                         unsigned long long* __restrict__ kept)
{
    extern __shared__ uint32_t tabs[];
    const int head = blockIdx.y;
    vsa_mask_spec m = specs[head];
    m.layout = VSA_LAYOUT_TILE_MAJOR;   // the total does not depend on the order; the runs are tile-major
    const int ws = (m.kind == VSA_MASK_STRIPE) ? d.sbits_words : 0;
    const int wt = (m.kind == VSA_MASK_STRIPE) ? vsa_ttab_words(d.T) : 0;
    uint32_t* stab = tabs;
    uint32_t* ttab = tabs + ws;
    for (int i = threadIdx.x; i < ws; i += blockDim.x) stab[i] = sbits[(size_t)head * d.sbits_words + i];
    for (int i = threadIdx.x; i < wt; i += blockDim.x) ttab[i] = vsa_stripe_tword(m, d.T, i);
    __syncthreads();
    const long long slot = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    unsigned long long cnt = 0;
    if (slot < d.Npad) {
        const vsa_row_ctx q = vsa_row_init(d, m, slot);
        if (q.real) {
            const long long nruns = (long long)d.nK * d.nseg;
            for (long long r = 0; r < nruns; ++r) {
                const int2 v = __ldg(seg + r);
                cnt += __popc(vsa_run_bits(m, d, q, stab, ttab, v.x & 0xFFFF, v.x >> 16, v.y & 0xFFFF, v.y >> 16));
            }
        }
    }
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, off);
    if ((threadIdx.x & 31) == 0 && cnt) atomicAdd(&kept[head], cnt);
}

__global__ void perm_kernel(vsa_dims d, int layout, int32_t* __restrict__ perm)
{
    const long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= d.Nslots) return;
    int t, h, w;
    perm[p] = vsa_slot_coords_any(d, layout, p, t, h, w) ? (int32_t)(((long long)t * d.H + h) * d.W + w) : -1;
}

// Both token orders as lookup tables: slot -> natural token and back.
__global__ void order_tables_kernel(vsa_dims d, int32_t* __restrict__ s2t, int32_t* __restrict__ t2s)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int layout = blockIdx.y;
    if (i < d.Nslots) {
        int t, h, w;
        const bool real = vsa_slot_coords_any(d, layout, i, t, h, w);
        const long long n = ((long long)t * d.H + h) * d.W + w;
        s2t[layout * d.Nslots + i] = real ? (int32_t)n : -1;
        if (real) t2s[layout * d.N + n] = (int32_t)i;
    }
}

bool tile_fits_unit(int B, int U, int bh, int bw)
{
    if (B >= U) return B % U == 0;
    if (U % B) return false;
    const int hw = bh * bw;
    return (B % hw == 0) || (B % bw == 0 && hw % B == 0) || (bw % B == 0);
}

// Execution pairs: two 128-row blocks whose kv-tile lists hold the same kv
// tiles, in the same order, run in one attention CTA, which loads each K and
// V tile once for both.  Blocks of 256-row q tiles pair with their neighbour
// (both carry the q tile's list); blocks of 64-row q tiles never pair (a
// 128-row block already carries two q tiles' classes).  For 128-row q tiles
// each head takes the partner stride that pairs more blocks: 1 (block 2i
// with 2i + 1, e.g. inside a frame of an SVG spatial head) or one t-slab of
// units (the same spatial unit one slab later, e.g. an SVG temporal head,
// whose kv tiles do not depend on the query's frame).  pair[e] is the
// partner of a leading block, -1 for a block that runs alone, -2 for a block
// that runs in its leader's CTA.
//
// Candidate c of stride st leads with block (c / st) * 2 st + c mod st (the
// blocks whose index / st is even) and partners with the block st later.

// Blocks per t-slab of units, when whole (0 otherwise).
__host__ __device__ inline int pair_slab(const vsa_dims& d)
{
    const long long slab = (long long)d.nTh * d.nTw * d.U;
    return slab % VSA_EXEC_ROWS == 0 ? (int)(slab / VSA_EXEC_ROWS) : 0;
}

// One warp per (head, stride, candidate): flag[head][k][c] = 1 when the two
// blocks list the same kv tiles; votes[head][k] counts them.
__global__ void pair_flags_kernel(vsa_dims d, const int32_t* __restrict__ list_cnt,
                                  const int32_t* __restrict__ list, int8_t* __restrict__ flag,
                                  int* __restrict__ votes)
{
    const int nC = (d.nE + 1) / 2;                     // candidates per stride (at most)
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= (long long)d.heads * 2 * nC) return;
    const int head = (int)(gw / (2 * nC));
    const int k = (int)(gw / nC) & 1;
    const int c = (int)(gw % nC);
    const int F = pair_slab(d);
    const int st = k == 0 ? 1 : F;
    int same = 0;
    if (d.Bq == 128 && st >= 1 && !(k == 1 && st == 1)) {
        const int ea = (c / st) * 2 * st + c % st, eb = ea + st;
        if (eb < d.nE) {
            const int ca = list_cnt[(size_t)head * d.nE + ea];
            if (ca > 0 && ca == list_cnt[(size_t)head * d.nE + eb]) {
                const int32_t* la = list + ((size_t)head * d.nE + ea) * d.nK;
                const int32_t* lb = list + ((size_t)head * d.nE + eb) * d.nK;
                bool eq = true;
                for (int i = lane; i < ca; i += 32) eq = eq && VSA_ENTRY_KV(la[i]) == VSA_ENTRY_KV(lb[i]);
                same = __all_sync(0xFFFFFFFFu, eq) ? 1 : 0;
            }
        }
    }
    if (lane == 0) {
        flag[((size_t)head * 2 + k) * nC + c] = (int8_t)same;
        if (same) atomicAdd(&votes[head * 2 + k], 1);
    }
}

// One thread per (head, block): the partner array from the stride each head
// takes (the one with more pairs; the neighbour on ties).
__global__ void pair_assign_kernel(vsa_dims d, const int8_t* __restrict__ flag, const int* __restrict__ votes,
                                   int32_t* __restrict__ pair)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)d.heads * d.nE) return;
    const int head = (int)(i / d.nE), e = (int)(i % d.nE);
    int v = -1;
    if (d.Bq == 256) {
        v = (e & 1) ? -2 : (e + 1 < d.nE ? e + 1 : -1);
    } else if (d.Bq == 128) {
        const int nC = (d.nE + 1) / 2;
        const int F = pair_slab(d);
        const int k = (F > 1 && votes[head * 2 + 1] > votes[head * 2]) ? 1 : 0;
        const int st = k ? F : 1;
        const int ea = ((e / st) & 1) ? e - st : e;     // the candidate's leader
        const int c = (ea / (2 * st)) * st + ea % st;
        if (ea + st < d.nE && flag[((size_t)head * 2 + k) * nC + c]) v = (ea == e) ? e + st : -2;
    }
    pair[i] = v;
}

// Launch order of the attention grid: heads by decreasing executed steps
// (ties by index), so the longest CTAs start first and the last wave holds
// the short ones.  order[rank] = head; one thread per head.
__global__ void head_order_kernel(int heads, const unsigned long long* __restrict__ steps, int32_t* __restrict__ order)
{
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= heads) return;
    const unsigned long long sh = steps[h];
    int rank = 0;
    for (int g = 0; g < heads; ++g) {
        const unsigned long long sg = steps[g];
        rank += (sg > sh || (sg == sh && g < h)) ? 1 : 0;
    }
    order[rank] = h;
}

unsigned blocks_for(long long n, int threads) { return (unsigned)((n + threads - 1) / threads); }

// Tiles of at most eight boxes (every frame-0-first tile; tile-major tiles of
// at most eight units) take the blocked kernel, the rest one thread per cell.
void launch_tile_map(const vsa_dims& d, const vsa_mask_spec* specs, const uint32_t* sbits, int8_t* map,
                     cudaStream_t s)
{
    const bool few = d.Bq <= kMaxTileBoxes * d.U && d.Bk <= kMaxTileBoxes * d.U && d.heads <= 65535;
    if (few) {
        const dim3 g(blocks_for(d.nK, kMapKB), blocks_for(d.nQ, kMapQB), d.heads);
        tile_map_blocked_kernel<<<g, kMapKB, 0, s>>>(d, specs, sbits, map);
    } else {
        const long long cells = (long long)d.heads * d.nQ * d.nK;
        tile_map_kernel<<<blocks_for(cells, 256), 256, 0, s>>>(d, specs, sbits, map);
    }
}

}  // namespace

int vsa_build_plan_kernels(vsa_plan_s* p, cudaStream_t s)
{
    const vsa_dims& d = p->d;
    VSA_CUDA_TRY(cudaMemsetAsync(p->d_counts, 0, sizeof(unsigned long long) * 3 * d.heads, s));
    VSA_CUDA_TRY(cudaMemsetAsync(p->d_steps, 0, sizeof(unsigned long long) * d.heads, s));
    seg_table_kernel<<<blocks_for((long long)d.nK * d.nseg, 256), 256, 0, s>>>(d, p->d_seg);
    VSA_CUDA_TRY(cudaGetLastError());
    if (p->has_stripe) {
        dim3 g(blocks_for(d.sbits_words, 128), d.heads);
        stripe_bits_kernel<<<g, 128, 0, s>>>(d, p->d_specs, p->d_sbits);
        VSA_CUDA_TRY(cudaGetLastError());
    }
    launch_tile_map(d, p->d_specs, p->has_stripe ? p->d_sbits : nullptr, p->d_map, s);
    VSA_CUDA_TRY(cudaGetLastError());
    kv_list_kernel<<<blocks_for((long long)d.heads * d.nE * 32, 256), 256, 0, s>>>(
        d, p->d_specs, p->d_map, p->d_list_cnt, p->d_list, p->d_counts, p->d_steps);
    VSA_CUDA_TRY(cudaGetLastError());
    {
        const long long nC = (d.nE + 1) / 2;
        VSA_CUDA_TRY(cudaMemsetAsync(p->d_pair_votes, 0, sizeof(int) * 2 * d.heads, s));
        pair_flags_kernel<<<blocks_for((long long)d.heads * 2 * nC * 32, 256), 256, 0, s>>>(
            d, p->d_list_cnt, p->d_list, p->d_pair_flag, p->d_pair_votes);
        VSA_CUDA_TRY(cudaGetLastError());
        pair_assign_kernel<<<blocks_for((long long)d.heads * d.nE, 256), 256, 0, s>>>(
            d, p->d_pair_flag, p->d_pair_votes, p->d_pair);
        VSA_CUDA_TRY(cudaGetLastError());
    }
    head_order_kernel<<<blocks_for(d.heads, 256), 256, 0, s>>>(d.heads, p->d_steps, p->d_order);
    VSA_CUDA_TRY(cudaGetLastError());
    return VSA_OK;
}

static int validate_spec(const vsa_mask_spec& m)
{
    if (m.kind < VSA_MASK_FULL || m.kind > VSA_MASK_STRIPE) return VSA_ERR_INVALID_ARG;
    if (m.sink != 0 && m.sink != 1) return VSA_ERR_INVALID_ARG;
    if (m.layout != VSA_LAYOUT_TILE_MAJOR && m.layout != VSA_LAYOUT_FRAME0_FIRST) return VSA_ERR_INVALID_ARG;
    if (m.layout == VSA_LAYOUT_FRAME0_FIRST && m.kind != VSA_MASK_SVG_TEMPORAL && m.kind != VSA_MASK_FULL)
        return VSA_ERR_UNSUPPORTED;
    if (m.tile_round != 0 && m.tile_round != 1) return VSA_ERR_INVALID_ARG;
    if (m.tile_round && m.kind != VSA_MASK_FULL && m.kind != VSA_MASK_SVG_SPATIAL && m.kind != VSA_MASK_SVG_TEMPORAL)
        return VSA_ERR_UNSUPPORTED;
    const int lim = 1 << 20;
    switch (m.kind) {
    case VSA_MASK_SVG_SPATIAL:
        if (m.rt < 0 || m.rt > lim) return VSA_ERR_INVALID_ARG;
        break;
    case VSA_MASK_SVG_TEMPORAL:
        if (m.rh < 0 || m.rw < 0 || m.rh > lim || m.rw > lim) return VSA_ERR_INVALID_ARG;
        break;
    case VSA_MASK_STA:
        if (m.kt < 1 || m.kh < 1 || m.kw < 1) return VSA_ERR_INVALID_ARG;
        break;
    case VSA_MASK_STRIPE:
        if (m.Tw < 1 || m.Ts < 1 || m.Sw < 1 || m.Ss < 1) return VSA_ERR_INVALID_ARG;
        if (m.To < -lim || m.To > lim || m.So < -lim || m.So > lim || m.Tw > lim || m.Sw > lim ||
            m.Ts > lim || m.Ss > lim)
            return VSA_ERR_INVALID_ARG;
        break;
    default:
        break;
    }
    return VSA_OK;
}

static void free_plan(vsa_plan_s* p)
{
    if (!p) return;
    cudaFree(p->d_specs);
    cudaFree(p->d_map);
    cudaFree(p->d_list_cnt);
    cudaFree(p->d_list);
    cudaFree(p->d_seg);
    cudaFree(p->d_sbits);
    cudaFree(p->d_counts);
    cudaFree(p->d_steps);
    cudaFree(p->d_status);
    cudaFree(p->d_cand);
    cudaFree(p->d_slot2tok);
    cudaFree(p->d_tok2slot);
    cudaFree(p->d_pair);
    cudaFree(p->d_pair_flag);
    cudaFree(p->d_pair_votes);
    cudaFree(p->d_order);
    delete p;
}

// Validates the grid / unit / tile arguments and derives every shape of a plan.
static int compute_dims(int num_heads, int T, int H, int W, int bt, int bh, int bw, int q_tile,
                        int kv_tile, int has_stripe, vsa_dims* out)
{
    if (num_heads < 1 || T < 1 || H < 1 || W < 1 || bt < 1 || bh < 1 || bw < 1)
        return VSA_ERR_INVALID_ARG;
    if (T > 32767 || H > 32767 || W > 32767 || bt > 32767 || bh > 32767) return VSA_ERR_UNSUPPORTED;
    if (q_tile != 64 && q_tile != 128 && q_tile != 256) return VSA_ERR_UNSUPPORTED;
    if (kv_tile != 64 && kv_tile != 128) return VSA_ERR_UNSUPPORTED;
    if (bw > 32 || (bw & (bw - 1))) return VSA_ERR_UNSUPPORTED;
    vsa_dims d;
    memset(&d, 0, sizeof d);
    d.T = T; d.H = H; d.W = W; d.bt = bt; d.bh = bh; d.bw = bw;
    d.Tp = (T + bt - 1) / bt * bt;
    d.Hp = (H + bh - 1) / bh * bh;
    d.Wp = (W + bw - 1) / bw * bw;
    if (d.Tp > 32767 || d.Hp > 32767 || d.Wp > 32767) return VSA_ERR_UNSUPPORTED;
    d.nTt = d.Tp / bt; d.nTh = d.Hp / bh; d.nTw = d.Wp / bw;
    const long long U = (long long)bt * bh * bw;
    if (U > (1 << 24)) return VSA_ERR_UNSUPPORTED;
    d.U = (int)U;
    if (!tile_fits_unit(q_tile, d.U, bh, bw) || !tile_fits_unit(kv_tile, d.U, bh, bw))
        return VSA_ERR_UNSUPPORTED;
    if (has_stripe && (long long)H * W > 65536) return VSA_ERR_UNSUPPORTED;
    d.heads = num_heads;
    d.Bq = q_tile; d.Bk = kv_tile;
    d.N = (long long)T * H * W;
    d.Npad = (long long)d.Tp * d.Hp * d.Wp;
    const long long L = std::max(VSA_EXEC_ROWS, std::max(q_tile, kv_tile));
    d.Nslots = (d.Npad + L - 1) / L * L;
    if (d.Nslots > (1LL << 24)) return VSA_ERR_UNSUPPORTED;  // 24-bit kv tile index, int32 rows
    d.nQ = (int)(d.Nslots / q_tile);
    d.nK = (int)(d.Nslots / kv_tile);
    d.nE = (int)(d.Nslots / VSA_EXEC_ROWS);
    d.nseg = kv_tile / bw;
    if (kv_tile <= d.U) d.box_nh = (kv_tile % (bh * bw) == 0) ? bh : kv_tile / bw;
    else d.box_nh = 0;
    d.sbits_words = has_stripe ? (int)((2LL * H * W - 1 + 31) / 32 + 1) : 0;
    *out = d;
    return VSA_OK;
}

static void fill_info(const vsa_dims& d, vsa_plan_info_t* out)
{
    out->T = d.T; out->H = d.H; out->W = d.W;
    out->bt = d.bt; out->bh = d.bh; out->bw = d.bw;
    out->num_heads = d.heads;
    out->q_tile = d.Bq; out->kv_tile = d.Bk;
    out->n_q_tiles = d.nQ; out->n_kv_tiles = d.nK;
    out->n_tokens = d.N; out->n_padded = d.Npad; out->n_slots = d.Nslots;
    out->map_bytes = (int64_t)d.heads * d.nQ * d.nK;
}

extern "C" int vsa_layout_info(int num_heads, int T, int H, int W, int bt, int bh, int bw, int q_tile,
                               int kv_tile, vsa_plan_info_t* out)
{
    if (!out) return VSA_ERR_INVALID_ARG;
    vsa_dims d;
    const int r = compute_dims(num_heads, T, H, W, bt, bh, bw, q_tile, kv_tile, 0, &d);
    if (r != VSA_OK) return r;
    fill_info(d, out);
    return VSA_OK;
}

extern "C" int vsa_plan_create(const vsa_mask_spec* specs, int num_heads, int T, int H, int W,
                               int bt, int bh, int bw, int q_tile, int kv_tile, void* stream,
                               vsa_plan_t* out)
{
    if (!out) return VSA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!specs || num_heads < 1) return VSA_ERR_INVALID_ARG;
    int has_stripe = 0;
    for (int h = 0; h < num_heads; ++h) {
        const int r = validate_spec(specs[h]);
        if (r != VSA_OK) return r;
        has_stripe |= specs[h].kind == VSA_MASK_STRIPE;
    }
    vsa_dims d;
    {
        const int r = compute_dims(num_heads, T, H, W, bt, bh, bw, q_tile, kv_tile, has_stripe, &d);
        if (r != VSA_OK) return r;
    }

    vsa_plan_s* p = new (std::nothrow) vsa_plan_s;
    if (!p) return VSA_ERR_OOM;
    memset(p, 0, sizeof *p);
    p->d = d;
    p->has_stripe = has_stripe;
    if (cudaGetDevice(&p->device) != cudaSuccess) { delete p; return VSA_ERR_CUDA; }
    bool ok = true;
    ok = ok && cudaMalloc(&p->d_specs, sizeof(vsa_mask_spec) * num_heads) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_map, (size_t)num_heads * d.nQ * d.nK) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_list_cnt, sizeof(int32_t) * (size_t)num_heads * d.nE) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_list, sizeof(int32_t) * (size_t)num_heads * d.nE * d.nK) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_pair, sizeof(int32_t) * (size_t)num_heads * d.nE) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_pair_flag, (size_t)num_heads * 2 * ((d.nE + 1) / 2)) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_pair_votes, sizeof(int) * 2 * (size_t)num_heads) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_order, sizeof(int32_t) * (size_t)num_heads) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_seg, sizeof(int2) * (size_t)d.nK * d.nseg) == cudaSuccess;
    if (has_stripe)
        ok = ok && cudaMalloc(&p->d_sbits, sizeof(uint32_t) * (size_t)num_heads * d.sbits_words) ==
                       cudaSuccess;
    ok = ok && cudaMalloc(&p->d_counts, sizeof(unsigned long long) * 3 * num_heads) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_steps, sizeof(unsigned long long) * num_heads) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_status, sizeof(unsigned int)) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_slot2tok, sizeof(int32_t) * 2 * (size_t)d.Nslots) == cudaSuccess;
    ok = ok && cudaMalloc(&p->d_tok2slot, sizeof(int32_t) * 2 * (size_t)d.N) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        free_plan(p);
        return VSA_ERR_OOM;
    }
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(p->d_specs, specs, sizeof(vsa_mask_spec) * num_heads, cudaMemcpyHostToDevice,
                        s) != cudaSuccess ||
        cudaMemsetAsync(p->d_status, 0, sizeof(unsigned int), s) != cudaSuccess) {
        free_plan(p);
        return VSA_ERR_CUDA;
    }
    // the host copy of specs may be released as soon as the copy is done
    if (cudaStreamSynchronize(s) != cudaSuccess) {
        free_plan(p);
        return VSA_ERR_CUDA;
    }
    order_tables_kernel<<<dim3(blocks_for(d.Nslots, 256), 2), 256, 0, s>>>(d, p->d_slot2tok, p->d_tok2slot);
    if (cudaGetLastError() != cudaSuccess) {
        free_plan(p);
        return VSA_ERR_CUDA;
    }
    const int r = vsa_build_plan_kernels(p, s);
    if (r != VSA_OK) {
        free_plan(p);
        return r;
    }
    *out = p;
    return VSA_OK;
}

// Launch helpers for other translation units (same kernels and launch shapes
// as the plan build above).
int vsa_dims_for(int num_heads, int T, int H, int W, int bt, int bh, int bw, int q_tile, int kv_tile,
                 int has_stripe, vsa_dims* out)
{
    return compute_dims(num_heads, T, H, W, bt, bh, bw, q_tile, kv_tile, has_stripe, out);
}

int vsa_check_spec(const vsa_mask_spec* m) { return validate_spec(*m); }

int vsa_launch_stripe_bits(const vsa_dims& d, const vsa_mask_spec* specs, uint32_t* sbits, cudaStream_t s)
{
    dim3 g(blocks_for(d.sbits_words, 128), d.heads);
    stripe_bits_kernel<<<g, 128, 0, s>>>(d, specs, sbits);
    return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int vsa_launch_tile_map(const vsa_dims& d, const vsa_mask_spec* specs, const uint32_t* sbits, int8_t* map,
                        cudaStream_t s)
{
    launch_tile_map(d, specs, sbits, map, s);
    return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

extern "C" int vsa_plan_build(vsa_plan_t plan, void* stream)
{
    if (!plan) return VSA_ERR_INVALID_ARG;
    return vsa_build_plan_kernels(plan, (cudaStream_t)stream);
}

extern "C" int vsa_plan_info(vsa_plan_t plan, vsa_plan_info_t* out)
{
    if (!plan || !out) return VSA_ERR_INVALID_ARG;
    fill_info(plan->d, out);
    return VSA_OK;
}

extern "C" int vsa_plan_tile_map(vsa_plan_t plan, int8_t* host_dst, size_t bytes, void* stream)
{
    if (!plan || !host_dst) return VSA_ERR_INVALID_ARG;
    const size_t need = (size_t)plan->d.heads * plan->d.nQ * plan->d.nK;
    if (bytes < need) return VSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    VSA_CUDA_TRY(cudaMemcpyAsync(host_dst, plan->d_map, need, cudaMemcpyDeviceToHost, s));
    VSA_CUDA_TRY(cudaStreamSynchronize(s));
    return VSA_OK;
}

extern "C" int vsa_plan_tile_counts(vsa_plan_t plan, int64_t* host_counts, size_t n, void* stream)
{
    if (!plan || !host_counts || n < (size_t)3 * plan->d.heads) return VSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    VSA_CUDA_TRY(cudaMemcpyAsync(host_counts, plan->d_counts,
                                 sizeof(unsigned long long) * 3 * plan->d.heads,
                                 cudaMemcpyDeviceToHost, s));
    VSA_CUDA_TRY(cudaStreamSynchronize(s));
    return VSA_OK;
}

extern "C" int vsa_plan_exec_steps(vsa_plan_t plan, int64_t* host_dst, size_t n, void* stream)
{
    if (!plan || !host_dst || n < (size_t)plan->d.heads) return VSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    VSA_CUDA_TRY(cudaMemcpyAsync(host_dst, plan->d_steps, sizeof(unsigned long long) * plan->d.heads,
                                 cudaMemcpyDeviceToHost, s));
    VSA_CUDA_TRY(cudaStreamSynchronize(s));
    return VSA_OK;
}

extern "C" int vsa_plan_exec_pairs(vsa_plan_t plan, int32_t* host_dst, size_t n, void* stream)
{
    if (!plan || !host_dst || n < (size_t)plan->d.heads * plan->d.nE) return VSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    VSA_CUDA_TRY(cudaMemcpyAsync(host_dst, plan->d_pair, sizeof(int32_t) * (size_t)plan->d.heads * plan->d.nE,
                                 cudaMemcpyDeviceToHost, s));
    VSA_CUDA_TRY(cudaStreamSynchronize(s));
    return VSA_OK;
}

extern "C" int vsa_plan_kept_pairs(vsa_plan_t plan, int64_t* host_dst, size_t n, void* stream)
{
    if (!plan || !host_dst || n < (size_t)plan->d.heads) return VSA_ERR_INVALID_ARG;
    const vsa_dims& d = plan->d;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned long long* tmp = nullptr;
    if (cudaMalloc(&tmp, sizeof(unsigned long long) * d.heads) != cudaSuccess) {
        cudaGetLastError();
        return VSA_ERR_OOM;
    }
    const int smem = 4 * ((plan->has_stripe ? d.sbits_words : 0) + vsa_ttab_words(d.T));
    cudaError_t e = cudaMemsetAsync(tmp, 0, sizeof(unsigned long long) * d.heads, s);
    if (e == cudaSuccess && smem > 48 * 1024)
        e = cudaFuncSetAttribute(kept_pairs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) {
        dim3 g(blocks_for(d.Npad, 256), d.heads);
        kept_pairs_kernel<<<g, 256, smem, s>>>(d, plan->d_specs, plan->d_sbits, plan->d_seg, tmp);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(host_dst, tmp, sizeof(unsigned long long) * d.heads, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    cudaFree(tmp);
    return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

extern "C" int vsa_plan_perm(vsa_plan_t plan, int32_t* host_dst, size_t n, void* stream)
{
    return vsa_plan_layout_perm(plan, VSA_LAYOUT_TILE_MAJOR, host_dst, n, stream);
}

extern "C" int vsa_plan_layout_perm(vsa_plan_t plan, int layout, int32_t* host_dst, size_t n, void* stream)
{
    if (!plan || !host_dst || n < (size_t)plan->d.Nslots) return VSA_ERR_INVALID_ARG;
    if (layout != VSA_LAYOUT_TILE_MAJOR && layout != VSA_LAYOUT_FRAME0_FIRST) return VSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t* tmp = nullptr;
    if (cudaMalloc(&tmp, sizeof(int32_t) * plan->d.Nslots) != cudaSuccess) {
        cudaGetLastError();
        return VSA_ERR_OOM;
    }
    perm_kernel<<<blocks_for(plan->d.Nslots, 256), 256, 0, s>>>(plan->d, layout, tmp);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(host_dst, tmp, sizeof(int32_t) * plan->d.Nslots, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    cudaFree(tmp);
    return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

extern "C" int vsa_plan_destroy(vsa_plan_t plan)
{
    if (!plan) return VSA_ERR_INVALID_ARG;
    int prev = -1;
    const int dev = plan->device;
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
    const cudaError_t e = cudaDeviceSynchronize();
    free_plan(plan);
    if (prev >= 0 && prev != dev) cudaSetDevice(prev);
    return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

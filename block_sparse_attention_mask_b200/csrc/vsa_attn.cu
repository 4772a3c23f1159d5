// Block-sparse attention forward for sm_100a: TMA + tcgen05 (TMEM) + online
// softmax, with separate full-tile and boundary-tile paths.
//
// What it computes: for each real query row, softmax over the kept keys of
// scale * q.k, times v ("Fast Video Generation with Sliding Tile Attention",
// section 2, Eq. 1), visiting only the kv tiles the plan lists for the query
// block, skipping empty tiles, running full tiles with no per-element mask
// and evaluating the exact predicate only on boundary tiles; partial results
// merge by online softmax ("Sparse VideoGen: accelerating video diffusion
// attention on TPU", "avoid in-tile masking when nothing needs masking").
//
// One CTA = one (batch, head, 128-row query block).  The block's kv-tile list
// is split between two softmax warpgroups by position: warpgroup X takes the
// entries j with j mod 2 = X and keeps its own running max, running sum and
// output accumulator O_X, so the two are independent streams that the tensor
// core serves alternately; the epilogue merges the two partial softmaxes.  On
// every scheduler one warp of each warpgroup runs, and as the two streams are
// out of phase, one warp's exponentials (MUFU) overlap the other's loads,
// masks and maxima.  12 warps:
//   warp 8      TMA producer: lane 0 loads Q once and the K tiles of the list
//               through a K ring, lane 1 the V tiles through a V ring
//               (full/empty mbarriers per stage).
//   warp 9      MMA issuer: the whole warp runs the loop so the descriptor
//               arithmetic stays warp-uniform; one elected lane issues.
//               S_j = Q K_j^T (both operands in shared memory) into S_{j mod 2};
//               O_{j mod 2} += P_j V_j with P_j read from TMEM (it overwrites
//               the first BK/2 columns of S_{j mod 2}) and V as an MN-major
//               shared-memory operand.  kind::f16, bf16 in, fp32 accumulate;
//               tcgen05.commit signals the mbarriers.  Issue order: QK_0,
//               QK_1, PV_0, QK_2, PV_1, QK_3, ...; the tensor core runs one
//               thread's MMAs in order, so by the time S_{j+2} is complete,
//               PV_j has read P_j and finished accumulating into O_{j mod 2}.
//   warps 10,11 mask workers: for every boundary tile of the list, thread t
//               evaluates the exact predicate for rows t and t + 64 and stores
//               the per-row keep bits in a shared-memory ring ahead of the
//               softmax, so the softmax only applies them.
//   warps 0..3  softmax warpgroup 0 and warps 4..7 warpgroup 1: thread r of a
//               warpgroup owns query row r (TMEM lane r).  Per tile: load S_j,
//               apply the keep bits on boundary tiles only, keep the running
//               max (log2 units; O_X rescaled in TMEM only when the max grows
//               by more than 8, a factor 256) and sum in fp32, and write P_j as
//               bf16.  At the end both warpgroups merge their partial results
//               and write o and lse, each half of the head dimension.
// TMEM columns: S0 [0,BK), S1 [BK,2BK), O0 [2BK,2BK+D), O1 [2BK+D,2BK+2D):
// 512 columns for D = BK = 128.
// Every mbarrier wait is bounded: on expiry the CTA records VSA_DEV_TIMEOUT
// in the plan's status word, all roles leave their loops, TMEM is freed and
// the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "vsa_internal.h"
#include "vsa_sm100.cuh"

namespace {

constexpr int kSoftmaxWarps = 8;                  // warps 0..7: two warpgroups
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kMaskWarp0 = 10;                    // warps 10, 11
constexpr int kThreads = 32 * (kMaskWarp0 + 2);
// Registers per thread: 168 at launch (65536 / 384 rounded down to 8); the
// softmax warpgroups raise theirs with setmaxnreg and the third warpgroup
// (producer, MMA, mask workers) gives the difference back.
constexpr int kRegsLaunch = 168;
constexpr int kMaskSlots = 4;                     // boundary-tile masks in flight
constexpr int kRows = VSA_EXEC_ROWS;              // 128 query rows per CTA
constexpr float kRescaleThreshold = 8.0f;         // log2 units

template <int D, int BK>
struct Cfg {
    static constexpr int KV_BYTES = BK * D * 2;
    static constexpr int Q_BYTES = kRows * D * 2;
    // a softmax thread holds a whole S row (BK values) and its bf16 P
    static constexpr int REGS_SOFTMAX = BK == 128 ? 208 : 176;
    static constexpr int REGS_OTHER = 3 * kRegsLaunch - 2 * REGS_SOFTMAX;
    static_assert(REGS_OTHER >= 24 && REGS_OTHER % 8 == 0, "setmaxnreg split");
    static constexpr int RING_BYTES = 192 * 1024 - Q_BYTES;
    // K stages are refilled once QK_j completes, V stages only once PV_j
    // does, so K gets the deeper ring
    static constexpr int STAGES_V = (RING_BYTES / KV_BYTES) / 2 > 4 ? 4 : (RING_BYTES / KV_BYTES) / 2;
    static constexpr int STAGES_K = (RING_BYTES / KV_BYTES - STAGES_V) > 4 ? 4 : (RING_BYTES / KV_BYTES - STAGES_V);
    static_assert(STAGES_V >= 2 && STAGES_K >= 2, "shared-memory ring");
    static constexpr int COL_S0 = 0;
    static constexpr int COL_S1 = BK;
    static constexpr int COL_O0 = 2 * BK;
    static constexpr int COL_O1 = 2 * BK + D;
    // Q also goes to TMEM (bf16 pairs, D/2 columns) when it fits: QK then
    // reads only K from shared memory (the TS form), which keeps the
    // half-width QK of 64-key tiles at the math rate
    static constexpr bool Q_TMEM = 2 * BK + 2 * D + D / 2 <= 512;
    static constexpr int COL_Q = 2 * BK + 2 * D;
    static constexpr int COLS_USED = COL_Q + (Q_TMEM ? D / 2 : 0);
    static constexpr int TMEM_COLS = COLS_USED <= 256 ? 256 : 512;
    static_assert(COLS_USED <= 512, "TMEM budget");
    // shared memory map (offsets from a 1024-aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES_K * KV_BYTES;
    // boundary masks: [slot][word][row] uint32, word = 32 key columns
    static constexpr int OFF_MASK = OFF_V + STAGES_V * KV_BYTES;
    static constexpr int MASK_SLOT_WORDS = (BK / 32) * kRows;
    // per-warpgroup row statistics (running max, running sum) for the merge
    static constexpr int OFF_STAT = OFF_MASK + kMaskSlots * MASK_SLOT_WORDS * 4;
    // per-row mask context (query coordinates, STA window), read on boundary tiles
    static constexpr int OFF_ROWCTX = OFF_STAT + 2 * kRows * 8;
    static constexpr int OFF_BAR = OFF_ROWCTX + kRows * (int)sizeof(vsa_row_ctx);
    // barriers: k_full[SK], k_empty[SK], v_full[SV], v_empty[SV], q_full,
    //           s_full[2], p_full[2], pv_done[2], mask_full[M], mask_empty[M], mma_drain
    static constexpr int NBAR = 2 * STAGES_K + 2 * STAGES_V + 9 + 2 * kMaskSlots;
    // tmem addr, abort flag, and for the teardown after an abort: K and V
    // copies started, MMAs started (4 bytes each)
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_TAB = (OFF_MISC + 20 + 15) / 16 * 16;
    // instruction descriptors (kind::f16): D fp32, A and B bf16
    //   bits [4,6) D format = 1 (f32); [7,10) A = 1 (bf16); [10,13) B = 1 (bf16);
    //   bit 15 A major (0 = K); bit 16 B major (1 = MN); [17,23) N >> 3; [24,29) M >> 4
    static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) |
                                         ((uint32_t)(BK >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
};

struct AttnParams {
    CUtensorMap tm_q, tm_k, tm_v;       // 2D [rows = B*heads*n_slots, D] bf16, box {64, 128 | BK}
    __nv_bfloat16* o;
    float* lse;
    const int32_t* list_cnt;
    const int32_t* list;
    const int32_t* pair;                // [heads][nE]: partner of a pair's leader, -1 alone, -2 in the leader's CTA
    const int32_t* order;               // [heads]: heads by decreasing executed steps
    const int2* seg;
    const vsa_mask_spec* specs;
    const uint32_t* sbits;
    unsigned int* status;
    vsa_dims d;
    float scale_log2;
    int tab_words_s;                    // stripe offset table words in smem
    int tab_words_t;                    // stripe frame-offset table words in smem
};

// Keep bits of query row q for a kv tile that is one box inside a unit
// (box_nh > 0): run r of the tile (bw keys sharing t and h) sits at
// (t0 + r / box_nh, h0 + r mod box_nh) with the same first column w0 and the
// same number of real keys for every run, so a run costs a few operations.
// v is the tile's first run descriptor; bit c of words[c / 32] is key c.
template <int KIND, int BK>
__device__ __forceinline__ void box_row_bits(const vsa_mask_spec& m, const vsa_dims& d, const vsa_row_ctx& q,
                                             const uint32_t* stab, const uint32_t* ttab, int2 v, bool tile_real,
                                             uint32_t (&words)[BK / 32])
{
    const int t0 = v.x & 0xFFFF, h0 = v.x >> 16, w0 = v.y & 0xFFFF;
    const int bw = d.bw;
    const int wv = tile_real ? max(0, min(bw, d.W - w0)) : 0;
    const uint32_t vm = vsa_low_bits(wv);
    // row-invariant parts for this tile
    uint32_t wmask = 0;             // temporal: kept w offsets of a run
    bool sta_in = false;            // STA: the tile's unit is in the row's window
    if (KIND == VSA_MASK_SVG_TEMPORAL) {
        const int lo = max(q.wq - m.rw, w0) - w0;
        const int hi = min(q.wq + m.rw, w0 + wv - 1) - w0;
        wmask = (lo <= hi) ? (vsa_low_bits(hi - lo + 1) << lo) : 0u;
    }
    if (KIND == VSA_MASK_STA) {
        const int ut = t0 / d.bt, uh = h0 / d.bh, uw = w0 / d.bw;
        sta_in = ut >= q.sta_t && ut < q.sta_t + q.kk_t && uh >= q.sta_h && uh < q.sta_h + q.kk_h &&
                 uw >= q.sta_w && uw < q.sta_w + q.kk_w;
    }
#pragma unroll
    for (int wi = 0; wi < BK / 32; ++wi) words[wi] = 0u;
    uint32_t acc = 0;
    int tt = t0, dh = 0;
    bool tvalid = false, sinkhit = false, tkeep = true;
    int xbase = 0;
    for (int r = 0; r < d.nseg; ++r) {
        if (dh == 0) {              // a new t-slice of the tile: everything but h is fixed
            tvalid = q.real && tt < d.T;
            sinkhit = m.sink && tt == 0;
            tkeep = true;
            if (KIND == VSA_MASK_SVG_SPATIAL) tkeep = vsa_iabs(tt - q.tq) <= m.rt;
            if (KIND == VSA_MASK_STRIPE) {
                const int it = tt - q.tq + d.T - 1;
                tkeep = tvalid && ((ttab[it >> 5] >> (it & 31)) & 1u);
            }
            xbase = h0 * d.W + w0 - q.sq + d.H * d.W - 1;
        }
        const int hh = h0 + dh;
        uint32_t b = 0;
        if (KIND == VSA_MASK_STRIPE) {
            const int x = xbase + dh * d.W;
            const uint32_t win = __funnelshift_r(stab[x >> 5], stab[(x >> 5) + 1], x & 31) & vm;
            b = tkeep ? win : 0u;
        } else if (KIND == VSA_MASK_SVG_TEMPORAL) {
            b = vsa_iabs(hh - q.hq) <= m.rh ? wmask : 0u;
        } else if (KIND == VSA_MASK_SVG_SPATIAL) {
            b = tkeep ? vm : 0u;
        } else if (KIND == VSA_MASK_STA) {
            b = sta_in ? vm : 0u;
        } else {
            b = vm;
        }
        if (sinkhit) b = vm;
        if (!(tvalid && hh < d.H)) b = 0u;
        const int col = r * bw;
        acc |= b << (col & 31);
        if (((col + bw) & 31) == 0) {          // last run of a 32-key word (bw divides 32)
#pragma unroll
            for (int wi = 0; wi < BK / 32; ++wi) words[wi] = (col >> 5) == wi ? acc : words[wi];
            acc = 0;
        }
        if (++dh == d.box_nh) {
            dh = 0;
            ++tt;
        }
    }
}

// Keep bits of query row q for kv tile kv of a frame-0-first head (temporal or
// full mask): the frame-0 keys of the tile come in runs along w inside one
// latent row, kept by the sink or by the w window; every other key sits in a
// run of frames of one spatial position, all kept or none.
template <int BK>
__device__ __forceinline__ void f0_row_bits(const vsa_mask_spec& m, const vsa_dims& d, const vsa_row_ctx& q,
                                            int kv, uint32_t (&words)[BK / 32])
{
#pragma unroll
    for (int wi = 0; wi < BK / 32; ++wi) words[wi] = 0u;
    if (!q.real) return;
    const long long HW = (long long)d.H * d.W, N = HW * d.T;
    const long long p0 = (long long)kv * BK, p1 = p0 + BK;
    const bool all_keys = m.kind == VSA_MASK_FULL;
    auto set_range = [&](int lo, int hi) {          // tile bits [lo, hi), 0 <= lo < hi <= BK
#pragma unroll
        for (int wi = 0; wi < BK / 32; ++wi) {
            const int a = max(lo, 32 * wi), b = min(hi, 32 * wi + 32);
            if (a < b) words[wi] |= (b - a == 32 ? 0xFFFFFFFFu : ((1u << (b - a)) - 1u)) << (a - 32 * wi);
        }
    };
    long long p = p0;
    while (p < p1 && p < HW) {                      // frame 0
        const int h = (int)(p / d.W), w = (int)(p - (long long)h * d.W);
        const int len = (int)min((long long)(d.W - w), min(p1, HW) - p);
        int lo = 0, hi = len;
        if (!(m.sink || all_keys)) {
            if (vsa_iabs(h - q.hq) > m.rh) {
                hi = 0;
            } else {
                lo = max(q.wq - m.rw, w) - w;
                hi = min(q.wq + m.rw + 1, w + len) - w;
            }
        }
        if (lo < hi) set_range((int)(p - p0) + lo, (int)(p - p0) + hi);
        p += len;
    }
    if (d.T > 1 && p < p1 && p < N) {               // frames 1..T-1, position-major
        const int F = d.T - 1;
        const long long r = p - HW;
        const long long pos = r / F;
        int f = (int)(r - pos * F);
        int h = (int)(pos / d.W), w = (int)(pos - (long long)h * d.W);
        while (p < p1 && p < N) {
            const int len = (int)min((long long)(F - f), min(p1, N) - p);
            if (all_keys || (vsa_iabs(h - q.hq) <= m.rh && vsa_iabs(w - q.wq) <= m.rw))
                set_range((int)(p - p0), (int)(p - p0) + len);
            p += len;
            f = 0;
            if (++w == d.W) {
                w = 0;
                ++h;
            }
        }
    }
}
// Keep bits of query row q for a kv tile that is one box inside a unit, for
// the masks whose kept keys in such a tile form one rectangle per t-slice:
// full, SVG spatial, SVG temporal and STA.  In a slice every kept latent row
// keeps the same columns (all real ones; for the temporal mask the query's w
// window) and the kept rows are one range (all real rows; for the temporal
// mask the query's h window), so the words come from the range and the
// column pattern replicated every bw bits, with no per-run loop.  Same bits
// as box_row_bits for these kinds; the frame-0 sink keeps a whole slice.
template <int BK>
__device__ __forceinline__ void rect_row_bits(const vsa_mask_spec& m, const vsa_dims& d, const vsa_row_ctx& q,
                                              int2 v, bool tile_real, uint32_t (&words)[BK / 32])
{
    const int t0 = v.x & 0xFFFF, h0 = v.x >> 16, w0 = v.y & 0xFFFF;
    const int bw = d.bw, nh = d.box_nh;
    const int wv = tile_real ? max(0, min(bw, d.W - w0)) : 0;
    const uint32_t vm = vsa_low_bits(wv);
    const uint32_t rep1 = bw >= 32 ? 1u : 0xFFFFFFFFu / ((1u << bw) - 1u);   // one bit per run of bw
    const int hv = min(nh, d.H - h0);              // latent rows of a slice inside the grid
    int klo = 0, khi = hv - 1;                     // the mask's own rows and columns
    uint32_t kpat = vm;
    bool tile_on = true;
    if (m.kind == VSA_MASK_SVG_TEMPORAL) {
        klo = max(klo, q.hq - m.rh - h0);
        khi = min(khi, q.hq + m.rh - h0);
        const int lo = max(q.wq - m.rw, w0) - w0;
        const int hi = min(q.wq + m.rw, w0 + wv - 1) - w0;
        kpat = (lo <= hi) ? (vsa_low_bits(hi - lo + 1) << lo) : 0u;
    } else if (m.kind == VSA_MASK_STA) {
        const int ut = t0 / d.bt, uh = h0 / d.bh, uw = w0 / d.bw;
        tile_on = ut >= q.sta_t && ut < q.sta_t + q.kk_t && uh >= q.sta_h && uh < q.sta_h + q.kk_h &&
                  uw >= q.sta_w && uw < q.sta_w + q.kk_w;
    }
#pragma unroll
    for (int wi = 0; wi < BK / 32; ++wi) words[wi] = 0u;
    const int ns = d.nseg / nh;                    // t-slices of the tile
    for (int sl = 0; sl < ns; ++sl) {
        const int tt = t0 + sl;
        int lo = 0, hi = hv - 1;
        uint32_t pat = vm;
        if (!(m.sink && tt == 0)) {
            if (m.kind == VSA_MASK_SVG_TEMPORAL) {
                lo = klo;
                hi = khi;
                pat = kpat;
            }
            const bool on = m.kind == VSA_MASK_SVG_SPATIAL ? vsa_iabs(tt - q.tq) <= m.rt : tile_on;
            if (!on) hi = -1;
        }
        if (!q.real || tt >= d.T) hi = -1;
        const int a = (sl * nh + lo) * bw, b = (sl * nh + hi + 1) * bw;    // bit range of the kept runs
        const uint32_t rep = pat * rep1;
#pragma unroll
        for (int wi = 0; wi < BK / 32; ++wi) {
            const int x0 = max(a, 32 * wi), x1 = min(b, 32 * wi + 32);
            if (x0 < x1) words[wi] |= (vsa_low_bits(x1 - x0) << (x0 - 32 * wi)) & rep;
        }
    }
}

// Key of a single-box tile's keep bits for one query row: the tile's first
// run descriptor (x = t | h << 16), with the frame reduced to what the mask
// reads of it when the tile is one t-slice: full and SVG temporal masks see
// the key's frame only as frame 0 (the sink) or past the grid.  Tiles with
// equal keys have equal bits, so a row reuses the previous tile's bits while
// the key stays the same (kv lists visit all frames of a unit position in a
// row).
__device__ __forceinline__ int bits_key_x(const vsa_mask_spec& m, const vsa_dims& d, int x)
{
    if (d.nseg != d.box_nh || (m.kind != VSA_MASK_SVG_TEMPORAL && m.kind != VSA_MASK_FULL)) return x;
    const int t = x & 0xFFFF;
    return (x & ~0xFFFF) | (t == 0 ? 0 : t < d.T ? 1 : 2);
}

// Keep bits of a single-box boundary tile: the stripe mask run by run, the
// others as a rectangle per slice.
template <int BK>
__device__ __forceinline__ void box_tile_bits(const vsa_mask_spec& m, const vsa_dims& d, const vsa_row_ctx& q,
                                              const uint32_t* stab, const uint32_t* ttab, int2 v, bool tile_real,
                                              uint32_t (&words)[BK / 32])
{
    if (m.kind == VSA_MASK_STRIPE) {
        vsa_mask_spec mk = m;
        mk.kind = VSA_MASK_STRIPE;
        box_row_bits<VSA_MASK_STRIPE, BK>(mk, d, q, stab, ttab, v, tile_real, words);
    } else {
        rect_row_bits<BK>(m, d, q, v, tile_real, words);
    }
}

// Stripe keep bits of a single-slice tile before the frame test: run r
// (latent row h0 + r) keeps the columns the intra-frame offset table allows.
// The frame enters only as one bit for the whole tile (the frame-offset
// table), so these words serve every frame of the unit position.
template <int BK>
__device__ __forceinline__ void stripe_win_words(const vsa_dims& d, const vsa_row_ctx& q, const uint32_t* stab, int2 v,
                                                 bool tile_real, uint32_t (&words)[BK / 32])
{
    const int h0 = v.x >> 16, w0 = v.y & 0xFFFF;
    const int bw = d.bw;
    const int wv = tile_real ? max(0, min(bw, d.W - w0)) : 0;
    const uint32_t vm = vsa_low_bits(wv);
#pragma unroll
    for (int wi = 0; wi < BK / 32; ++wi) words[wi] = 0u;
    const int xbase = h0 * d.W + w0 - q.sq + d.H * d.W - 1;
    uint32_t acc = 0;
    for (int r = 0; r < d.nseg; ++r) {
        uint32_t b = 0u;
        if (h0 + r < d.H) {
            const int x = xbase + r * d.W;
            b = __funnelshift_r(stab[x >> 5], stab[(x >> 5) + 1], x & 31) & vm;
        }
        const int col = r * bw;
        acc |= b << (col & 31);
        if (((col + bw) & 31) == 0) {
#pragma unroll
            for (int wi = 0; wi < BK / 32; ++wi) words[wi] = (col >> 5) == wi ? acc : words[wi];
            acc = 0;
        }
    }
}

// Keep bits of a single-box boundary tile for one query row, reusing the
// words of the row's previous tile where they are the same: cw / (ck_x, ck_y)
// hold the last computed words and their key.  Stripe tiles of one t-slice
// cache the frame-free window words and apply the frame bit per tile (the
// sink frame is computed whole); other masks cache by bits_key_x.
template <int BK>
__device__ __forceinline__ void cached_box_bits(const vsa_mask_spec& m, const vsa_dims& d, const vsa_row_ctx& q,
                                                const uint32_t* stab, const uint32_t* ttab, int2 v, bool tile_real,
                                                uint32_t (&cw)[BK / 32], int& ck_x, int& ck_y,
                                                uint32_t (&mw)[BK / 32])
{
    if (m.kind == VSA_MASK_STRIPE && d.nseg == d.box_nh) {
        const int t0 = v.x & 0xFFFF;
        if (!q.real || t0 >= d.T) {
#pragma unroll
            for (int wi = 0; wi < BK / 32; ++wi) mw[wi] = 0u;
            return;
        }
        if (m.sink && t0 == 0) {
            box_tile_bits<BK>(m, d, q, stab, ttab, v, tile_real, mw);
            return;
        }
        const int kx = v.x | 0xFFFF;                 // the frame does not enter the window words
        if (kx != ck_x || v.y != ck_y) {
            stripe_win_words<BK>(d, q, stab, v, tile_real, cw);
            ck_x = kx;
            ck_y = v.y;
        }
        const int it = t0 - q.tq + d.T - 1;
        const bool tk = (ttab[it >> 5] >> (it & 31)) & 1u;
#pragma unroll
        for (int wi = 0; wi < BK / 32; ++wi) mw[wi] = tk ? cw[wi] : 0u;
        return;
    }
    const int kx = bits_key_x(m, d, v.x);
    if (kx != ck_x || v.y != ck_y) {
        box_tile_bits<BK>(m, d, q, stab, ttab, v, tile_real, cw);
        ck_x = kx;
        ck_y = v.y;
    }
#pragma unroll
    for (int wi = 0; wi < BK / 32; ++wi) mw[wi] = cw[wi];
}

// Mask-worker loop for kv tiles made of several boxes (box_nh = 0),
// specialised on the mask kind (uniform per CTA) so that no per-run branch on
// the kind remains.  Thread t of the two mask warps writes the keep bits of
// rows t and t + 64 for every boundary tile of the list into slot
// (k mod kMaskSlots) of the ring, k = boundary tiles so far.  The run
// descriptors of a tile (bw keys sharing t and h each) are loaded once per
// warp, one per lane, and broadcast with warp shuffles.
template <int KIND, int BK>
__device__ __forceinline__ void mask_worker_loop(const vsa_mask_spec& m_in, const vsa_dims& d,
                                                 const vsa_row_ctx& q0, const vsa_row_ctx& q1,
                                                 const uint32_t* stab, const uint32_t* ttab,
                                                 const int2* __restrict__ seg, const int32_t* __restrict__ entries,
                                                 int cnt, int t, int lane, uint32_t* maskbuf, uint32_t bar_mf0,
                                                 uint32_t bar_me0, const Ctl& ctl)
{
    constexpr int MASK_SLOT_WORDS = (BK / 32) * kRows;
    vsa_mask_spec m = m_in;
    m.kind = KIND;                                  // lets the predicate's switch fold away
    const int nseg = d.nseg;                        // BK / bw runs per tile, at most BK
    const int bw = d.bw;
    int kb = 0;
    int ent_next = cnt > 0 ? __ldg(entries) : 0;
    for (int j = 0; j < cnt; ++j) {
        const int ent = ent_next;
        if (j + 1 < cnt) ent_next = __ldg(entries + j + 1);
        if (VSA_ENTRY_CLS(ent, 0) != VSA_TILE_BOUNDARY && VSA_ENTRY_CLS(ent, 1) != VSA_TILE_BOUNDARY) continue;
        const int slot = kb % kMaskSlots;
        const int kv = VSA_ENTRY_KV(ent);
        const int2* sg = seg + (size_t)kv * nseg;
        int2 rr[BK / 32];
#pragma unroll
        for (int i = 0; i < BK / 32; ++i) rr[i] = (i * 32 + lane < nseg) ? __ldg(sg + i * 32 + lane) : make_int2(0, 0);
        if (kb >= kMaskSlots &&
            !mbar_wait_warp(bar_me0 + 8u * slot, (uint32_t)(kb / kMaskSlots - 1) & 1, ctl))
            return;
        uint32_t* dst = maskbuf + slot * MASK_SLOT_WORDS;
        uint32_t acc0 = 0, acc1 = 0;
        for (int r = 0; r < nseg; ++r) {
            const int src_reg = r >> 5;
            int2 v = rr[0];
#pragma unroll
            for (int i = 1; i < BK / 32; ++i) v = (src_reg == i) ? rr[i] : v;
            v.x = __shfl_sync(0xFFFFFFFFu, v.x, r & 31);
            v.y = __shfl_sync(0xFFFFFFFFu, v.y, r & 31);
            const int tt = v.x & 0xFFFF, hh = v.x >> 16, w0 = v.y & 0xFFFF, nv = v.y >> 16;
            const uint32_t b0 = vsa_run_bits(m, d, q0, stab, ttab, tt, hh, w0, nv);
            const uint32_t b1 = vsa_run_bits(m, d, q1, stab, ttab, tt, hh, w0, nv);
            const int col = r * bw;                  // first key column of the run
            const int sh = col & 31;                 // runs never straddle a word: bw divides 32
            acc0 |= b0 << sh;
            acc1 |= b1 << sh;
            if (sh + bw == 32) {                     // last run of the 32-column word
                dst[(col >> 5) * kRows + t] = acc0;
                dst[(col >> 5) * kRows + t + 64] = acc1;
                acc0 = 0;
                acc1 = 0;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_mf0 + 8u * slot);
        ++kb;
    }
}

// One 128-row execution block e of (batch, head) hb.
template <int D, int BK>
__device__ __forceinline__ void attn_single(const AttnParams& P, int e, int hb)
{
    using C = Cfg<D, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

    const vsa_dims& d = P.d;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int head = hb % d.heads;
    const long long base_row = (long long)hb * d.Nslots;
    const long long row0 = base_row + (long long)e * kRows;
    const int list_idx = head * d.nE + e;
    const int cnt = P.list_cnt[list_idx];
    const int32_t* entries = P.list + (size_t)list_idx * d.nK;

    const uint32_t s_base = smem_addr(smem);
    const uint32_t bar0 = s_base + C::OFF_BAR;
    auto BAR_KF = [&](int s) { return bar0 + 8u * s; };
    auto BAR_KE = [&](int s) { return bar0 + 8u * (C::STAGES_K + s); };
    auto BAR_VF = [&](int s) { return bar0 + 8u * (2 * C::STAGES_K + s); };
    auto BAR_VE = [&](int s) { return bar0 + 8u * (2 * C::STAGES_K + C::STAGES_V + s); };
    constexpr int B1 = 2 * C::STAGES_K + 2 * C::STAGES_V;
    const uint32_t BAR_QF = bar0 + 8u * B1;
    auto BAR_SF = [&](int x) { return bar0 + 8u * (B1 + 1 + x); };
    auto BAR_PF = [&](int x) { return bar0 + 8u * (B1 + 3 + x); };
    auto BAR_PV = [&](int x) { return bar0 + 8u * (B1 + 5 + x); };
    auto BAR_MF = [&](int k) { return bar0 + 8u * (B1 + 7 + k); };
    auto BAR_ME = [&](int k) { return bar0 + 8u * (B1 + 7 + kMaskSlots + k); };
    const uint32_t BAR_DR = bar0 + 8u * (B1 + 7 + 2 * kMaskSlots);
    const uint32_t BAR_QT = bar0 + 8u * (B1 + 8 + 2 * kMaskSlots);     // Q copied into TMEM
    uint32_t* maskbuf = (uint32_t*)(smem + C::OFF_MASK);
    float2* stat = (float2*)(smem + C::OFF_STAT);
    vsa_row_ctx* rowctx = (vsa_row_ctx*)(smem + C::OFF_ROWCTX);

    uint32_t* tmem_slot = (uint32_t*)(smem + C::OFF_MISC);
    volatile int* abort_flag = (volatile int*)(smem + C::OFF_MISC + 4);
    // for the teardown after an abort, kept in shared memory rather than in
    // registers live across every role: [K copies, V copies, MMAs] started
    volatile int* issued = (volatile int*)(smem + C::OFF_MISC + 8);
    uint32_t* stab = (uint32_t*)(smem + C::OFF_TAB);
    uint32_t* ttab = stab + P.tab_words_s;
    const Ctl ctl{abort_flag, P.status};

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES_K; ++s) {
            mbar_init(BAR_KF(s), 1);
            mbar_init(BAR_KE(s), 1);
        }
        for (int s = 0; s < C::STAGES_V; ++s) {
            mbar_init(BAR_VF(s), 1);
            mbar_init(BAR_VE(s), 1);
        }
        mbar_init(BAR_QF, 1);
        mbar_init(BAR_DR, 1);
        mbar_init(BAR_QT, 4);                           // the four warps of softmax warpgroup 0
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR_SF(x), 1);
            mbar_init(BAR_PF(x), 4);                    // the four warps of softmax warpgroup x
            mbar_init(BAR_PV(x), 1);
        }
        for (int k = 0; k < kMaskSlots; ++k) {
            mbar_init(BAR_MF(k), 2);
            mbar_init(BAR_ME(k), 4);                    // the warpgroup that consumed the slot
        }
        *abort_flag = 0;
        issued[0] = issued[1] = issued[2] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProducerWarp) {
        // ---------------- TMA producer: lane 0 Q and K, lane 1 V ----------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
        if (lane == 0 && cnt > 0) {
            mbar_expect_tx(BAR_QF, C::Q_BYTES);
            for (int c = 0; c < D / 64; ++c)
                tma_load_2d(s_base + C::OFF_Q + c * kRows * 128, &P.tm_q, c * 64, (int)row0, BAR_QF);
            int nk = 0;
            for (int j = 0; j < cnt; ++j, nk = j) {
                const int st = j % C::STAGES_K;
                if (j >= C::STAGES_K && !mbar_wait(BAR_KE(st), (uint32_t)(j / C::STAGES_K - 1) & 1, ctl)) break;
                const int krow = (int)(base_row + (long long)VSA_ENTRY_KV(__ldg(entries + j)) * BK);
                mbar_expect_tx(BAR_KF(st), C::KV_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + C::OFF_K + st * C::KV_BYTES + c * BK * 128, &P.tm_k, c * 64, krow,
                                BAR_KF(st));
            }
            issued[0] = nk;
        } else if (lane == 1 && cnt > 0) {
            int nv = 0;
            for (int j = 0; j < cnt; ++j, nv = j) {
                const int st = j % C::STAGES_V;
                if (j >= C::STAGES_V && !mbar_wait(BAR_VE(st), (uint32_t)(j / C::STAGES_V - 1) & 1, ctl)) break;
                const int vrow = (int)(base_row + (long long)VSA_ENTRY_KV(__ldg(entries + j)) * BK);
                mbar_expect_tx(BAR_VF(st), C::KV_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + C::OFF_V + st * C::KV_BYTES + c * BK * 128, &P.tm_v, c * 64, vrow,
                                BAR_VF(st));
            }
            issued[1] = nv;
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        // Descriptors are built once; per MMA only a compile-time offset is
        // added (the start-address field sits in the low bits and never carries).
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
        const uint32_t leader = elect_one();
        if (cnt > 0 && mbar_wait_warp(C::Q_TMEM ? BAR_QT : BAR_QF, 0, ctl)) {
            tc_fence_after();
            const uint64_t qdesc = smem_desc(s_base + C::OFF_Q, 16, 1024);
            const uint64_t kdesc0 = smem_desc(s_base + C::OFF_K, 16, 1024);
            const uint64_t vdesc0 = smem_desc(s_base + C::OFF_V, BK * 128, 1024);
            constexpr uint64_t kStageStep = (uint64_t)(C::KV_BYTES >> 4);
            // S_j = Q K_j^T into S_{j mod 2}; K_j's stage is released when it completes
            auto issue_qk = [&](int j, bool waited) -> bool {
                const int st = j % C::STAGES_K;
                if (!waited && !mbar_wait_warp(BAR_KF(st), (uint32_t)(j / C::STAGES_K) & 1, ctl)) return false;
                tc_fence_after();
                const uint32_t dS = tmem + ((j & 1) ? C::COL_S1 : C::COL_S0);
                const uint64_t kd = kdesc0 + (uint64_t)st * kStageStep;
                if constexpr (C::Q_TMEM) {
                    // A = Q from TMEM: 16 elements of D per step are 8 columns
                    mma_ts_lead<0>(dS, tmem + C::COL_Q, kd, C::IDESC_QK, leader);
#pragma unroll
                    for (int kk = 1; kk < D / 16; ++kk)
                        mma_ts_lead<1>(dS, tmem + C::COL_Q + kk * 8,
                                       kd + (uint64_t)((((kk >> 2) * (BK * 128)) + (kk & 3) * 32) >> 4),
                                       C::IDESC_QK, leader);
                } else {
                    mma_ss_lead<0>(dS, qdesc, kd, C::IDESC_QK, leader);
#pragma unroll
                    for (int kk = 1; kk < D / 16; ++kk)
                        mma_ss_lead<1>(dS, qdesc + (uint64_t)((((kk >> 2) * (kRows * 128)) + (kk & 3) * 32) >> 4),
                                       kd + (uint64_t)((((kk >> 2) * (BK * 128)) + (kk & 3) * 32) >> 4),
                                       C::IDESC_QK, leader);
                }
                tc_commit_lead(BAR_SF(j & 1), leader);
                tc_commit_lead(BAR_KE(st), leader);
                return true;
            };
            bool go = issue_qk(0, false);
            if (go && leader) issued[2] = 1;
            go = go && (cnt < 2 || issue_qk(1, false));
            for (int j = 0; go && j < cnt; ++j) {
                const int x = j & 1, vs = j % C::STAGES_V;
                // V_j and K_{j+2} have usually landed long before P_j: wait for
                // them first, so only the MMAs follow P_j's arrival
                if (!mbar_wait_warp(BAR_VF(vs), (uint32_t)(j / C::STAGES_V) & 1, ctl)) break;
                if (j + 2 < cnt &&
                    !mbar_wait_warp(BAR_KF((j + 2) % C::STAGES_K), (uint32_t)((j + 2) / C::STAGES_K) & 1, ctl))
                    break;
                if (!mbar_wait_warp(BAR_PF(x), (uint32_t)(j >> 1) & 1, ctl)) break;
                tc_fence_after();
                // O_x (+)= P_j V_j, P_j in the first BK/2 columns of S_x
                const uint32_t dO = tmem + (x ? C::COL_O1 : C::COL_O0);
                const uint32_t aP = tmem + (x ? C::COL_S1 : C::COL_S0);
                const uint64_t vd = vdesc0 + (uint64_t)vs * kStageStep;
                if (j < 2) mma_ts_lead<0>(dO, aP, vd, C::IDESC_PV, leader);
                else mma_ts_lead<1>(dO, aP, vd, C::IDESC_PV, leader);
#pragma unroll
                for (int kk = 1; kk < BK / 16; ++kk)
                    mma_ts_lead<1>(dO, aP + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV, leader);
                tc_commit_lead(BAR_PV(x), leader);
                tc_commit_lead(BAR_VE(vs), leader);
                // S_{j+2} reuses S_x: queued behind PV_j, so P_j is read first
                if (j + 2 < cnt) go = issue_qk(j + 2, true);
            }
        }
    } else if (warp >= kMaskWarp0) {
        // ---------------- mask workers (warps 10, 11) ----------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
        const int t = threadIdx.x - kMaskWarp0 * 32;      // rows t and t + 64
        const vsa_mask_spec m0 = P.specs[head];
        // a rounded head keeps whole tiles: only its padding is masked
        vsa_mask_spec m = m0;
        if (m0.tile_round) {
            m.kind = VSA_MASK_FULL;
            m.sink = 0;
        }
        const vsa_row_ctx q0 = vsa_row_init(d, m, (long long)e * kRows + t);
        const vsa_row_ctx q1 = vsa_row_init(d, m, (long long)e * kRows + t + 64);
        if (m.kind == VSA_MASK_STRIPE) {
            const uint32_t* src = P.sbits + (size_t)head * d.sbits_words;
            for (int i = t; i < P.tab_words_s; i += 64) stab[i] = src[i];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * (kSoftmaxWarps + 2)) : "memory");
        // single-box tiles and frame-0-first heads are evaluated by the softmax threads
        if (d.box_nh == 0 && m.layout != VSA_LAYOUT_FRAME0_FIRST) switch (m.kind) {
        case VSA_MASK_FULL:
            mask_worker_loop<VSA_MASK_FULL, BK>(m, d, q0, q1, stab, ttab, P.seg, entries, cnt, t, lane, maskbuf,
                                                BAR_MF(0), BAR_ME(0), ctl);
            break;
        case VSA_MASK_SVG_SPATIAL:
            mask_worker_loop<VSA_MASK_SVG_SPATIAL, BK>(m, d, q0, q1, stab, ttab, P.seg, entries, cnt, t, lane,
                                                       maskbuf, BAR_MF(0), BAR_ME(0), ctl);
            break;
        case VSA_MASK_SVG_TEMPORAL:
            mask_worker_loop<VSA_MASK_SVG_TEMPORAL, BK>(m, d, q0, q1, stab, ttab, P.seg, entries, cnt, t, lane,
                                                        maskbuf, BAR_MF(0), BAR_ME(0), ctl);
            break;
        case VSA_MASK_STA:
            mask_worker_loop<VSA_MASK_STA, BK>(m, d, q0, q1, stab, ttab, P.seg, entries, cnt, t, lane, maskbuf,
                                               BAR_MF(0), BAR_ME(0), ctl);
            break;
        default:
            mask_worker_loop<VSA_MASK_STRIPE, BK>(m, d, q0, q1, stab, ttab, P.seg, entries, cnt, t, lane,
                                                  maskbuf, BAR_MF(0), BAR_ME(0), ctl);
            break;
        }
    } else {
        // ---------------- softmax warpgroups (warps 0..3: X = 0, 4..7: X = 1) ----------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
        const int X = warp >> 2;                          // list entries j with j mod 2 = X
        const int row = threadIdx.x & (kRows - 1);        // TMEM lane
        const int half = row >> 6;                        // 64-row q tile of the row (warp-uniform)
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + (X ? C::COL_S1 : C::COL_S0);
        const uint32_t tO = tmem + lane_off + (X ? C::COL_O1 : C::COL_O0);
        const vsa_mask_spec m = P.specs[head];
        if (m.kind == VSA_MASK_STRIPE)
            for (int i = threadIdx.x; i < P.tab_words_t; i += 32 * kSoftmaxWarps)
                ttab[i] = vsa_stripe_tword(m, d.T, i);
        if (X == 0) rowctx[row] = vsa_row_init(d, m, (long long)e * kRows + row);
        asm volatile("bar.sync 1, %0;" ::"n"(32 * (kSoftmaxWarps + 2)) : "memory");

        const bool f0 = m.layout == VSA_LAYOUT_FRAME0_FIRST;
        // a rounded head keeps whole tiles: its boundary tiles only mask padding
        vsa_mask_spec mb = m;
        if (m.tile_round) {
            mb.kind = VSA_MASK_FULL;
            mb.sink = 0;
        }
        const bool box = d.box_nh > 0 && !f0;             // boundary bits computed here, not by mask workers
        float m_run = -INFINITY;  // running max of scale*log2(e)*s over this warpgroup's tiles
        float l_run = 0.0f;
        const float sl = P.scale_log2;
        const unsigned long long sl2 = f2_pack(sl, sl);
        bool ok = true;
        if constexpr (C::Q_TMEM) {
            // warpgroup 0 moves Q into TMEM: thread r reads row r from the
            // 128-byte-swizzled shared copy (chunk u of a 64-column block at
            // u ^ (r mod 8)) and stores it as bf16 pairs, row r = lane r
            if (X == 0 && cnt > 0) {
                ok = mbar_wait_warp(BAR_QF, 0, ctl);
                if (ok) {
#pragma unroll
                    for (int c = 0; c < D / 64; ++c) {
                        uint32_t qv[32];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const uint4 v4 = *reinterpret_cast<const uint4*>(
                                smem + C::OFF_Q + c * (kRows * 128) + row * 128 + ((u ^ (row & 7)) << 4));
                            qv[4 * u] = v4.x;
                            qv[4 * u + 1] = v4.y;
                            qv[4 * u + 2] = v4.z;
                            qv[4 * u + 3] = v4.w;
                        }
                        tmem_st32(tmem + lane_off + C::COL_Q + c * 32, qv);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(BAR_QT);
                }
            }
        }
        const vsa_row_ctx qrow = rowctx[row];             // the row's mask context, kept in registers
        int ent_next = cnt > 0 ? __ldg(entries) : 0;
        int kb = 0;                                       // boundary tiles of the list so far
        uint32_t cw[BK / 32];                             // keep bits of the last single-box boundary tile
        int ck_x = -1, ck_y = -1;                         // and their key
        for (int j = 0; j < cnt && ok; ++j) {
            const int ent = ent_next;
            if (j + 1 < cnt) ent_next = __ldg(entries + j + 1);
            const bool bnd = VSA_ENTRY_CLS(ent, 0) == VSA_TILE_BOUNDARY || VSA_ENTRY_CLS(ent, 1) == VSA_TILE_BOUNDARY;
            if ((j & 1) != X) {                           // the other warpgroup's tile
                kb += bnd ? 1 : 0;
                continue;
            }
            const int cls = VSA_ENTRY_CLS(ent, half);
            // keep bits of a single-box boundary tile, computed while S_j is in flight
            uint32_t mw[BK / 32];
            if (bnd && box) {
                const int kv = VSA_ENTRY_KV(ent);
                cached_box_bits<BK>(mb, d, qrow, stab, ttab, __ldg(P.seg + (size_t)kv * d.nseg),
                                    (long long)kv * BK < d.Npad, cw, ck_x, ck_y, mw);
            }
            if (bnd && f0) f0_row_bits<BK>(mb, d, qrow, VSA_ENTRY_KV(ent), mw);
            if (!mbar_wait_warp(BAR_SF(X), (uint32_t)(j >> 1) & 1, ctl)) { ok = false; break; }
            tc_fence_after();
            float s[BK];
            {
                uint32_t sr[BK];
#pragma unroll
                for (int c = 0; c < BK / 32; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < BK; ++c) {
                    reg_fence(sr[c]);
                    s[c] = __uint_as_float(sr[c]);
                }
            }

            if (bnd) {
                if (!box && !f0) {
                    // keep bits from the mask workers; the slot is released after reading
                    const int slot = kb % kMaskSlots;
                    if (!mbar_wait_warp(BAR_MF(slot), (uint32_t)(kb / kMaskSlots) & 1, ctl)) { ok = false; break; }
                    const uint32_t* src = maskbuf + slot * C::MASK_SLOT_WORDS + row;
#pragma unroll
                    for (int wi = 0; wi < BK / 32; ++wi) mw[wi] = src[wi * kRows];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(BAR_ME(slot));
                    ++kb;
                }
                if (cls == VSA_TILE_BOUNDARY) {
#pragma unroll
                    for (int wi = 0; wi < BK / 32; ++wi)
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (!((mw[wi] >> c) & 1u)) s[wi * 32 + c] = -INFINITY;
                }
            }

            bool need_o = false;
            float alpha = 1.0f;
            if (cls == VSA_TILE_EMPTY) {
                uint32_t zero[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) zero[c] = 0u;
#pragma unroll
                for (int q = 0; q < BK / 32; ++q) tmem_st16(tS + 16 * q, zero);
            } else {
                // row max: independent chains of 3-input max over 32 columns each
                float mc[BK / 32];
#pragma unroll
                for (int g = 0; g < BK / 32; ++g) {
                    float a = s[g * 32];
#pragma unroll
                    for (int c = 1; c < 31; c += 2) a = max3(a, s[g * 32 + c], s[g * 32 + c + 1]);
                    mc[g] = fmaxf(a, s[g * 32 + 31]);
                }
                float mx = mc[0];
#pragma unroll
                for (int g = 1; g < BK / 32; ++g) mx = fmaxf(mx, mc[g]);
                const float mxs = mx * sl;
                if (mx != -INFINITY) {
                    if (m_run == -INFINITY) {
                        m_run = mxs;  // nothing accumulated for this row yet: O_X row is 0
                    } else if (mxs > m_run + kRescaleThreshold) {
                        alpha = ex2(m_run - mxs);
                        l_run *= alpha;
                        m_run = mxs;
                        need_o = true;
                    }
                }
                const float mneg = (m_run == -INFINITY) ? 0.0f : -m_run;
                const unsigned long long mneg2 = f2_pack(mneg, mneg);
                unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int q = 0; q < BK / 32; ++q) {
                    uint32_t pq[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int c = 32 * q + 2 * i;
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sl2, mneg2), x0, x1);
                        const float p0 = ex2(x0);
                        const float p1 = ex2(x1);
                        acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
                        pq[i] = pack_bf16(p0, p1);
                    }
                    tmem_st16(tS + 16 * q, pq);
                }
                float a0, a1, a2, a3, a4, a5, a6, a7;
                f2_unpack(acc[0], a0, a1);
                f2_unpack(acc[1], a2, a3);
                f2_unpack(acc[2], a4, a5);
                f2_unpack(acc[3], a6, a7);
                l_run += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
            }
            // S_j complete implies PV_{j-2}, the last MMA into O_X, is complete
            // (one thread's MMAs run in order), so O_X can be rescaled here
            if (__any_sync(0xFFFFFFFFu, need_o)) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(tO + c * 32, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        reg_fence(ov[i]);
                        ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    }
                    tmem_st32(tO + c * 32, ov);
                }
            }
            // P_j went over the first BK/2 columns of S_X 32 keys at a time, each
            // chunk stored as soon as its exponentials are done (fewer live
            // registers than holding all of P_j); one wait covers them all
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR_PF(X));
        }

        // ---------------- epilogue: merge the two warpgroups' partial softmaxes ----------------
        // Warpgroup 0 had (cnt + 1) / 2 tiles, warpgroup 1 cnt / 2.  Each waits
        // for the last PV into its own accumulator (its barrier is at most one
        // phase behind, so the parity wait is exact), then the named barrier
        // hands both results to both warpgroups.
        const int n0 = (cnt + 1) >> 1, n1 = cnt >> 1;
        const int nx = X ? n1 : n0;
        bool have_o = ok;
        if (have_o && nx > 0) have_o = mbar_wait_warp(BAR_PV(X), (uint32_t)(nx - 1) & 1, ctl);
        stat[X * kRows + row] = make_float2(m_run, l_run);
        tc_fence_before();
        asm volatile("bar.sync 2, %0;" ::"n"(32 * kSoftmaxWarps) : "memory");
        tc_fence_after();
        have_o = have_o && !*abort_flag;
        const float2 st0 = stat[row], st1 = stat[kRows + row];
        const float mm = fmaxf(st0.x, st1.x);
        const float w0 = st0.y > 0.0f ? ex2(st0.x - mm) : 0.0f;
        const float w1 = st1.y > 0.0f ? ex2(st1.x - mm) : 0.0f;
        const float l_row = w0 * st0.y + w1 * st1.y;
        const float inv = l_row > 0.0f ? 1.0f / l_row : 0.0f;
        const long long orow = row0 + row;
        // warpgroup X writes columns [X D/2, (X+1) D/2) of the output row
        uint4* optr = reinterpret_cast<uint4*>(P.o + orow * D + X * (D / 2));
        if (have_o && cnt > 0) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                const int col = X * (D / 2) + c * 32;
                uint32_t o0[32], o1[32];
                tmem_ld32(tmem + lane_off + C::COL_O0 + col, o0);
                if (n1 > 0) tmem_ld32(tmem + lane_off + C::COL_O1 + col, o1);
                tmem_ld_wait();
                uint32_t pkd[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float v[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        reg_fence(o0[i + h]);
                        const float x0 = w0 > 0.0f ? __uint_as_float(o0[i + h]) * w0 : 0.0f;
                        float x1 = 0.0f;
                        if (n1 > 0) {
                            reg_fence(o1[i + h]);
                            x1 = w1 > 0.0f ? __uint_as_float(o1[i + h]) * w1 : 0.0f;
                        }
                        v[h] = (x0 + x1) * inv;
                    }
                    pkd[i >> 1] = pack_bf16(v[0], v[1]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    optr[c * 4 + i] = make_uint4(pkd[4 * i], pkd[4 * i + 1], pkd[4 * i + 2], pkd[4 * i + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < D / 16; ++i) optr[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (X == 0) P.lse[orow] = (l_row > 0.0f) ? (mm + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // After a watchdog abort some copies or MMAs may still be in flight:
        // each role waits (bounded) for its own before TMEM is freed.  A
        // normal run consumed all of them already.
        if (warp == kProducerWarp && lane == 0 && cnt > 0) {
            const int nk = issued[0];
            mbar_drain(BAR_QF, 0, kDrainCycles);
            for (int j = nk > C::STAGES_K ? nk - C::STAGES_K : 0; j < nk; ++j)
                mbar_drain(BAR_KF(j % C::STAGES_K), (uint32_t)(j / C::STAGES_K) & 1, kDrainCycles);
        }
        if (warp == kProducerWarp && lane == 1) {
            const int nv = issued[1];
            for (int j = nv > C::STAGES_V ? nv - C::STAGES_V : 0; j < nv; ++j)
                mbar_drain(BAR_VF(j % C::STAGES_V), (uint32_t)(j / C::STAGES_V) & 1, kDrainCycles);
        }
        if (warp == kMmaWarp && issued[2]) {
            const uint32_t leader = elect_one();
            tc_commit_lead(BAR_DR, leader);
            if (leader) mbar_drain(BAR_DR, 0, kDrainCycles);
            __syncwarp();
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
    }
}

// ---- paired blocks: two 128-row sub-tiles per CTA ---------------------------
//
// Two adjacent 128-row execution blocks whose kv-tile lists hold the same kv
// tiles (both halves of a 256-row q tile always do; 128-row q tiles do where
// the mask repeats, e.g. inside a frame of an SVG spatial head) run in one
// CTA, which loads every K and V tile once for both ("Sparse VideoGen ... on
// TPU", "tile-size tuning can introduce trade-offs": how rows are grouped
// decides the work per loaded tile).  Softmax warpgroup X owns sub-tile X
// (rows [128 X, 128 X + 128)) with its own score buffer S_X and accumulator
// O_X, takes its classes from its own block's list and runs every tile; the
// two sub-tiles share the K/V ring, so the shared-memory traffic per step
// drops by a fifth (Q 32 KB + K 32 KB + V 32 KB read, plus half the 64 KB of
// fills, against the full fills of a single block).
// Warps: 0..7 softmax (warpgroup X = warp / 4), 8 TMA producer (lane 0 Q and
// K, lane 1 V), 9 MMA issuer, 10..11 idle (they keep the register split of
// the single-block body).  MMA order per tile j: PV_0(j), QK_0(j+1), PV_1(j),
// QK_1(j+1) after QK_0(0), QK_1(0); S_X of tile j+1 is queued behind PV_X(j),
// so when S_X(j) is complete, O_X holds the sum up to tile j-1.  Boundary
// bits: single-box tiles from the tile's first run descriptor, frame-0-first
// heads by runs of frames, other tiles run by run, all in the softmax threads.
// TMEM columns: S_0 [0,BK), S_1 [BK,2BK), O_0 [2BK,2BK+D), O_1 [2BK+D,2BK+2D).
template <int D, int BK>
struct PairCfg {
    static constexpr int KV_BYTES = BK * D * 2;
    static constexpr int QH_BYTES = kRows * D * 2;          // one 128-row sub-tile
    static constexpr int REGS_SOFTMAX = BK == 128 ? 208 : 176;
    static constexpr int REGS_OTHER = 3 * kRegsLaunch - 2 * REGS_SOFTMAX;
    static constexpr int RING_BYTES = 192 * 1024 - 2 * QH_BYTES;
    static constexpr int STAGES_V = (RING_BYTES / KV_BYTES) / 2 > 4 ? 4 : (RING_BYTES / KV_BYTES) / 2;
    static constexpr int STAGES_K = (RING_BYTES / KV_BYTES - STAGES_V) > 4 ? 4 : (RING_BYTES / KV_BYTES - STAGES_V);
    static_assert(STAGES_V >= 2 && STAGES_K >= 2, "shared-memory ring");
    static constexpr int COL_S0 = 0;
    static constexpr int COL_S1 = BK;
    static constexpr int COL_O0 = 2 * BK;
    static constexpr int COL_O1 = 2 * BK + D;
    static constexpr int COLS_USED = 2 * BK + 2 * D;
    static constexpr int TMEM_COLS = COLS_USED <= 256 ? 256 : 512;
    static_assert(COLS_USED <= 512, "TMEM budget");
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * QH_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES_K * KV_BYTES;
    static constexpr int OFF_ROWCTX = OFF_V + STAGES_V * KV_BYTES;
    static constexpr int OFF_BAR = OFF_ROWCTX + 2 * kRows * (int)sizeof(vsa_row_ctx);
    // barriers: k_full[SK], k_empty[SK], v_full[SV], v_empty[SV], q_full,
    //           s_full[2], p_full[2], pv_done[2], mma_drain
    static constexpr int NBAR = 2 * STAGES_K + 2 * STAGES_V + 8;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_TAB = (OFF_MISC + 20 + 15) / 16 * 16;
    static constexpr uint32_t IDESC_QK = Cfg<D, BK>::IDESC_QK;
    static constexpr uint32_t IDESC_PV = Cfg<D, BK>::IDESC_PV;
};

// Keep bits of query row q for a kv tile made of several boxes (a tile longer
// than a unit): run by run from the tile's run descriptors (bw keys sharing t
// and h each; bw divides 32, so no run straddles a 32-key word).
template <int BK>
__device__ __forceinline__ void multi_row_bits(const vsa_mask_spec& m, const vsa_dims& d, const vsa_row_ctx& q,
                                               const uint32_t* stab, const uint32_t* ttab,
                                               const int2* __restrict__ seg, int kv, uint32_t (&words)[BK / 32])
{
#pragma unroll
    for (int wi = 0; wi < BK / 32; ++wi) words[wi] = 0u;
    const int2* sg = seg + (size_t)kv * d.nseg;
    uint32_t acc = 0;
    for (int r = 0; r < d.nseg; ++r) {
        const int2 v = __ldg(sg + r);
        const uint32_t b = vsa_run_bits(m, d, q, stab, ttab, v.x & 0xFFFF, v.x >> 16, v.y & 0xFFFF, v.y >> 16);
        const int col = r * d.bw;
        acc |= b << (col & 31);
        if (((col + d.bw) & 31) == 0) {
#pragma unroll
            for (int wi = 0; wi < BK / 32; ++wi) words[wi] = (col >> 5) == wi ? acc : words[wi];
            acc = 0;
        }
    }
}

// The execution blocks ea and eb of (batch, head) hb, whose lists hold the
// same kv tiles in the same order, as one CTA of two 128-row sub-tiles.
template <int D, int BK>
__device__ __forceinline__ void attn_pair(const AttnParams& P, int ea, int eb, int hb)
{
    using C = PairCfg<D, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

    const vsa_dims& d = P.d;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int head = hb % d.heads;
    const long long base_row = (long long)hb * d.Nslots;
    const long long rowa = base_row + (long long)ea * kRows, rowb = base_row + (long long)eb * kRows;
    // the two blocks' lists name the same kv tiles: the copies follow the
    // first, each sub-tile takes its classes from its own
    const int list_idx = head * d.nE + ea;
    const int cnt = P.list_cnt[list_idx];
    const int32_t* entries = P.list + (size_t)list_idx * d.nK;
    const int32_t* entries_b = P.list + ((size_t)head * d.nE + eb) * d.nK;

    const uint32_t s_base = smem_addr(smem);
    const uint32_t bar0 = s_base + C::OFF_BAR;
    auto BAR_KF = [&](int s) { return bar0 + 8u * s; };
    auto BAR_KE = [&](int s) { return bar0 + 8u * (C::STAGES_K + s); };
    auto BAR_VF = [&](int s) { return bar0 + 8u * (2 * C::STAGES_K + s); };
    auto BAR_VE = [&](int s) { return bar0 + 8u * (2 * C::STAGES_K + C::STAGES_V + s); };
    constexpr int B1 = 2 * C::STAGES_K + 2 * C::STAGES_V;
    const uint32_t BAR_QF = bar0 + 8u * B1;
    auto BAR_SF = [&](int x) { return bar0 + 8u * (B1 + 1 + x); };
    auto BAR_PF = [&](int x) { return bar0 + 8u * (B1 + 3 + x); };
    auto BAR_PV = [&](int x) { return bar0 + 8u * (B1 + 5 + x); };
    const uint32_t BAR_DR = bar0 + 8u * (B1 + 7);
    vsa_row_ctx* rowctx = (vsa_row_ctx*)(smem + C::OFF_ROWCTX);
    uint32_t* tmem_slot = (uint32_t*)(smem + C::OFF_MISC);
    volatile int* abort_flag = (volatile int*)(smem + C::OFF_MISC + 4);
    volatile int* issued = (volatile int*)(smem + C::OFF_MISC + 8);
    uint32_t* stab = (uint32_t*)(smem + C::OFF_TAB);
    uint32_t* ttab = stab + P.tab_words_s;
    const Ctl ctl{abort_flag, P.status};

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES_K; ++s) {
            mbar_init(BAR_KF(s), 1);
            mbar_init(BAR_KE(s), 1);
        }
        for (int s = 0; s < C::STAGES_V; ++s) {
            mbar_init(BAR_VF(s), 1);
            mbar_init(BAR_VE(s), 1);
        }
        mbar_init(BAR_QF, 1);
        mbar_init(BAR_DR, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR_SF(x), 1);
            mbar_init(BAR_PF(x), 4);                    // the four warps of warpgroup x
            mbar_init(BAR_PV(x), 1);
        }
        *abort_flag = 0;
        issued[0] = issued[1] = issued[2] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProducerWarp) {
        // ---------------- TMA producer: lane 0 Q and K, lane 1 V ----------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
        if (lane == 0 && cnt > 0) {
            mbar_expect_tx(BAR_QF, 2 * C::QH_BYTES);
            for (int x = 0; x < 2; ++x)
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + C::OFF_Q + x * C::QH_BYTES + c * kRows * 128, &P.tm_q, c * 64,
                                (int)(x ? rowb : rowa), BAR_QF);
            int nk = 0;
            for (int j = 0; j < cnt; ++j, nk = j) {
                const int st = j % C::STAGES_K;
                if (j >= C::STAGES_K && !mbar_wait(BAR_KE(st), (uint32_t)(j / C::STAGES_K - 1) & 1, ctl)) break;
                const int krow = (int)(base_row + (long long)VSA_ENTRY_KV(__ldg(entries + j)) * BK);
                mbar_expect_tx(BAR_KF(st), C::KV_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + C::OFF_K + st * C::KV_BYTES + c * BK * 128, &P.tm_k, c * 64, krow,
                                BAR_KF(st));
            }
            issued[0] = nk;
        } else if (lane == 1 && cnt > 0) {
            int nv = 0;
            for (int j = 0; j < cnt; ++j, nv = j) {
                const int st = j % C::STAGES_V;
                if (j >= C::STAGES_V && !mbar_wait(BAR_VE(st), (uint32_t)(j / C::STAGES_V - 1) & 1, ctl)) break;
                const int vrow = (int)(base_row + (long long)VSA_ENTRY_KV(__ldg(entries + j)) * BK);
                mbar_expect_tx(BAR_VF(st), C::KV_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + C::OFF_V + st * C::KV_BYTES + c * BK * 128, &P.tm_v, c * 64, vrow,
                                BAR_VF(st));
            }
            issued[1] = nv;
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
        const uint32_t leader = elect_one();
        if (cnt > 0 && mbar_wait_warp(BAR_QF, 0, ctl)) {
            tc_fence_after();
            const uint64_t qdesc0 = smem_desc(s_base + C::OFF_Q, 16, 1024);
            const uint64_t kdesc0 = smem_desc(s_base + C::OFF_K, 16, 1024);
            const uint64_t vdesc0 = smem_desc(s_base + C::OFF_V, BK * 128, 1024);
            constexpr uint64_t kStageStep = (uint64_t)(C::KV_BYTES >> 4);
            constexpr uint64_t kQStep = (uint64_t)(C::QH_BYTES >> 4);
            // S_X(j) = Q_X K_j^T into S_X; K_j's stage is released after sub-tile 1's QK
            auto issue_qk = [&](int j, int x) {
                const int st = j % C::STAGES_K;
                const uint32_t dS = tmem + (x ? C::COL_S1 : C::COL_S0);
                const uint64_t kd = kdesc0 + (uint64_t)st * kStageStep;
                const uint64_t qd = qdesc0 + (uint64_t)x * kQStep;
                mma_ss_lead<0>(dS, qd, kd, C::IDESC_QK, leader);
#pragma unroll
                for (int kk = 1; kk < D / 16; ++kk)
                    mma_ss_lead<1>(dS, qd + (uint64_t)((((kk >> 2) * (kRows * 128)) + (kk & 3) * 32) >> 4),
                                   kd + (uint64_t)((((kk >> 2) * (BK * 128)) + (kk & 3) * 32) >> 4), C::IDESC_QK,
                                   leader);
                tc_commit_lead(BAR_SF(x), leader);
                if (x == 1) tc_commit_lead(BAR_KE(st), leader);
            };
            bool go = mbar_wait_warp(BAR_KF(0), 0, ctl);
            if (go) {
                tc_fence_after();
                issue_qk(0, 0);
                issue_qk(0, 1);
                if (leader) issued[2] = 1;
            }
            for (int j = 0; go && j < cnt; ++j) {
                const int vs = j % C::STAGES_V;
                if (!mbar_wait_warp(BAR_VF(vs), (uint32_t)(j / C::STAGES_V) & 1, ctl)) break;
                if (j + 1 < cnt &&
                    !mbar_wait_warp(BAR_KF((j + 1) % C::STAGES_K), (uint32_t)((j + 1) / C::STAGES_K) & 1, ctl))
                    break;
                const uint64_t vd = vdesc0 + (uint64_t)vs * kStageStep;
                for (int x = 0; x < 2; ++x) {
                    if (!mbar_wait_warp(BAR_PF(x), (uint32_t)j & 1, ctl)) {
                        go = false;
                        break;
                    }
                    tc_fence_after();
                    // O_X (+)= P_X(j) V_j, P in the first BK/2 columns of S_X
                    const uint32_t dO = tmem + (x ? C::COL_O1 : C::COL_O0);
                    const uint32_t aP = tmem + (x ? C::COL_S1 : C::COL_S0);
                    if (j == 0) mma_ts_lead<0>(dO, aP, vd, C::IDESC_PV, leader);
                    else mma_ts_lead<1>(dO, aP, vd, C::IDESC_PV, leader);
#pragma unroll
                    for (int kk = 1; kk < BK / 16; ++kk)
                        mma_ts_lead<1>(dO, aP + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV, leader);
                    tc_commit_lead(BAR_PV(x), leader);
                    if (x == 1) tc_commit_lead(BAR_VE(vs), leader);
                    // S_X(j+1) reuses S_X: queued behind PV_X(j), so P_X(j) is read first
                    if (j + 1 < cnt) issue_qk(j + 1, x);
                }
            }
        }
    } else if (warp >= kMaskWarp0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
    } else {
        // ---------------- softmax: warpgroup X owns sub-tile X ----------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
        const int X = warp >> 2;
        const int r = threadIdx.x & (kRows - 1);          // TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + (X ? C::COL_S1 : C::COL_S0);
        const uint32_t tO = tmem + lane_off + (X ? C::COL_O1 : C::COL_O0);
        const vsa_mask_spec m = P.specs[head];
        vsa_mask_spec mb = m;                             // a rounded head only masks padding
        if (m.tile_round) {
            mb.kind = VSA_MASK_FULL;
            mb.sink = 0;
        }
        if (mb.kind == VSA_MASK_STRIPE) {
            const uint32_t* src = P.sbits + (size_t)head * d.sbits_words;
            for (int i = threadIdx.x; i < P.tab_words_s; i += 32 * kSoftmaxWarps) stab[i] = src[i];
            for (int i = threadIdx.x; i < P.tab_words_t; i += 32 * kSoftmaxWarps)
                ttab[i] = vsa_stripe_tword(m, d.T, i);
        }
        rowctx[X * kRows + r] = vsa_row_init(d, mb, (long long)(X ? eb : ea) * kRows + r);
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kSoftmaxWarps) : "memory");
        const bool f0 = m.layout == VSA_LAYOUT_FRAME0_FIRST;
        const bool box = d.box_nh > 0 && !f0;
        float m_run = -INFINITY;  // running max of scale*log2(e)*s (log2 units)
        float l_run = 0.0f;
        const float sl = P.scale_log2;
        const unsigned long long sl2 = f2_pack(sl, sl);
        bool ok = true;
        const int32_t* own = X ? entries_b : entries;   // sub-tile X's own list
        const vsa_row_ctx qrow = rowctx[X * kRows + r];   // the row's mask context, kept in registers
        int ent_next = cnt > 0 ? __ldg(own) : 0;
        // first run descriptor of the next tile, loaded a tile ahead
        int2 v_next = (box && cnt > 0) ? __ldg(P.seg + (size_t)VSA_ENTRY_KV(ent_next) * d.nseg) : make_int2(0, 0);
        uint32_t cw[BK / 32];                             // keep bits of the last single-box boundary tile
        int ck_x = -1, ck_y = -1;                         // and their key (no descriptor has x = -1)
        for (int j = 0; j < cnt && ok; ++j) {
            const int ent = ent_next;
            const int2 v_cur = v_next;
            if (j + 1 < cnt) ent_next = __ldg(own + j + 1);
            // one class for the 128 rows of the sub-tile (q tiles of 128 or 256 rows)
            const int cls = VSA_ENTRY_CLS(ent, 0);
            const int kv = VSA_ENTRY_KV(ent);
            uint32_t mw[BK / 32];
            if (cls == VSA_TILE_BOUNDARY) {
                if (f0) {
                    f0_row_bits<BK>(mb, d, qrow, kv, mw);
                } else if (box) {
                    cached_box_bits<BK>(mb, d, qrow, stab, ttab, v_cur, (long long)kv * BK < d.Npad, cw, ck_x, ck_y,
                                        mw);
                } else {
                    multi_row_bits<BK>(mb, d, qrow, stab, ttab, P.seg, kv, mw);
                }
            }
            if (!mbar_wait_warp(BAR_SF(X), (uint32_t)j & 1, ctl)) { ok = false; break; }
            tc_fence_after();
            float s[BK];
            {
                uint32_t sr[BK];
#pragma unroll
                for (int c = 0; c < BK / 32; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < BK; ++c) {
                    reg_fence(sr[c]);
                    s[c] = __uint_as_float(sr[c]);
                }
            }
            if (cls == VSA_TILE_BOUNDARY) {
#pragma unroll
                for (int wi = 0; wi < BK / 32; ++wi)
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (!((mw[wi] >> c) & 1u)) s[wi * 32 + c] = -INFINITY;
            }
            bool need_o = false;
            float alpha = 1.0f;
            {
                float mc[BK / 32];
#pragma unroll
                for (int g = 0; g < BK / 32; ++g) {
                    float a = s[g * 32];
#pragma unroll
                    for (int c = 1; c < 31; c += 2) a = max3(a, s[g * 32 + c], s[g * 32 + c + 1]);
                    mc[g] = fmaxf(a, s[g * 32 + 31]);
                }
                float mx = mc[0];
#pragma unroll
                for (int g = 1; g < BK / 32; ++g) mx = fmaxf(mx, mc[g]);
                const float mxs = mx * sl;
                if (mx != -INFINITY) {
                    if (m_run == -INFINITY) {
                        m_run = mxs;      // nothing accumulated for this row yet: its O row is 0
                    } else if (mxs > m_run + kRescaleThreshold) {
                        alpha = ex2(m_run - mxs);
                        l_run *= alpha;
                        m_run = mxs;
                        need_o = true;
                    }
                }
                const float mneg = (m_run == -INFINITY) ? 0.0f : -m_run;
                const unsigned long long mneg2 = f2_pack(mneg, mneg);
                unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int q = 0; q < BK / 32; ++q) {
                    uint32_t pq[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int c = 32 * q + 2 * i;
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sl2, mneg2), x0, x1);
                        const float p0 = ex2(x0);
                        const float p1 = ex2(x1);
                        acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
                        pq[i] = pack_bf16(p0, p1);
                    }
                    tmem_st16(tS + 16 * q, pq);
                }
                float a0, a1, a2, a3, a4, a5, a6, a7;
                f2_unpack(acc[0], a0, a1);
                f2_unpack(acc[1], a2, a3);
                f2_unpack(acc[2], a4, a5);
                f2_unpack(acc[3], a6, a7);
                l_run += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
            }
            // S_X(j) complete implies PV_X(j-1), the last MMA into O_X, is
            // complete (one thread's MMAs run in order), so O_X can be rescaled
            if (__any_sync(0xFFFFFFFFu, need_o)) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(tO + c * 32, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        reg_fence(ov[i]);
                        ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    }
                    tmem_st32(tO + c * 32, ov);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR_PF(X));
            if (box && j + 1 < cnt) v_next = __ldg(P.seg + (size_t)VSA_ENTRY_KV(ent_next) * d.nseg);
        }

        // ---------------- epilogue: each warpgroup writes its own 128 rows ----------------
        bool have_o = ok;
        if (have_o && cnt > 0) have_o = mbar_wait_warp(BAR_PV(X), (uint32_t)(cnt - 1) & 1, ctl);
        tc_fence_after();
        have_o = have_o && !*abort_flag;
        const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
        const long long orow = (X ? rowb : rowa) + r;
        uint4* optr = reinterpret_cast<uint4*>(P.o + orow * D);
        if (have_o && cnt > 0) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32(tO + c * 32, ov);
                tmem_ld_wait();
                uint32_t pkd[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    reg_fence(ov[i]);
                    reg_fence(ov[i + 1]);
                    pkd[i >> 1] = pack_bf16(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    optr[c * 4 + i] = make_uint4(pkd[4 * i], pkd[4 * i + 1], pkd[4 * i + 2], pkd[4 * i + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < D / 8; ++i) optr[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        P.lse[orow] = (l_run > 0.0f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == kProducerWarp && lane == 0 && cnt > 0) {
            const int nk = issued[0];
            mbar_drain(BAR_QF, 0, kDrainCycles);
            for (int j = nk > C::STAGES_K ? nk - C::STAGES_K : 0; j < nk; ++j)
                mbar_drain(BAR_KF(j % C::STAGES_K), (uint32_t)(j / C::STAGES_K) & 1, kDrainCycles);
        }
        if (warp == kProducerWarp && lane == 1) {
            const int nv = issued[1];
            for (int j = nv > C::STAGES_V ? nv - C::STAGES_V : 0; j < nv; ++j)
                mbar_drain(BAR_VF(j % C::STAGES_V), (uint32_t)(j / C::STAGES_V) & 1, kDrainCycles);
        }
        if (warp == kMmaWarp && issued[2]) {
            const uint32_t leader = elect_one();
            tc_commit_lead(BAR_DR, leader);
            if (leader) mbar_drain(BAR_DR, 0, kDrainCycles);
            __syncwarp();
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
    }
}

// One CTA per (batch, head, 128-row block); where the plan pairs two blocks,
// the leader's CTA runs both and the partner's returns at once.  CTAs walk
// the heads in the plan's order (most executed steps first, every batch of
// a head together), so the longest CTAs start first.
template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams P)
{
    const vsa_dims& d = P.d;
    const int e = blockIdx.x % d.nE;
    const int u = blockIdx.x / d.nE;                    // rank * B + b
    const int nb = (int)(gridDim.x / d.nE) / d.heads;   // batch
    const int head = P.order[u / nb];
    const int hb = (u % nb) * d.heads + head;           // b * heads + head
    const int partner = P.pair[(size_t)head * d.nE + e];
    if (partner == -1) attn_single<D, BK>(P, e, hb);
    else if (partner >= 0) attn_pair<D, BK>(P, e, partner, hb);
}

// ---- host side ----------------------------------------------------------

template <int D, int BK>
int launch_attn(AttnParams& P, int B, cudaStream_t s)
{
    using C = Cfg<D, BK>;
    using PC = PairCfg<D, BK>;
    const int smem = 1024 + (C::OFF_TAB > PC::OFF_TAB ? C::OFF_TAB : PC::OFF_TAB) +
                     4 * (P.tab_words_s + P.tab_words_t);
    if (smem > 227 * 1024) return VSA_ERR_UNSUPPORTED;
    auto kern = attn_fwd_kernel<D, BK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return VSA_ERR_CUDA;
    const long long grid = (long long)P.d.nE * P.d.heads * B;
    if (grid > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
    kern<<<(unsigned)grid, kThreads, smem, s>>>(P);
    return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace

extern "C" int vsa_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                                   vsa_plan_t plan, int B, int D, float scale, void* stream)
{
    if (!plan || B < 0 || !(scale > 0.0f) || !(scale < 1e30f)) return VSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
    if (B == 0) return VSA_OK;
    if (!q || !k || !v || !o || !lse) return VSA_ERR_INVALID_ARG;
    if (!vsa_aligned16(q) || !vsa_aligned16(k) || !vsa_aligned16(v) || !vsa_aligned16(o) ||
        !vsa_aligned16(lse))
        return VSA_ERR_ALIGNMENT;
    const vsa_dims& d = plan->d;
    const long long rows = (long long)B * d.heads * d.Nslots;
    if (rows > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;

    AttnParams P;
    memset(&P, 0, sizeof P);
    if (!vsa_make_tmap_bf16(&P.tm_q, q, rows, D, kRows) || !vsa_make_tmap_bf16(&P.tm_k, k, rows, D, d.Bk) ||
        !vsa_make_tmap_bf16(&P.tm_v, v, rows, D, d.Bk))
        return VSA_ERR_CUDA;
    P.o = (__nv_bfloat16*)o;
    P.lse = lse;
    P.list_cnt = plan->d_list_cnt;
    P.list = plan->d_list;
    P.pair = plan->d_pair;
    P.order = plan->d_order;
    P.seg = plan->d_seg;
    P.specs = plan->d_specs;
    P.sbits = plan->d_sbits;
    P.status = plan->d_status;
    P.d = d;
    P.scale_log2 = scale * 1.4426950408889634f;
    P.tab_words_s = plan->has_stripe ? d.sbits_words : 0;
    P.tab_words_t = plan->has_stripe ? vsa_ttab_words(d.T) : 0;

    cudaStream_t s = (cudaStream_t)stream;
    if (D == 128 && d.Bk == 128) return launch_attn<128, 128>(P, B, s);
    if (D == 128 && d.Bk == 64) return launch_attn<128, 64>(P, B, s);
    if (D == 64 && d.Bk == 128) return launch_attn<64, 128>(P, B, s);
    return launch_attn<64, 64>(P, B, s);
}

// 2D tensor map over bf16 rows of D elements, box {64, box_rows}, 128-byte
// swizzle (the layout the tcgen05 kernels' shared-memory descriptors expect).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

bool vsa_make_tmap_bf16(CUtensorMap* m, const void* base, long long rows, int D, int box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// One warp waits, with the attention kernel's bounded wait, on an mbarrier
// that nothing arrives at; the wait expires after `limit` cycles and records
// the timeout in the status word.
__global__ void watchdog_selftest_kernel(unsigned int* status, long long limit)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const Ctl ctl{&abort_flag, status};
    if (threadIdx.x == 0) mbar_wait_limit(b, 0, ctl, limit);
    __syncthreads();
}

}  // namespace

extern "C" int vsa_selftest_watchdog(vsa_plan_t plan, long long cycles, void* stream)
{
    if (!plan || cycles <= 0 || cycles > kWatchdogCycles) return VSA_ERR_INVALID_ARG;
    watchdog_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(plan->d_status, cycles);
    return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

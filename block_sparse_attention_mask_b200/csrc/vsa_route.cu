// SVG online routing for sm_100a: for a sample of query rows, attention
// outputs under full attention and under each head's spatial and temporal
// candidate masks, their deviations, and the per-head choice.
//
// What it computes ("Sparse VideoGen: accelerating video diffusion attention
// on TPU", section on SVG heads): for every sampled natural token n of every
// (batch, head), o_full(n), o_spatial(n) and o_temporal(n) = softmax over the
// mask's kept keys of scale * q_n.k, times v; the deviation of a candidate is
// the mean over the sampled rows, the batch and the head dimension of
// (o_candidate - o_full)^2, and the head goes temporal only when its temporal
// deviation is strictly smaller.  The routing flags then select, per head,
// the candidate spec (and with it the head's token order) without changing
// any tensor shape ("Sparse VideoGen ... on TPU", "supporting dynamic routing
// with fixed tensor shapes").
//
// route_partial_kernel: one CTA = 128 sampled rows of one (batch, head) and a
// contiguous range of kv tiles (64 natural keys each; the key range of a
// head is split across CTAs so that the grid fills the SMs).  12 warps:
//   warps 8..11 gather the 128 sampled q rows into shared memory (128-byte
//               swizzled, K-major), then
//   warp 8      TMA producer: lane 0 K tiles, lane 1 V tiles (3-stage rings);
//   warp 9      MMA issuer (one elected lane): S_j = Q K_j^T into S_{j mod 2}
//               (both operands in shared memory), then O_full += P_full V_j
//               and O_sp += P_sp V_j with P read from TMEM (P_full over
//               columns [0, 32) of S_{j mod 2}, P_sp over [32, 64)) and
//               O_tm += P_tm V_j with P_tm in shared memory (two buffers).
//               Issue order QK_0, QK_1, PV_0, QK_2, PV_1, ...: S_{j+2} is
//               queued behind PV_j, so P_j is read before it is overwritten,
//               and QK_{j+1} runs while the softmax works on tile j.
//   warps 0..7  softmax: thread r of warpgroup G owns sampled row r and keys
//               [32G, 32G + 32) of every tile.  Both warpgroups read the
//               whole tile's scores for the row max, so both keep the same
//               running max with no exchange; one running max (of the full row)
//               serves all three accumulators: p = 2^(s*scale*log2e - m) once
//               per key, masked by the spatial and temporal keep bits into
//               P_sp and P_tm; three running sums per warpgroup.
// The three accumulators are shared by consecutive tiles, so a rescale (when
// the running max grows by more than 2^8) first waits for the previous
// tile's PV MMAs.
// TMEM: S_0 [0,64), S_1 [64,128), O_full [128,128+D), O_sp, O_tm after it:
// 512 columns for D = 128.  Each CTA writes its partial (max, three sums,
// three unnormalised outputs); route_combine_kernel merges the partials of a
// row, normalises, and forms the row's squared deviations;
// route_reduce_kernel sums them per head in a fixed order (deterministic)
// and sets the flag.  Every mbarrier wait is bounded (VSA_DEV_TIMEOUT in the
// status word).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "vsa_internal.h"
#include "vsa_sm100.cuh"

namespace {

constexpr int kRRows = 128;                 // sampled rows per CTA (TMEM lanes)
constexpr int kRBK = 64;                    // keys per kv tile
constexpr int kRSoftmaxWarps = 8;           // two warpgroups, 32 keys of a tile each
constexpr int kRProducerWarp = 8;
constexpr int kRMmaWarp = 9;
constexpr int kRThreads = 384;
constexpr float kRRescale = 8.0f;           // lazy rescale threshold, log2 units
constexpr int kRMaxSplits = 64;
constexpr int kRDChunk = 16;                // output columns per combine CTA

template <int D>
struct RCfg {
    static constexpr int Q_BYTES = kRRows * D * 2;
    static constexpr int P_BYTES = kRRows * kRBK * 2;      // one P_tm buffer (one 64-key block)
    static constexpr int KV_BYTES = kRBK * D * 2;
    static constexpr int STAGES = 3;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = OFF_Q + Q_BYTES;           // two P_tm buffers
    static constexpr int OFF_K = OFF_P + 2 * P_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
    // the two warpgroups' running sums for the epilogue [2][3][128]
    static constexpr int OFF_SUM = OFF_V + STAGES * KV_BYTES;
    static constexpr int OFF_BAR = OFF_SUM + 2 * 3 * kRRows * 4;
    // k_full[3], k_empty[3], v_full[3], v_empty[3], q_full, s_full[2], p_full[2], pv_done, drain,
    // all_done, s_read[2]
    static constexpr int NBAR = 4 * STAGES + 10;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;   // tmem addr, abort, issued[3]
    static constexpr int SMEM = OFF_MISC + 20;
    static constexpr int COL_S0 = 0;
    static constexpr int COL_S1 = kRBK;
    static constexpr int COL_OF = 2 * kRBK;
    static constexpr int TMEM_COLS = 512;
    static_assert(2 * kRBK + 3 * D <= TMEM_COLS, "TMEM budget");
    // kind::f16 instruction descriptors: D f32, A/B bf16, M = 128;
    // QK: A and B K-major, N = 64; PV: B MN-major, N = D
    static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) |
                                         ((uint32_t)(kRBK >> 3) << 17) | ((uint32_t)(kRRows >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kRRows >> 4) << 24);
    // partial record per (unit, split): m, l_full, l_sp, l_tm, then the three
    // unnormalised outputs, each [D][128 rows] (row fastest)
    static constexpr int PART_FLOATS = (4 + 3 * D) * kRRows;
};

struct RouteParams {
    CUtensorMap tm_k, tm_v;             // [B*heads*N, D] bf16 natural order, box {64, 64}
    const __nv_bfloat16* q;             // [B*heads*N, D]
    const int32_t* rows;                // [R] sampled natural tokens
    const vsa_mask_spec* cand;          // [2][heads]
    float* part;                        // [units][S] partial records
    unsigned int* status;
    int T, H, W, N, heads;
    int R, nRT, nK, S;
    float scale_log2;
};

// Bits [lo, hi) of a 32-key word, lo and hi relative to the word start.
__device__ __forceinline__ uint32_t span32(int lo, int hi)
{
    lo = max(lo, 0);
    hi = min(hi, 32);
    const int d = hi - lo;                        // 0 < d <= 32 and 0 <= lo < 32 when kept
    return d > 0 ? (0xFFFFFFFFu >> (32 - d)) << lo : 0u;
}

// Keep words of one sampled row over a walk of 32-key words (natural keys
// [kw, kw + 32), kw advancing by a fixed stride), for the spatial candidate
// (|t_k - tq| <= rt) and the temporal candidate (|h_k - hq| <= rh and
// |w_k - wq| <= rw), each also keeping frame 0 when its sink bit is set; keys
// past N are dropped.  The latent row g = kw / W, the column c = kw mod W and
// h = g mod H of the word start are carried from word to word, so a word
// costs a few 32-bit operations per latent row it meets.
struct RowWalk {
    int kw, c, hr;                      // word start, its column, its h
    int sp_lo, sp_hi, sink_hi_s, sink_hi_t;
    int hq, rh, wlo, whi1;
    int W, H, N;

    __device__ __forceinline__ void init(const vsa_mask_spec& ms, const vsa_mask_spec& mt, int T, int Hh, int Wd,
                                         int Nn, int tq, int hq_, int wq, int kw0)
    {
        const int HW = Hh * Wd;
        W = Wd;
        H = Hh;
        N = Nn;
        kw = kw0;
        c = kw0 % Wd;
        hr = (kw0 / Wd) % Hh;
        sp_lo = max(0, tq - ms.rt) * HW;
        sp_hi = min(T, tq + min(ms.rt, T) + 1) * HW;
        sink_hi_s = ms.sink ? HW : 0;
        sink_hi_t = mt.sink ? HW : 0;
        hq = hq_;
        rh = mt.rh;
        wlo = max(0, wq - mt.rw);
        whi1 = min(Wd - 1, wq + min(mt.rw, Wd)) + 1;
    }

    __device__ __forceinline__ void bits(uint32_t& sp, uint32_t& tm) const
    {
        sp = kw < sink_hi_s ? span32(-kw, sink_hi_s - kw) : 0u;
        if (kw < sp_hi && kw + 32 > sp_lo) sp |= span32(sp_lo - kw, sp_hi - kw);
        tm = kw < sink_hi_t ? span32(-kw, sink_hi_t - kw) : 0u;
        int hh = hr;
        for (int off = -c; off < 32; off += W) {
            const int dh = hh - hq;
            if (dh <= rh && -dh <= rh) tm |= span32(off + wlo, off + whi1);
            if (++hh == H) hh = 0;
        }
        if (kw + 32 > N) {
            const uint32_t real = span32(0, N - kw);
            sp &= real;
            tm &= real;
        }
    }

    __device__ __forceinline__ void advance(int stride)
    {
        kw += stride;
        c += stride;
        while (c >= W) {
            c -= W;
            if (++hr == H) hr = 0;
        }
    }
};

template <int D>
__global__ void __launch_bounds__(kRThreads, 1) route_partial_kernel(const __grid_constant__ RouteParams P)
{
    using C = RCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // CTA -> (unit = (b*heads + h)*nRT + row tile, split)
    const int split = blockIdx.x % P.S;
    const int unit = blockIdx.x / P.S;
    const int rt = unit % P.nRT;
    const int bh = unit / P.nRT;
    const int head = bh % P.heads;
    const int j0 = (int)((long long)split * P.nK / P.S);
    const int n = (int)((long long)(split + 1) * P.nK / P.S) - j0;   // >= 1 since S <= nK
    const long long base_row = (long long)bh * P.N;

    const uint32_t s_base = smem_addr(smem);
    const uint32_t bar0 = s_base + C::OFF_BAR;
    auto BAR_KF = [&](int s) { return bar0 + 8u * s; };
    auto BAR_KE = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
    auto BAR_VF = [&](int s) { return bar0 + 8u * (2 * C::STAGES + s); };
    auto BAR_VE = [&](int s) { return bar0 + 8u * (3 * C::STAGES + s); };
    const uint32_t BAR_QF = bar0 + 8u * (4 * C::STAGES);
    auto BAR_SF = [&](int x) { return BAR_QF + 8u * (1 + x); };
    auto BAR_PF = [&](int x) { return BAR_QF + 8u * (3 + x); };
    const uint32_t BAR_PV = BAR_QF + 40u;
    const uint32_t BAR_DR = BAR_QF + 48u;
    const uint32_t BAR_FIN = BAR_QF + 56u;        // one phase: every MMA of the CTA complete
    auto BAR_SC = [&](int x) { return BAR_QF + 8u * (8 + x); };   // all 8 softmax warps read S_x
    uint32_t* tmem_slot = (uint32_t*)(smem + C::OFF_MISC);
    volatile int* abort_flag = (volatile int*)(smem + C::OFF_MISC + 4);
    volatile int* issued = (volatile int*)(smem + C::OFF_MISC + 8);   // K copies, V copies, MMAs
    const Ctl ctl{abort_flag, P.status};

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(BAR_KF(s), 1);
            mbar_init(BAR_KE(s), 1);
            mbar_init(BAR_VF(s), 1);
            mbar_init(BAR_VE(s), 1);
        }
        mbar_init(BAR_QF, 128);                 // the four gathering warps' threads
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR_SF(x), 1);
            mbar_init(BAR_PF(x), kRSoftmaxWarps);
        }
        mbar_init(BAR_PV, 1);
        mbar_init(BAR_DR, 1);
        mbar_init(BAR_FIN, 1);
        for (int x = 0; x < 2; ++x) mbar_init(BAR_SC(x), kRSoftmaxWarps);
        *abort_flag = 0;
        issued[0] = issued[1] = issued[2] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kRMmaWarp) {
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

    if (warp >= kRProducerWarp) {
        // ---- gather the sampled q rows: thread i -> row i, 16-byte chunks
        // into the 128-byte-swizzled K-major layout (chunk u of row i at
        // u ^ (i mod 8)), in D/64 column blocks of 128 rows x 128 bytes
        const int i = threadIdx.x - 32 * kRProducerWarp;
        int tok = __ldg(P.rows + min(rt * kRRows + i, P.R - 1));
        if (tok < 0 || tok >= P.N) {
            atomicOr(P.status, VSA_DEV_BADSTATE);
            tok = 0;
        }
        const uint4* src = reinterpret_cast<const uint4*>(P.q + (base_row + tok) * D);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint4 x = __ldg(src + c * 8 + u);
                const uint32_t dst = s_base + C::OFF_Q + c * (kRRows * 128) + i * 128 + ((u ^ (i & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(x.x), "r"(x.y), "r"(x.z),
                             "r"(x.w)
                             : "memory");
            }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(BAR_QF);
    }

    if (warp == kRProducerWarp) {
        // ---------------- TMA producer: lane 0 K, lane 1 V ----------------
        if (lane < 2) {
            const bool is_k = lane == 0;
            const CUtensorMap* map = is_k ? &P.tm_k : &P.tm_v;
            const int off = is_k ? C::OFF_K : C::OFF_V;
            int cnt = 0;
            for (int j = 0; j < n; ++j, cnt = j) {
                const int st = j % C::STAGES;
                const uint32_t empty = is_k ? BAR_KE(st) : BAR_VE(st);
                const uint32_t full = is_k ? BAR_KF(st) : BAR_VF(st);
                if (j >= C::STAGES && !mbar_wait(empty, (uint32_t)(j / C::STAGES - 1) & 1, ctl)) break;
                const int row = (int)(base_row + (long long)(j0 + j) * kRBK);
                mbar_expect_tx(full, C::KV_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + off + st * C::KV_BYTES + c * kRBK * 128, map, c * 64, row, full);
            }
            issued[is_k ? 0 : 1] = cnt;
        }
        __syncwarp();
    } else if (warp == kRMmaWarp) {
        // ---------------- MMA issuer ----------------
        const uint32_t leader = elect_one();
        if (mbar_wait_warp(BAR_QF, 0, ctl)) {
            tc_fence_after();
            const uint64_t qdesc = smem_desc(s_base + C::OFF_Q, 16, 1024);
            const uint64_t pdesc0 = smem_desc(s_base + C::OFF_P, 16, 1024);
            const uint64_t kdesc0 = smem_desc(s_base + C::OFF_K, 16, 1024);
            const uint64_t vdesc0 = smem_desc(s_base + C::OFF_V, kRBK * 128, 1024);
            constexpr uint64_t kStageStep = (uint64_t)(C::KV_BYTES >> 4);
            // K-major operand step kk (16 elements): block kk/4 of 64, 32 bytes per step inside it
            auto kstep = [](int kk, int rows) -> uint64_t {
                return (uint64_t)((((kk >> 2) * (rows * 128)) + (kk & 3) * 32) >> 4);
            };
            auto issue_qk = [&](int j) -> bool {
                const int st = j % C::STAGES;
                if (!mbar_wait_warp(BAR_KF(st), (uint32_t)(j / C::STAGES) & 1, ctl)) return false;
                tc_fence_after();
                const uint32_t dS = tmem + ((j & 1) ? C::COL_S1 : C::COL_S0);
                const uint64_t kd = kdesc0 + (uint64_t)st * kStageStep;
                mma_ss_lead<0>(dS, qdesc, kd, C::IDESC_QK, leader);
#pragma unroll
                for (int kk = 1; kk < D / 16; ++kk)
                    mma_ss_lead<1>(dS, qdesc + kstep(kk, kRRows), kd + kstep(kk, kRBK), C::IDESC_QK, leader);
                tc_commit_lead(BAR_SF(j & 1), leader);
                tc_commit_lead(BAR_KE(st), leader);
                return true;
            };
            bool go = issue_qk(0);
            if (go && leader) issued[2] = 1;
            go = go && (n < 2 || issue_qk(1));
            for (int j = 0; go && j < n; ++j) {
                const int x = j & 1, vs = j % C::STAGES;
                go = mbar_wait_warp(BAR_PF(x), (uint32_t)(j >> 1) & 1, ctl) &&
                     mbar_wait_warp(BAR_VF(vs), (uint32_t)(j / C::STAGES) & 1, ctl);
                if (!go) break;
                tc_fence_after();
                const uint64_t vd = vdesc0 + (uint64_t)vs * kStageStep;
                const uint32_t aS = tmem + (x ? C::COL_S1 : C::COL_S0);
                const uint64_t pd = pdesc0 + (uint64_t)x * (C::P_BYTES >> 4);
                // O_full += P_full V (TMEM columns [0, 32) of S_x), O_sp += P_sp V
                // ([32, 64)), O_tm += P_tm V (shared memory); the first tile of
                // the CTA initialises the accumulators
#pragma unroll
                for (int kk = 0; kk < kRBK / 16; ++kk) {
                    const uint64_t vk = vd + (uint64_t)((kk * 16 * 128) >> 4);
                    if (j == 0 && kk == 0) {
                        mma_ts_lead<0>(tmem + C::COL_OF, aS, vk, C::IDESC_PV, leader);
                        mma_ts_lead<0>(tmem + C::COL_OF + D, aS + 32, vk, C::IDESC_PV, leader);
                        mma_ss_lead<0>(tmem + C::COL_OF + 2 * D, pd, vk, C::IDESC_PV, leader);
                    } else {
                        mma_ts_lead<1>(tmem + C::COL_OF, aS + kk * 8, vk, C::IDESC_PV, leader);
                        mma_ts_lead<1>(tmem + C::COL_OF + D, aS + 32 + kk * 8, vk, C::IDESC_PV, leader);
                        mma_ss_lead<1>(tmem + C::COL_OF + 2 * D, pd + (uint64_t)(kk * 2), vk, C::IDESC_PV, leader);
                    }
                }
                tc_commit_lead(BAR_PV, leader);
                tc_commit_lead(BAR_VE(vs), leader);
                // S_{j+2} reuses S_x: queued behind PV_j, so P_j is read first
                if (j + 2 < n) go = issue_qk(j + 2);
            }
            // a single-phase barrier for the epilogue (the PV barrier's parity
            // cannot tell its last phase from the one before)
            if (go) tc_commit_lead(BAR_FIN, leader);
        }
    } else if (warp < kRSoftmaxWarps) {
        // ---------------- softmax: warpgroup G, thread r owns sampled row r ----------------
        const int G = warp >> 2;
        const int r = threadIdx.x & (kRRows - 1);
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        int tok = __ldg(P.rows + min(rt * kRRows + r, P.R - 1));
        if (tok < 0 || tok >= P.N) tok = 0;              // flagged by the gather
        const int HW = P.H * P.W;
        const int tq = tok / HW, hq = (tok % HW) / P.W, wq = tok % P.W;
        RowWalk walk;
        walk.init(P.cand[head], P.cand[P.heads + head], P.T, P.H, P.W, P.N, tq, hq, wq, j0 * kRBK + 32 * G);
        const float sl = P.scale_log2;
        const unsigned long long sl2 = f2_pack(sl, sl);
        float* sums = (float*)(smem + C::OFF_SUM);        // [G][3][row]
        float m_run = -INFINITY;                          // log2 units, identical in both warpgroups
        float lf = 0.0f, ls = 0.0f, lt = 0.0f;            // this warpgroup's keys only
        bool ok = true;
        for (int j = 0; j < n && ok; ++j) {
            const int x = j & 1;
            const uint32_t tS = tmem + lane_off + (x ? C::COL_S1 : C::COL_S0);
            const int left = P.N - (walk.kw - 32 * G);    // real keys of the tile (>= 1)
            uint32_t ws, wt;
            walk.bits(ws, wt);
            walk.advance(kRBK);
            if (!mbar_wait_warp(BAR_SF(x), (uint32_t)(j >> 1) & 1, ctl)) { ok = false; break; }
            tc_fence_after();
            // both warpgroups read the whole tile: the row max needs all 64
            // keys, and each exponentiates its own 32
            float s[32];
            float mx;
            {
                uint32_t sr[32], so[32];
                tmem_ld32(tS + 32 * G, sr);
                tmem_ld32(tS + 32 * (G ^ 1), so);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR_SC(x));    // S_x read: P may overwrite it
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    reg_fence(sr[c]);
                    reg_fence(so[c]);
                    s[c] = __uint_as_float(sr[c]);
                }
                float b;
                if (left >= kRBK) {                       // every key real (all but the last tile)
                    float a = s[0], a2 = __uint_as_float(so[0]);
#pragma unroll
                    for (int c = 1; c < 31; c += 2) {
                        a = max3(a, s[c], s[c + 1]);
                        a2 = max3(a2, __uint_as_float(so[c]), __uint_as_float(so[c + 1]));
                    }
                    a = max3(a, s[31], a2);
                    b = __uint_as_float(so[31]);
                    mx = fmaxf(a, b);
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (32 * G + c >= left) s[c] = -INFINITY;
                    float a = s[0];
#pragma unroll
                    for (int c = 1; c < 32; ++c) a = fmaxf(a, s[c]);
                    b = -INFINITY;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (32 * (G ^ 1) + c < left) b = fmaxf(b, __uint_as_float(so[c]));
                    mx = fmaxf(a, b);
                }
            }
            const float mxs = mx * sl;                    // finite: every tile holds a real key
            float alpha = 1.0f;
            bool need_o = false;
            if (m_run == -INFINITY) {
                m_run = mxs;                              // nothing accumulated yet
            } else if (mxs > m_run + kRRescale) {
                alpha = ex2(m_run - mxs);
                lf *= alpha;
                ls *= alpha;
                lt *= alpha;
                m_run = mxs;
                need_o = true;
            }
            if (__any_sync(0xFFFFFFFFu, need_o)) {
                // the accumulators still take PV_{j-1}: wait for it, then this
                // warpgroup rescales its half of the 3 D columns
                ok = mbar_wait_warp(BAR_PV, (uint32_t)(j - 1) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
#pragma unroll 1
                for (int c = G * (3 * D / 64); c < (G + 1) * (3 * D / 64); ++c) {
                    uint32_t ov[32];
                    const uint32_t ta = tmem + lane_off + C::COL_OF + c * 32;
                    tmem_ld32(ta, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        reg_fence(ov[i]);
                        ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    }
                    tmem_st32(ta, ov);
                }
            }
            const float mneg = -m_run;
            const unsigned long long mneg2 = f2_pack(mneg, mneg);
            float p[32];
            uint32_t pf[16], ps[16], pt[16];
            unsigned long long af2 = 0ull;                // packed pair sums
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float x0, x1;
                f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), sl2, mneg2), x0, x1);
                p[2 * i] = ex2(x0);
                p[2 * i + 1] = ex2(x1);
                af2 = f2_add(af2, f2_pack(p[2 * i], p[2 * i + 1]));
                pf[i] = pack_bf16(p[2 * i], p[2 * i + 1]);
            }
            float af, af1;
            f2_unpack(af2, af, af1);
            af += af1;
            lf += af;
            // spatial keep bits are usually all set or all clear across the
            // warp (the sampled rows are sorted, so a warp's rows share frames)
            if (__all_sync(0xFFFFFFFFu, ws == 0xFFFFFFFFu)) {
#pragma unroll
                for (int i = 0; i < 16; ++i) ps[i] = pf[i];
                ls += af;
            } else if (__all_sync(0xFFFFFFFFu, ws == 0u)) {
#pragma unroll
                for (int i = 0; i < 16; ++i) ps[i] = 0u;
            } else {
                unsigned long long a2 = 0ull;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float s0 = (ws & (1u << (2 * i))) ? p[2 * i] : 0.0f;
                    const float s1 = (ws & (1u << (2 * i + 1))) ? p[2 * i + 1] : 0.0f;
                    a2 = f2_add(a2, f2_pack(s0, s1));
                    ps[i] = pack_bf16(s0, s1);
                }
                float a0, a1;
                f2_unpack(a2, a0, a1);
                ls += a0 + a1;
            }
            if (__all_sync(0xFFFFFFFFu, wt == 0u)) {
#pragma unroll
                for (int i = 0; i < 16; ++i) pt[i] = 0u;
            } else {
                unsigned long long a2 = 0ull;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float t0 = (wt & (1u << (2 * i))) ? p[2 * i] : 0.0f;
                    const float t1 = (wt & (1u << (2 * i + 1))) ? p[2 * i + 1] : 0.0f;
                    a2 = f2_add(a2, f2_pack(t0, t1));
                    pt[i] = pack_bf16(t0, t1);
                }
                float a0, a1;
                f2_unpack(a2, a0, a1);
                lt += a0 + a1;
            }
            // S_j complete implies PV_{j-2} complete, the last reader of S_x's
            // P columns and of P_tm buffer x; the other warpgroup must have
            // read its S_x columns too
            ok = mbar_wait_warp(BAR_SC(x), (uint32_t)(j >> 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            tmem_st16(tS + 16 * G, pf);                   // P_full: S_x columns [0, 32)
            tmem_st16(tS + 32 + 16 * G, ps);              // P_sp:   S_x columns [32, 64)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int chunk = 4 * G + u;              // keys 32G + 8u .. + 8 of row r
                const uint32_t dst = s_base + C::OFF_P + x * C::P_BYTES + r * 128 + ((chunk ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pt[4 * u]),
                             "r"(pt[4 * u + 1]), "r"(pt[4 * u + 2]), "r"(pt[4 * u + 3])
                             : "memory");
            }
            tmem_st_wait();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR_PF(x));
        }

        // ---------------- partial record of this CTA ----------------
        const bool have = ok && mbar_wait_warp(BAR_FIN, 0, ctl);
        tc_fence_after();
        sums[(G * 3 + 0) * kRRows + r] = lf;
        sums[(G * 3 + 1) * kRRows + r] = ls;
        sums[(G * 3 + 2) * kRRows + r] = lt;
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kRSoftmaxWarps) : "memory");
        float* rec = P.part + ((size_t)unit * P.S + split) * C::PART_FLOATS;
        const bool all = !*abort_flag && have;
        if (G == 0) {
            rec[r] = all ? m_run : -INFINITY;
#pragma unroll
            for (int k = 0; k < 3; ++k)
                rec[(1 + k) * kRRows + r] = all ? sums[k * kRRows + r] + sums[(3 + k) * kRRows + r] : 0.0f;
        }
        if (have) {
            // warpgroup G writes its half of the 3 D accumulator columns
#pragma unroll 1
            for (int c = G * (3 * D / 64); c < (G + 1) * (3 * D / 64); ++c) {
                uint32_t ov[32];
                tmem_ld32(tmem + lane_off + C::COL_OF + c * 32, ov);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    reg_fence(ov[i]);
                    rec[(4 + c * 32 + i) * kRRows + r] = __uint_as_float(ov[i]);
                }
            }
        }
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // copies or MMAs of an aborted CTA may still be in flight: each role
        // waits (bounded) for its own before TMEM is freed
        if (warp == kRProducerWarp && lane < 2) {
            const int cnt = issued[lane];
            for (int j = cnt > C::STAGES ? cnt - C::STAGES : 0; j < cnt; ++j)
                mbar_drain(lane == 0 ? BAR_KF(j % C::STAGES) : BAR_VF(j % C::STAGES),
                           (uint32_t)(j / C::STAGES) & 1, kDrainCycles);
        }
        if (warp == kRMmaWarp && issued[2]) {
            const uint32_t leader = elect_one();
            tc_commit_lead(BAR_DR, leader);
            if (leader) mbar_drain(BAR_DR, 0, kDrainCycles);
            __syncwarp();
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == kRMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
    }
}

// Merge the S partial records of one unit's 128 rows for 16 of the D output
// columns (blockIdx.y), normalise the three outputs and write each row's
// squared deviations (spatial, temporal) from the full output over those
// columns.  Grid (units, D / 16): many CTAs and 48 independent loads per
// split keep enough reads in flight.
template <int D>
__global__ void __launch_bounds__(kRRows) route_combine_kernel(const float* part, int S, int R, int nRT,
                                                              float2* row_err)
{
    using C = RCfg<D>;
    __shared__ float wsm[kRMaxSplits][kRRows];
    const int unit = blockIdx.x, dc = blockIdx.y, r = threadIdx.x;
    const float* base = part + (size_t)unit * S * C::PART_FLOATS;
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, base[(size_t)s * C::PART_FLOATS + r]);
    float lf = 0.0f, ls = 0.0f, lt = 0.0f;
    for (int s = 0; s < S; ++s) {
        const float* b = base + (size_t)s * C::PART_FLOATS;
        const float w = (b[r] == -INFINITY) ? 0.0f : ex2(b[r] - m);
        wsm[s][r] = w;
        lf += w * b[kRRows + r];
        ls += w * b[2 * kRRows + r];
        lt += w * b[3 * kRRows + r];
    }
    float af[kRDChunk], as[kRDChunk], at[kRDChunk];
#pragma unroll
    for (int i = 0; i < kRDChunk; ++i) af[i] = as[i] = at[i] = 0.0f;
    for (int s = 0; s < S; ++s) {
        const float w = wsm[s][r];
        const float* b = base + (size_t)s * C::PART_FLOATS + (size_t)(4 + dc * kRDChunk) * kRRows + r;
#pragma unroll
        for (int i = 0; i < kRDChunk; ++i) {
            af[i] += w * b[(size_t)i * kRRows];
            as[i] += w * b[(size_t)(D + i) * kRRows];
            at[i] += w * b[(size_t)(2 * D + i) * kRRows];
        }
    }
    const float inf_ = lf > 0.0f ? 1.0f / lf : 0.0f;
    const float ins = ls > 0.0f ? 1.0f / ls : 0.0f;
    const float int_ = lt > 0.0f ? 1.0f / lt : 0.0f;
    float es = 0.0f, et = 0.0f;
#pragma unroll
    for (int i = 0; i < kRDChunk; ++i) {
        const float of = af[i] * inf_;
        const float ds = as[i] * ins - of, dt = at[i] * int_ - of;
        es += ds * ds;
        et += dt * dt;
    }
    const bool real = (unit % nRT) * kRRows + r < R;
    row_err[((size_t)unit * gridDim.y + dc) * kRRows + r] = real ? make_float2(es, et) : make_float2(0.0f, 0.0f);
}

// Per head: mean squared deviation over the batch, the sampled rows and the
// head dimension, in a fixed summation order; flag 1 = temporal.  row_err
// holds [unit][D / 16][128] (zeros for padding rows).
__global__ void __launch_bounds__(256) route_reduce_kernel(const float2* row_err, int B, int heads, int nRT, int R,
                                                          int D, float* err, int32_t* flags)
{
    __shared__ double red[2][256];
    const int h = blockIdx.x, t = threadIdx.x;
    const long long per_bh = (long long)nRT * (D / kRDChunk) * kRRows;
    double es = 0.0, et = 0.0;
    for (int b = 0; b < B; ++b) {
        const float2* e = row_err + ((long long)b * heads + h) * per_bh;
        for (long long i = t; i < per_bh; i += 256) {
            es += (double)e[i].x;
            et += (double)e[i].y;
        }
    }
    red[0][t] = es;
    red[1][t] = et;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (t < w) {
            red[0][t] += red[0][t + w];
            red[1][t] += red[1][t + w];
        }
        __syncthreads();
    }
    if (t == 0) {
        const double den = (double)B * R * D;
        const float e_s = (float)(red[0][0] / den), e_t = (float)(red[1][0] / den);
        err[2 * h] = e_s;
        err[2 * h + 1] = e_t;
        flags[h] = e_t < e_s ? 1 : 0;
    }
}

// specs[h] = flags[h] ? temporal candidate : spatial candidate
__global__ void route_apply_kernel(const vsa_mask_spec* cand, const int32_t* flags, int heads, vsa_mask_spec* specs)
{
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h < heads) specs[h] = flags[h] ? cand[heads + h] : cand[h];
}

}  // namespace

// ---- host side ----------------------------------------------------------

namespace {

struct RouteShape {
    int nRT, nK, S;
    long long units;
    size_t part_bytes, err_bytes;
};

// Splits of the key range: fewest waves x tiles per CTA (+8 tiles of fixed
// cost for the gather and the ~200 KB partial record), the smaller split on a
// tie.
int choose_splits(long long units, int nK, int sms)
{
    int best = 1;
    long long best_cost = -1;
    const int smax = nK < kRMaxSplits ? nK : kRMaxSplits;
    for (int s = 1; s <= smax; ++s) {
        const long long waves = (units * s + sms - 1) / sms;
        const long long cost = waves * ((nK + s - 1) / s + 8);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

int route_shape(vsa_plan_t plan, int B, int D, int n_rows, RouteShape* out)
{
    if (!plan || B < 1 || n_rows < 1) return VSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
    const vsa_dims& d = plan->d;
    if ((long long)B * d.heads * d.N + 2 * kRBK > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return VSA_ERR_CUDA;
    RouteShape r;
    r.nRT = (n_rows + kRRows - 1) / kRRows;
    r.nK = (int)((d.N + kRBK - 1) / kRBK);
    r.units = (long long)B * d.heads * r.nRT;
    r.S = choose_splits(r.units, r.nK, sms);
    const int pf = (4 + 3 * D) * kRRows;
    r.part_bytes = (size_t)r.units * r.S * pf * sizeof(float);
    r.err_bytes = (size_t)r.units * (D / kRDChunk) * kRRows * sizeof(float2);
    if (r.units * r.S > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
    *out = r;
    return VSA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <int D>
int launch_route(const RouteParams& P, float2* row_err, int B, int D_, float* err, int32_t* flags, cudaStream_t s)
{
    using C = RCfg<D>;
    const int smem = 1024 + C::SMEM;
    if (smem > 227 * 1024) return VSA_ERR_UNSUPPORTED;
    auto kern = route_partial_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return VSA_ERR_CUDA;
    const long long units = (long long)B * P.heads * P.nRT;
    kern<<<(unsigned)(units * P.S), kRThreads, smem, s>>>(P);
    VSA_CUDA_TRY(cudaGetLastError());
    route_combine_kernel<D><<<dim3((unsigned)units, D / kRDChunk), kRRows, 0, s>>>(P.part, P.S, P.R, P.nRT,
                                                                                    row_err);
    VSA_CUDA_TRY(cudaGetLastError());
    route_reduce_kernel<<<P.heads, 256, 0, s>>>(row_err, B, P.heads, P.nRT, P.R, D_, err, flags);
    VSA_CUDA_TRY(cudaGetLastError());
    return VSA_OK;
}

}  // namespace

extern "C" int vsa_plan_set_route_candidates(vsa_plan_t plan, const vsa_mask_spec* spatial,
                                             const vsa_mask_spec* temporal, void* stream)
{
    if (!plan || !spatial || !temporal) return VSA_ERR_INVALID_ARG;
    const int heads = plan->d.heads;
    for (int h = 0; h < heads; ++h) {
        if (spatial[h].kind != VSA_MASK_SVG_SPATIAL || temporal[h].kind != VSA_MASK_SVG_TEMPORAL)
            return VSA_ERR_INVALID_ARG;
        int r = vsa_check_spec(&spatial[h]);
        if (r == VSA_OK) r = vsa_check_spec(&temporal[h]);
        if (r != VSA_OK) return r;
    }
    cudaStream_t s = (cudaStream_t)stream;
    if (!plan->d_cand) {
        if (cudaMalloc(&plan->d_cand, sizeof(vsa_mask_spec) * 2 * heads) != cudaSuccess) {
            cudaGetLastError();
            plan->d_cand = nullptr;
            return VSA_ERR_OOM;
        }
    }
    VSA_CUDA_TRY(cudaMemcpyAsync(plan->d_cand, spatial, sizeof(vsa_mask_spec) * heads, cudaMemcpyHostToDevice, s));
    VSA_CUDA_TRY(cudaMemcpyAsync(plan->d_cand + heads, temporal, sizeof(vsa_mask_spec) * heads,
                                 cudaMemcpyHostToDevice, s));
    // the host arrays may be released on return
    VSA_CUDA_TRY(cudaStreamSynchronize(s));
    plan->has_cand = 1;
    return VSA_OK;
}

extern "C" int vsa_svg_route_workspace_size(vsa_plan_t plan, int B, int D, int n_rows, size_t* bytes)
{
    if (!bytes) return VSA_ERR_INVALID_ARG;
    RouteShape r;
    const int e = route_shape(plan, B, D, n_rows, &r);
    if (e != VSA_OK) return e;
    *bytes = align256(r.part_bytes) + r.err_bytes;
    return VSA_OK;
}

extern "C" int vsa_svg_route(vsa_plan_t plan, const void* q, const void* k, const void* v, int B, int D,
                             const int32_t* rows, int n_rows, float scale, float* err, int32_t* flags,
                             void* workspace, size_t workspace_bytes, void* stream)
{
    if (!plan || !q || !k || !v || !rows || !err || !flags || !workspace) return VSA_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || !(scale < 1e30f)) return VSA_ERR_INVALID_ARG;
    if (!plan->has_cand) return VSA_ERR_INVALID_ARG;
    RouteShape r;
    const int e = route_shape(plan, B, D, n_rows, &r);
    if (e != VSA_OK) return e;
    if (workspace_bytes < align256(r.part_bytes) + r.err_bytes) return VSA_ERR_INVALID_ARG;
    if (!vsa_aligned16(q) || !vsa_aligned16(k) || !vsa_aligned16(v) || !vsa_aligned16(workspace) ||
        ((uintptr_t)rows & 3u) || ((uintptr_t)err & 3u) || ((uintptr_t)flags & 3u))
        return VSA_ERR_ALIGNMENT;
    const vsa_dims& d = plan->d;
    RouteParams P;
    memset(&P, 0, sizeof P);
    const long long nrows_total = (long long)B * d.heads * d.N;
    if (!vsa_make_tmap_bf16(&P.tm_k, k, nrows_total, D, kRBK) || !vsa_make_tmap_bf16(&P.tm_v, v, nrows_total, D, kRBK))
        return VSA_ERR_CUDA;
    P.q = (const __nv_bfloat16*)q;
    P.rows = rows;
    P.cand = plan->d_cand;
    P.part = (float*)workspace;
    P.status = plan->d_status;
    P.T = d.T;
    P.H = d.H;
    P.W = d.W;
    P.N = (int)d.N;
    P.heads = d.heads;
    P.R = n_rows;
    P.nRT = r.nRT;
    P.nK = r.nK;
    P.S = r.S;
    P.scale_log2 = scale * 1.4426950408889634f;
    float2* row_err = (float2*)((uint8_t*)workspace + align256(r.part_bytes));
    cudaStream_t s = (cudaStream_t)stream;
    if (D == 128) return launch_route<128>(P, row_err, B, D, err, flags, s);
    return launch_route<64>(P, row_err, B, D, err, flags, s);
}

extern "C" int vsa_plan_apply_route(vsa_plan_t plan, const int32_t* flags, void* stream)
{
    if (!plan || !flags) return VSA_ERR_INVALID_ARG;
    if (!plan->has_cand) return VSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const int heads = plan->d.heads;
    route_apply_kernel<<<(heads + 127) / 128, 128, 0, s>>>(plan->d_cand, flags, heads, plan->d_specs);
    VSA_CUDA_TRY(cudaGetLastError());
    return vsa_build_plan_kernels(plan, s);
}

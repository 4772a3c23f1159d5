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
// contiguous range of kv tiles (128 natural keys each; the key range of a
// head is split across CTAs so that the grid fills the SMs).  8 warps:
//   warps 4..7  gather the 128 sampled q rows into shared memory (128-byte
//               swizzled, K-major), then
//   warp 4      TMA producer: lane 0 K tiles, lane 1 V tiles, 2-stage rings;
//   warp 5      MMA issuer (one elected lane): S = Q K^T into TMEM (both
//               operands in shared memory); then O_full += P_full V and
//               O_sp += P_sp V with P read from TMEM (P_full over the first
//               64 columns of S, P_sp over the next 64), O_tm += P_tm V with
//               P_tm in shared memory.  The next tile's S is queued behind
//               the three PV MMAs, so P is read before S is overwritten.
//   warps 0..3  softmax: thread r owns sampled row r.  One running max (of
//               the full row) serves all three accumulators: p = 2^(s*scale*
//               log2e - m) once per key, masked by the spatial and temporal
//               keep bits into P_sp and P_tm; three running sums.
// TMEM: S [0,128), O_full [128,128+D), O_sp, O_tm after it: 512 columns for
// D = 128.  Each CTA writes its partial (max, three sums, three unnormalised
// outputs); route_combine_kernel merges the partials of a row, normalises,
// and forms the row's squared deviations; route_reduce_kernel sums them per
// head in a fixed order (deterministic) and sets the flag.
// Every mbarrier wait is bounded (VSA_DEV_TIMEOUT in the status word).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "vsa_internal.h"
#include "vsa_sm100.cuh"

namespace {

constexpr int kRRows = 128;                 // sampled rows per CTA (TMEM lanes)
constexpr int kRBK = 128;                   // keys per kv tile
constexpr int kRThreads = 256;
constexpr int kRProducerWarp = 4;
constexpr int kRMmaWarp = 5;
constexpr float kRRescale = 8.0f;           // lazy rescale threshold, log2 units
constexpr int kRMaxSplits = 64;
constexpr int kRDChunk = 16;                // output columns per combine CTA

template <int D>
struct RCfg {
    static constexpr int Q_BYTES = kRRows * D * 2;
    static constexpr int P_BYTES = kRRows * kRBK * 2;
    static constexpr int KV_BYTES = kRBK * D * 2;
    static constexpr int STAGES = 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = OFF_Q + Q_BYTES;
    static constexpr int OFF_K = OFF_P + P_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
    // k_full[2], k_empty[2], v_full[2], v_empty[2], q_full, s_full, p_full, pv_done, drain
    static constexpr int NBAR = 4 * STAGES + 5;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;   // tmem addr, abort, issued[3]
    static constexpr int SMEM = OFF_MISC + 20;
    static constexpr int COL_S = 0;
    static constexpr int COL_OF = kRBK;
    static constexpr int COL_OS = kRBK + D;
    static constexpr int COL_OT = kRBK + 2 * D;
    static constexpr int TMEM_COLS = 512;
    static_assert(kRBK + 3 * D <= TMEM_COLS, "TMEM budget");
    // kind::f16 instruction descriptors: D f32, A/B bf16, M = 128;
    // QK: A and B K-major, N = 128; PV: B MN-major, N = D
    static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) |
                                         ((uint32_t)(kRBK >> 3) << 17) | ((uint32_t)(kRRows >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kRRows >> 4) << 24);
    // partial record per (unit, split): m, l_full, l_sp, l_tm, then the three
    // unnormalised outputs, each [D][128 rows] (row fastest)
    static constexpr int PART_FLOATS = (4 + 3 * D) * kRRows;
};

struct RouteParams {
    CUtensorMap tm_k, tm_v;             // [B*heads*N, D] bf16 natural order, box {64, 128}
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
__device__ __forceinline__ uint32_t span_bits(int lo, int hi)
{
    lo = max(lo, 0);
    hi = min(hi, 32);
    if (hi <= lo) return 0u;
    return (uint32_t)(((1ull << hi) - 1ull) ^ ((1ull << lo) - 1ull));
}

// OR the natural-key interval [lo, hi) into the tile's keep words (tile keys
// start at k0).
__device__ __forceinline__ void or_span(uint32_t (&w)[kRBK / 32], long long k0, long long lo, long long hi)
{
    const long long a = lo - k0, b = hi - k0;
    if (b <= 0 || a >= kRBK) return;
#pragma unroll
    for (int i = 0; i < kRBK / 32; ++i) w[i] |= span_bits((int)max(a - 32 * i, -1LL), (int)min(b - 32 * i, 33LL));
}

// Keep words of a sampled row (frame tq, row hq, column wq) over natural keys
// [k0, k0 + 128) for the spatial candidate (|t_k - tq| <= rt) and the
// temporal candidate (|h_k - hq| <= rh and |w_k - wq| <= rw), each also
// keeping frame 0 when its sink bit is set.  Keys past N are dropped.
__device__ __forceinline__ void route_row_bits(const vsa_mask_spec& ms, const vsa_mask_spec& mt, int T, int H,
                                               int W, long long N, int tq, int hq, int wq, long long k0,
                                               uint32_t (&sp)[kRBK / 32], uint32_t (&tm)[kRBK / 32])
{
    const long long HW = (long long)H * W;
#pragma unroll
    for (int i = 0; i < kRBK / 32; ++i) sp[i] = tm[i] = 0u;
    if (ms.sink) or_span(sp, k0, 0, HW);
    or_span(sp, k0, (long long)max(0, tq - ms.rt) * HW, (long long)min(T, tq + ms.rt + 1) * HW);
    if (mt.sink) or_span(tm, k0, 0, HW);
    // latent rows g = t*H + h that meet the tile: keep columns |w - wq| <= rw
    const long long wlo = max(0, wq - mt.rw), whi = min(W - 1, wq + mt.rw) + 1;
    const long long g1 = min(k0 + kRBK, N) - 1;
    for (long long g = k0 / W; g * W <= g1; ++g) {
        const int h = (int)(g % H);
        if (h - hq <= mt.rh && hq - h <= mt.rh) or_span(tm, k0, g * W + wlo, g * W + whi);
    }
    if (k0 + kRBK > N) {
        const int nreal = (int)(N - k0);
#pragma unroll
        for (int i = 0; i < kRBK / 32; ++i) {
            const uint32_t r = span_bits(0, nreal - 32 * i);
            sp[i] &= r;
            tm[i] &= r;
        }
    }
}

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
    const uint32_t BAR_SF = BAR_QF + 8u;
    const uint32_t BAR_PF = BAR_QF + 16u;
    const uint32_t BAR_PV = BAR_QF + 24u;
    const uint32_t BAR_DR = BAR_QF + 32u;
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
        mbar_init(BAR_SF, 1);
        mbar_init(BAR_PF, 4);                   // the four softmax warps
        mbar_init(BAR_PV, 1);
        mbar_init(BAR_DR, 1);
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

    if (warp >= 4) {
        // ---- gather the sampled q rows: thread i -> row i, 16-byte chunks
        // into the 128-byte-swizzled K-major layout (chunk u of row i at
        // u ^ (i mod 8)), in D/64 column blocks of 128 rows x 128 bytes
        const int i = threadIdx.x - 128;
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
            const uint64_t pdesc = smem_desc(s_base + C::OFF_P, 16, 1024);
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
                const uint64_t kd = kdesc0 + (uint64_t)st * kStageStep;
                mma_ss_lead<0>(tmem + C::COL_S, qdesc, kd, C::IDESC_QK, leader);
#pragma unroll
                for (int kk = 1; kk < D / 16; ++kk)
                    mma_ss_lead<1>(tmem + C::COL_S, qdesc + kstep(kk, kRRows), kd + kstep(kk, kRBK), C::IDESC_QK,
                                   leader);
                tc_commit_lead(BAR_SF, leader);
                tc_commit_lead(BAR_KE(st), leader);
                return true;
            };
            bool go = issue_qk(0);
            if (go && leader) issued[2] = 1;
            for (int j = 0; go && j < n; ++j) {
                const int vs = j % C::STAGES;
                if (!mbar_wait_warp(BAR_PF, (uint32_t)j & 1, ctl)) break;
                if (!mbar_wait_warp(BAR_VF(vs), (uint32_t)(j / C::STAGES) & 1, ctl)) break;
                tc_fence_after();
                const uint64_t vd = vdesc0 + (uint64_t)vs * kStageStep;
                // O_full += P_full V (P_full: TMEM columns [0, 64) of S)
                if (j == 0) mma_ts_lead<0>(tmem + C::COL_OF, tmem + C::COL_S, vd, C::IDESC_PV, leader);
                else mma_ts_lead<1>(tmem + C::COL_OF, tmem + C::COL_S, vd, C::IDESC_PV, leader);
#pragma unroll
                for (int kk = 1; kk < kRBK / 16; ++kk)
                    mma_ts_lead<1>(tmem + C::COL_OF, tmem + C::COL_S + kk * 8,
                                   vd + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV, leader);
                // O_sp += P_sp V (P_sp: TMEM columns [64, 128))
                if (j == 0) mma_ts_lead<0>(tmem + C::COL_OS, tmem + C::COL_S + 64, vd, C::IDESC_PV, leader);
                else mma_ts_lead<1>(tmem + C::COL_OS, tmem + C::COL_S + 64, vd, C::IDESC_PV, leader);
#pragma unroll
                for (int kk = 1; kk < kRBK / 16; ++kk)
                    mma_ts_lead<1>(tmem + C::COL_OS, tmem + C::COL_S + 64 + kk * 8,
                                   vd + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV, leader);
                // O_tm += P_tm V (P_tm in shared memory, K-major, swizzled)
                if (j == 0) mma_ss_lead<0>(tmem + C::COL_OT, pdesc, vd, C::IDESC_PV, leader);
                else mma_ss_lead<1>(tmem + C::COL_OT, pdesc, vd, C::IDESC_PV, leader);
#pragma unroll
                for (int kk = 1; kk < kRBK / 16; ++kk)
                    mma_ss_lead<1>(tmem + C::COL_OT, pdesc + kstep(kk, kRRows),
                                   vd + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV, leader);
                tc_commit_lead(BAR_PV, leader);
                tc_commit_lead(BAR_VE(vs), leader);
                // the next S overwrites P_full / P_sp: queued behind the PV MMAs
                if (j + 1 < n) go = issue_qk(j + 1);
            }
        }
    } else if (warp < 4) {
        // ---------------- softmax: thread r owns sampled row r ----------------
        const int r = threadIdx.x;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t tS = tmem + lane_off + C::COL_S;
        int tok = __ldg(P.rows + min(rt * kRRows + r, P.R - 1));
        if (tok < 0 || tok >= P.N) tok = 0;              // flagged by the gather
        const int HW = P.H * P.W;
        const int tq = tok / HW, hq = (tok % HW) / P.W, wq = tok % P.W;
        const vsa_mask_spec ms = P.cand[head];
        const vsa_mask_spec mt = P.cand[P.heads + head];
        const float sl = P.scale_log2;
        const unsigned long long sl2 = f2_pack(sl, sl);
        float m_run = -INFINITY;                          // log2 units, shared by the three softmaxes
        float lf = 0.0f, ls = 0.0f, lt = 0.0f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const long long k0 = (long long)(j0 + j) * kRBK;
            uint32_t bsp[kRBK / 32], btm[kRBK / 32];
            route_row_bits(ms, mt, P.T, P.H, P.W, P.N, tq, hq, wq, k0, bsp, btm);
            if (!mbar_wait_warp(BAR_SF, (uint32_t)j & 1, ctl)) { ok = false; break; }
            tc_fence_after();
            float s[kRBK];
            {
                uint32_t sr[kRBK];
#pragma unroll
                for (int c = 0; c < kRBK / 32; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < kRBK; ++c) {
                    reg_fence(sr[c]);
                    s[c] = __uint_as_float(sr[c]);
                }
            }
            const long long left = (long long)P.N - k0;
            if (left < kRBK) {
#pragma unroll
                for (int c = 0; c < kRBK; ++c)
                    if (c >= left) s[c] = -INFINITY;
            }
            float mc[kRBK / 32];
#pragma unroll
            for (int g = 0; g < kRBK / 32; ++g) {
                float a = s[g * 32];
#pragma unroll
                for (int c = 1; c < 31; c += 2) a = max3(a, s[g * 32 + c], s[g * 32 + c + 1]);
                mc[g] = fmaxf(a, s[g * 32 + 31]);
            }
            float mx = mc[0];
#pragma unroll
            for (int g = 1; g < kRBK / 32; ++g) mx = fmaxf(mx, mc[g]);
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
            // S_j complete implies the PV MMAs of tile j-1 are complete (one
            // thread issues them in order), so O and P_tm may be touched now
            if (__any_sync(0xFFFFFFFFu, need_o)) {
#pragma unroll 1
                for (int c = 0; c < 3 * D / 32; ++c) {
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
#pragma unroll
            for (int cc = 0; cc < kRBK / 32; ++cc) {
                uint32_t pf[16], ps[16], pt[16];
                const uint32_t ws = bsp[cc], wt = btm[cc];
                float af = 0.0f, as = 0.0f, at = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(s[cc * 32 + 2 * i], s[cc * 32 + 2 * i + 1]), sl2, mneg2), x0, x1);
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    const float s0 = ((ws >> (2 * i)) & 1u) ? p0 : 0.0f;
                    const float s1 = ((ws >> (2 * i + 1)) & 1u) ? p1 : 0.0f;
                    const float t0 = ((wt >> (2 * i)) & 1u) ? p0 : 0.0f;
                    const float t1 = ((wt >> (2 * i + 1)) & 1u) ? p1 : 0.0f;
                    af += p0 + p1;
                    as += s0 + s1;
                    at += t0 + t1;
                    pf[i] = pack_bf16(p0, p1);
                    ps[i] = pack_bf16(s0, s1);
                    pt[i] = pack_bf16(t0, t1);
                }
                lf += af;
                ls += as;
                lt += at;
                tmem_st16(tS + cc * 16, pf);              // P_full: S columns [0, 64)
                tmem_st16(tS + 64 + cc * 16, ps);         // P_sp:   S columns [64, 128)
                // P_tm keys [32cc, 32cc + 32): block cc/2, chunks 4(cc%2)..+3 of row r
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int chunk = (cc & 1) * 4 + u;
                    const uint32_t dst = s_base + C::OFF_P + (cc >> 1) * (kRRows * 128) + r * 128 +
                                         ((chunk ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pt[4 * u]),
                                 "r"(pt[4 * u + 1]), "r"(pt[4 * u + 2]), "r"(pt[4 * u + 3])
                                 : "memory");
                }
            }
            tmem_st_wait();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR_PF);
        }

        // ---------------- partial record of this CTA ----------------
        bool have = ok && mbar_wait_warp(BAR_PV, (uint32_t)(n - 1) & 1, ctl);
        tc_fence_after();
        float* rec = P.part + ((size_t)unit * P.S + split) * C::PART_FLOATS;
        rec[r] = have ? m_run : -INFINITY;
        rec[kRRows + r] = have ? lf : 0.0f;
        rec[2 * kRRows + r] = have ? ls : 0.0f;
        rec[3 * kRRows + r] = have ? lt : 0.0f;
        if (have) {
#pragma unroll 1
            for (int c = 0; c < 3 * D / 32; ++c) {
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

// Splits of the key range: fewest waves x tiles per CTA (+4 tiles of fixed
// cost for the gather and the ~200 KB partial record), the smaller split on a
// tie.
int choose_splits(long long units, int nK, int sms)
{
    int best = 1;
    long long best_cost = -1;
    const int smax = nK < kRMaxSplits ? nK : kRMaxSplits;
    for (int s = 1; s <= smax; ++s) {
        const long long waves = (units * s + sms - 1) / sms;
        const long long cost = waves * ((nK + s - 1) / s + 4);
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
    if ((long long)B * d.heads * d.N > 0x7FFFFFFFLL) return VSA_ERR_UNSUPPORTED;
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

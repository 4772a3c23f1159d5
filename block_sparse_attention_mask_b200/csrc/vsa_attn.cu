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
// One CTA = two consecutive 128-row query blocks X = 0, 1 of one (batch,
// head); 12 warps in three warpgroups:
//   warp 8      TMA producer: Q of both blocks once, then the K/V tiles of the
//               merged (sorted) union of the two blocks' kv-tile lists through
//               a STAGES-deep shared-memory ring; a tile both blocks list is
//               loaded once and used by both.
//   warp 9      MMA issuer (one thread): per block X, S_X = Q_X K^T into TMEM
//               and O_X += P_X V with P_X read from TMEM (kind::f16, fp32
//               accumulate).  Per block the order is PV(X, j-1), QK(X, j), so
//               the tensor core alternates between the blocks while each
//               block's softmax runs (ping-pong); tcgen05.commit signals the
//               mbarriers.
//   warps 10-11 idle (they complete the third warpgroup).
//   warps 0..3  softmax of block 0, warps 4..7 softmax of block 1: thread r
//               owns query row r (TMEM lane r).  It loads S, applies the
//               boundary mask on boundary tiles, keeps the running max (log2
//               units; O rescaled in TMEM only when the max grows by more than
//               8, a factor 256) and sum in fp32, and writes P as bf16 over S
//               in 32-column chunks; at the end it normalises O and writes o
//               and lse.
// Registers: launched at 168 per thread (384 x 168); the producer/MMA
// warpgroup gives back down to 56 and the two softmax warpgroups take 224 each
// (2 x 128 x 224 + 128 x 56 = 384 x 168), checked on the host before launch.
// Every mbarrier wait is bounded: on expiry the CTA records VSA_DEV_TIMEOUT
// in the plan's status word, all roles leave their loops, TMEM is freed and
// the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstring>

#include "vsa_internal.h"

namespace {

constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;        // 65536 / 384, rounded down to a multiple of 8
constexpr int kSoftmaxRegs = 224;
constexpr int kControlRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kRows = VSA_EXEC_ROWS;              // 128 query rows per block
constexpr long long kWatchdogCycles = 1LL << 31;  // ~1 s at 2 GHz per wait
constexpr float kRescaleThreshold = 8.0f;         // log2 units

template <int D, int BK>
struct Cfg {
    static constexpr int Q_BYTES = kRows * D * 2;   // one query block
    static constexpr int KV_BYTES = BK * D * 2;
    static constexpr int STAGES = (2 * Q_BYTES + 4 * 2 * KV_BYTES <= 200 * 1024) ? 4
                                  : (2 * Q_BYTES + 3 * 2 * KV_BYTES <= 200 * 1024) ? 3 : 2;
    // TMEM: block X holds S_X (BK columns, P_X over its first BK/2) then O_X (D columns)
    static constexpr int SPAN = BK + D;
    static constexpr int TMEM_COLS = 2 * SPAN <= 256 ? 256 : 512;
    // shared memory map (offsets from a 1024-aligned base)
    static constexpr int OFF_Q = 0;                 // block X at OFF_Q + X * Q_BYTES
    static constexpr int OFF_K = 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
    // barriers: q_full[2], k_full[S], v_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2]
    static constexpr int NBAR = 2 + 3 * STAGES + 6;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;      // tmem addr (4) + abort (4)
    static constexpr int OFF_TAB = (OFF_MISC + 8 + 15) / 16 * 16;
    // instruction descriptors (kind::f16): D fp32, A and B bf16
    //   bits [4,6) D format = 1 (f32); [7,10) A = 1 (bf16); [10,13) B = 1 (bf16);
    //   bit 15 A major (0 = K); bit 16 B major (1 = MN); [17,23) N >> 3; [24,29) M >> 4
    static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) |
                                         ((uint32_t)(BK >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
};

struct AttnParams {
    CUtensorMap tm_q, tm_k, tm_v;       // 2D [rows = B*heads*n_slots, D] bf16, box {64, rows}
    __nv_bfloat16* o;
    float* lse;
    const int32_t* list_cnt;
    const int32_t* list;
    const int2* seg;
    const vsa_mask_spec* specs;
    const uint32_t* sbits;
    unsigned int* status;
    vsa_dims d;
    float scale_log2;
    int tab_words_s;                    // stripe offset table words in smem
    int tab_words_t;                    // stripe frame-offset table words in smem
};

// ---- PTX wrappers -------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

struct Ctl {
    volatile int* abort;
    unsigned int* status;
};

// Bounded wait for the phase of `bar` with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Ctl& c)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*c.abort) return false;
        if (clock64() - t0 > kWatchdogCycles) {
            atomicOr(c.status, VSA_DEV_TIMEOUT);
            *c.abort = 1;
            return false;
        }
    }
}

// Same, with the outcome made uniform across the warp (tcgen05.ld / st and
// __syncwarp after the wait need every lane on the same path).
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const Ctl& c)
{
    const bool ok = mbar_wait(bar, parity, c);
    return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"((unsigned long long)map), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

// 32 lanes x 32 columns of 32 bit: thread i of the warp gets lane (base + i), columns c..c+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Pin a register value after a tcgen05.wait so no use is scheduled before it.
__device__ __forceinline__ void reg_fence(uint32_t& x) { asm volatile("" : "+r"(x)); }

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Two fp32 lanes in one 64-bit register (packed f32x2 arithmetic).
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// tcgen05 shared-memory matrix descriptor, 128-byte swizzle (layout type 2),
// version 1, base offset 0.  Addresses and offsets in bytes.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Ordered union of two sorted kv-tile lists: each step yields the next kv
// tile and which of the two lists hold it (bit X).
struct ListMerge {
    const int32_t* L[2];
    int n[2];
    int i[2];
    __device__ __forceinline__ bool next(int& kv, int& mask)
    {
        const int a = i[0] < n[0] ? VSA_ENTRY_KV(__ldg(L[0] + i[0])) : INT_MAX;
        const int b = i[1] < n[1] ? VSA_ENTRY_KV(__ldg(L[1] + i[1])) : INT_MAX;
        if (a == INT_MAX && b == INT_MAX) return false;
        kv = a < b ? a : b;
        mask = (a == kv ? 1 : 0) | (b == kv ? 2 : 0);
        i[0] += mask & 1;
        i[1] += mask >> 1;
        return true;
    }
};

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams P)
{
    using C = Cfg<D, BK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

    const vsa_dims& d = P.d;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int npairs = (d.nE + 1) >> 1;
    const int pair = blockIdx.x % npairs;
    const int hb = blockIdx.x / npairs;                 // b * heads + head
    const int head = hb % d.heads;
    const long long base_row = (long long)hb * d.Nslots;
    int eX[2], cnt[2];
    const int32_t* list[2];
#pragma unroll
    for (int X = 0; X < 2; ++X) {
        eX[X] = 2 * pair + X;
        const bool present = eX[X] < d.nE;
        const int li = head * d.nE + (present ? eX[X] : 0);
        cnt[X] = present ? P.list_cnt[li] : 0;
        list[X] = P.list + (size_t)li * d.nK;
    }

    const uint32_t s_base = smem_addr(smem);
    const uint32_t bar0 = s_base + C::OFF_BAR;
    auto BAR_Q = [&](int X) { return bar0 + 8u * X; };
    auto BAR_KF = [&](int s) { return bar0 + 8u * (2 + s); };
    auto BAR_VF = [&](int s) { return bar0 + 8u * (2 + C::STAGES + s); };
    auto BAR_KE = [&](int s) { return bar0 + 8u * (2 + 2 * C::STAGES + s); };
    auto BAR_SF = [&](int X) { return bar0 + 8u * (2 + 3 * C::STAGES + X); };
    auto BAR_PF = [&](int X) { return bar0 + 8u * (4 + 3 * C::STAGES + X); };
    auto BAR_OF = [&](int X) { return bar0 + 8u * (6 + 3 * C::STAGES + X); };

    uint32_t* tmem_slot = (uint32_t*)(smem + C::OFF_MISC);
    volatile int* abort_flag = (volatile int*)(smem + C::OFF_MISC + 4);
    const Ctl ctl{abort_flag, P.status};

    if (threadIdx.x == 0) {
        for (int X = 0; X < 2; ++X) {
            mbar_init(BAR_Q(X), 1);
            mbar_init(BAR_SF(X), 1);
            mbar_init(BAR_PF(X), 4);
            mbar_init(BAR_OF(X), 1);
        }
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(BAR_KF(s), 1);
            mbar_init(BAR_VF(s), 1);
            mbar_init(BAR_KE(s), 1);
        }
        *abort_flag = 0;
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

    // Each role starts with its setmaxnreg; every warp of a warpgroup executes
    // the same one (warps 8..11 give registers back, warps 0..7 take them).
    if (warp == kProducerWarp) {
        // ---------------- TMA producer ----------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
        if (lane == 0) {
#pragma unroll
            for (int X = 0; X < 2; ++X) {
                if (cnt[X] == 0) continue;
                mbar_expect_tx(BAR_Q(X), C::Q_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + C::OFF_Q + X * C::Q_BYTES + c * kRows * 128, &P.tm_q, c * 64,
                                (int)(base_row + (long long)eX[X] * kRows), BAR_Q(X));
            }
            ListMerge mg{{list[0], list[1]}, {cnt[0], cnt[1]}, {0, 0}};
            int kv, mask;
            for (int u = 0; mg.next(kv, mask); ++u) {
                const int st = u % C::STAGES;
                const uint32_t use = (uint32_t)(u / C::STAGES);
                if (u >= C::STAGES && !mbar_wait(BAR_KE(st), (use - 1) & 1, ctl)) break;
                const int krow = (int)(base_row + (long long)kv * BK);
                mbar_expect_tx(BAR_KF(st), C::KV_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + C::OFF_K + st * C::KV_BYTES + c * BK * 128, &P.tm_k, c * 64, krow,
                                BAR_KF(st));
                mbar_expect_tx(BAR_VF(st), C::KV_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(s_base + C::OFF_V + st * C::KV_BYTES + c * BK * 128, &P.tm_v, c * 64, krow,
                                BAR_VF(st));
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
        bool ok = true;
        int pend_stage[2] = {-1, -1}, pend_item[2] = {0, 0}, nqk[2] = {0, 0}, npv[2] = {0, 0};
        uint32_t users = 0;                      // per stage: 2-bit count of blocks still to run PV
        bool qready[2] = {false, false};

        auto issue_pv = [&](int X) -> bool {
            const int st = pend_stage[X];
            if (!mbar_wait_warp(BAR_PF(X), (uint32_t)(nqk[X] - 1) & 1, ctl)) return false;
            if (!mbar_wait_warp(BAR_VF(st), (uint32_t)(pend_item[X] / C::STAGES) & 1, ctl)) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t aP = tmem + X * C::SPAN;
                const uint32_t dO = tmem + X * C::SPAN + BK;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t va = s_base + C::OFF_V + st * C::KV_BYTES + kk * 16 * 128;
                    mma_ts(dO, aP + kk * 8, smem_desc(va, BK * 128, 1024), C::IDESC_PV,
                           (nqk[X] > 1 || kk > 0) ? 1u : 0u);
                }
            }
            // O_X is complete after its last PV, wherever that PV is issued
            // (a block whose list ended can get its last PV from the
            // stage-release step below)
            if (++npv[X] == cnt[X] && lane == 0) tc_commit(BAR_OF(X));
            users -= 1u << (2 * st);
            if (((users >> (2 * st)) & 3u) == 0 && lane == 0) tc_commit(BAR_KE(st));
            __syncwarp();
            pend_stage[X] = -1;
            return true;
        };

        ListMerge mg{{list[0], list[1]}, {cnt[0], cnt[1]}, {0, 0}};
        int kv, mask;
        for (int u = 0; ok && mg.next(kv, mask); ++u) {
            const int st = u % C::STAGES;
            // PVs of the item that last used this stage must be issued before
            // its K/V can be replaced
#pragma unroll
            for (int X = 0; X < 2; ++X)
                if (ok && pend_stage[X] >= 0 && pend_item[X] <= u - C::STAGES) ok = issue_pv(X);
            bool kready = false;
#pragma unroll
            for (int X = 0; X < 2; ++X) {
                if (!ok || !((mask >> X) & 1)) continue;
                // S_X is overwritten by QK(X): its previous P must be consumed first
                if (pend_stage[X] >= 0) ok = issue_pv(X);
                if (ok && !qready[X]) ok = qready[X] = mbar_wait_warp(BAR_Q(X), 0, ctl);
                if (ok && !kready) {
                    ok = kready = mbar_wait_warp(BAR_KF(st), (uint32_t)(u / C::STAGES) & 1, ctl);
                    users |= (uint32_t)__popc(mask) << (2 * st);
                }
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t dS = tmem + X * C::SPAN;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t qa = s_base + C::OFF_Q + X * C::Q_BYTES + (kk >> 2) * (kRows * 128) +
                                            (kk & 3) * 32;
                        const uint32_t ka = s_base + C::OFF_K + st * C::KV_BYTES + (kk >> 2) * (BK * 128) +
                                            (kk & 3) * 32;
                        mma_ss(dS, smem_desc(qa, 16, 1024), smem_desc(ka, 16, 1024), C::IDESC_QK,
                               kk > 0 ? 1u : 0u);
                    }
                    tc_commit(BAR_SF(X));
                }
                __syncwarp();
                pend_stage[X] = st;
                pend_item[X] = u;
                ++nqk[X];
            }
        }
#pragma unroll
        for (int X = 0; X < 2; ++X)
            if (ok && pend_stage[X] >= 0) ok = issue_pv(X);
    } else if (warp < 8) {
        // ---------------- softmax: warps 4X .. 4X+3 own block X ----------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        const int X = warp >> 2;
        const int row = threadIdx.x & 127;                // TMEM lane
        const int half = row >> 6;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + X * C::SPAN;
        const uint32_t tO = tS + BK;
        const vsa_mask_spec m = P.specs[head];
        const int n = cnt[X];
        const vsa_row_ctx q = vsa_row_init(d, m, (long long)eX[X] * kRows + row);
        uint32_t* stab = (uint32_t*)(smem + C::OFF_TAB) + X * (P.tab_words_s + P.tab_words_t);
        uint32_t* ttab = stab + P.tab_words_s;
        if (m.kind == VSA_MASK_STRIPE) {
            const uint32_t* src = P.sbits + (size_t)head * d.sbits_words;
            for (int i = row; i < P.tab_words_s; i += kRows) stab[i] = src[i];
            for (int i = row; i < P.tab_words_t; i += kRows) ttab[i] = vsa_stripe_tword(m, d.T, i);
        }
        if (X == 0) asm volatile("bar.sync 1, 128;" ::: "memory");
        else asm volatile("bar.sync 2, 128;" ::: "memory");

        float m_run = -INFINITY;  // running max of scale*log2(e)*s
        float l_run = 0.0f;
        const float sl = P.scale_log2;
        const unsigned long long sl2 = f2_pack(sl, sl);
        bool ok = true;
        for (int j = 0; j < n && ok; ++j) {
            const int ent = __ldg(list[X] + j);
            const int cls = VSA_ENTRY_CLS(ent, half);
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
                const int kv = VSA_ENTRY_KV(ent);
                const int2* sg = P.seg + (size_t)kv * d.nseg;
                const int runs_per_word = 32 / d.bw;
#pragma unroll
                for (int wi = 0; wi < BK / 32; ++wi) {
                    uint32_t bits = 0;
                    for (int r = 0; r < runs_per_word; ++r) {
                        const int2 v = __ldg(sg + wi * runs_per_word + r);
                        const uint32_t rb = vsa_run_bits(m, d, q, stab, ttab, v.x & 0xFFFF, v.x >> 16,
                                                         v.y & 0xFFFF, v.y >> 16);
                        bits |= rb << (r * d.bw);
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (!((bits >> c) & 1u)) s[wi * 32 + c] = -INFINITY;
                }
            }

            if (cls == VSA_TILE_EMPTY) {
                uint32_t z[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
                for (int c = 0; c < BK / 32; ++c) tmem_st16(tS + c * 16, z);
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
                bool need_o = false;
                float alpha = 1.0f;
                if (mx != -INFINITY) {
                    if (m_run == -INFINITY) {
                        m_run = mxs;  // nothing accumulated for this row yet: O row is 0
                    } else if (mxs > m_run + kRescaleThreshold) {
                        alpha = ex2(m_run - mxs);
                        l_run *= alpha;
                        m_run = mxs;
                        need_o = true;
                    }
                }
                // O_X = P_X(<j) V is complete here: PV(X, j-1) was issued before
                // QK(X, j), whose completion the s_full wait observed
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
                const float mneg = (m_run == -INFINITY) ? 0.0f : -m_run;
                const unsigned long long mneg2 = f2_pack(mneg, mneg);
                unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int c = 0; c < BK / 32; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int k = c * 32 + 2 * i;
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(s[k], s[k + 1]), sl2, mneg2), x0, x1);
                        const float p0 = ex2(x0), p1 = ex2(x1);
                        acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
                        pk[i] = pack_bf16(p0, p1);
                    }
                    // P chunk c over S columns [16c, 16c+16): two bf16 per column
                    tmem_st16(tS + c * 16, pk);
                }
                float a0, a1, a2, a3, a4, a5, a6, a7;
                f2_unpack(acc[0], a0, a1);
                f2_unpack(acc[1], a2, a3);
                f2_unpack(acc[2], a4, a5);
                f2_unpack(acc[3], a6, a7);
                l_run += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR_PF(X));
        }

        // ---------------- epilogue ----------------
        if (eX[X] < d.nE) {
            const long long orow = base_row + (long long)eX[X] * kRows + row;
            bool have_o = ok && n > 0;
            if (have_o) {
                have_o = mbar_wait_warp(BAR_OF(X), 0, ctl);
                tc_fence_after();
            }
            uint4* optr = reinterpret_cast<uint4*>(P.o + orow * D);
            if (have_o) {
                const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
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
    } else {
        // warps 10, 11: no work, but they belong to the control warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
    }
}

// ---- host side ----------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
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

bool make_map(CUtensorMap* m, const void* base, long long rows, int D, int box_rows)
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

template <int D, int BK>
int launch_attn(AttnParams& P, int B, cudaStream_t s)
{
    using C = Cfg<D, BK>;
    const int smem = 1024 + C::OFF_TAB + 2 * 4 * (P.tab_words_s + P.tab_words_t);
    if (smem > 227 * 1024) return VSA_ERR_UNSUPPORTED;
    auto kern = attn_fwd_kernel<D, BK>;
    // the setmaxnreg split assumes exactly kLaunchRegs registers per thread at launch
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return VSA_ERR_CUDA;
    if (fa.numRegs != kLaunchRegs) return VSA_ERR_DEVICE;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return VSA_ERR_CUDA;
    const long long grid = (long long)((P.d.nE + 1) / 2) * P.d.heads * B;
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
    if (!make_map(&P.tm_q, q, rows, D, kRows) || !make_map(&P.tm_k, k, rows, D, d.Bk) ||
        !make_map(&P.tm_v, v, rows, D, d.Bk))
        return VSA_ERR_CUDA;
    P.o = (__nv_bfloat16*)o;
    P.lse = lse;
    P.list_cnt = plan->d_list_cnt;
    P.list = plan->d_list;
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

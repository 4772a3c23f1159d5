// Head-sharded attention across GPUs: the sequence-to-head exchange fused with
// each head's token order, and its inverse.
//
// Inputs arrive sequence-sharded, rank r holding the natural tokens
// [off_r, off_{r+1}) of every head, off_r = floor(r N / world), as
// [B][n_r][world*heads][D]; an all-to-all gives each rank every token of its
// heads ("Sparse VideoGen: accelerating video diffusion attention on TPU",
// "performing layout transformation on local heads": [B,S/N,H,D] becomes
// [B,S,H/N,D]).  The pages permute a head's tokens only after that exchange,
// where all of them are local; here the two are one pass: rank r writes each
// of its (token, head) rows straight into the owning rank's tile-major (or
// frame-0-first) buffer at the token's slot, through that rank's memory
// (peer stores over NVLink; the same kernel on one GPU when every buffer is
// local).  The inverse reads a rank's output rows at their slots and writes
// them into the token owners' [B][n_r][world*heads][D] shards.
//
// The kernels only load and store: they wait on no other rank.  The caller
// orders them against the other ranks (a collective after each exchange) so
// that every rank's stores are complete before any rank reads its buffer.
// Each thread ends with a system-scope fence so its peer stores are ordered
// before that collective.
#include <cuda_runtime.h>

#include "vsa_internal.h"

namespace {

constexpr int kMaxWorld = 8;

struct PeerPtrs {
    uint4* p[kMaxWorld];
};

// dst.p[g] without a dynamically indexed (local-memory) copy of the table
__device__ __forceinline__ uint4* peer(const PeerPtrs& t, int g)
{
    uint4* q = t.p[0];
#pragma unroll
    for (int i = 1; i < kMaxWorld; ++i) q = (g == i) ? t.p[i] : q;
    return q;
}

__device__ __forceinline__ long long shard_off(long long N, int world, int r) { return (long long)r * N / world; }

// Natural token n -> slot in a head of the given layout.
__device__ __forceinline__ long long token_slot(const vsa_dims& d, int layout, long long n)
{
    const int HW = d.H * d.W;
    const int t = (int)(n / HW);
    const int rem = (int)(n - (long long)t * HW);
    const int h = rem / d.W, w = rem - (rem / d.W) * d.W;
    return layout == VSA_LAYOUT_FRAME0_FIRST ? vsa_token_slot_f0(d, t, h, w) : vsa_token_slot(d, t, h, w);
}

// Rank `rank`'s shard x [B][n_r][world*heads][D] -> every rank g's buffer
// dst[g] [B][heads][n_slots][D]; then zeros into the padding slots of this
// rank's own buffer (no token maps there).
template <int D>
__global__ void __launch_bounds__(256) ulysses_permute_kernel(vsa_dims d, const int32_t* __restrict__ layout,
                                                              int B, int rank, int world,
                                                              const uint4* __restrict__ x, PeerPtrs dst)
{
    constexpr int VPR = D * 2 / 16;   // 16-byte vectors per row
    constexpr int RPW = 32 / VPR;     // rows per warp step
    const int lane = threadIdx.x & 31;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int sub = lane / VPR, v = lane % VPR;
    const int htot = world * d.heads;
    const long long off = shard_off(d.N, world, rank);
    const long long n_r = shard_off(d.N, world, rank + 1) - off;
    const long long rows = (long long)B * n_r * htot;
    for (long long r = warp * RPW + sub; r < rows; r += nwarps * RPW) {
        const int hg = (int)(r % htot);
        const long long bs = r / htot;
        const long long s = bs % n_r;
        const long long b = bs / n_r;
        const int g = hg / d.heads, hl = hg - g * d.heads;
        const long long p = token_slot(d, __ldg(layout + hg), off + s);
        peer(dst, g)[((b * d.heads + hl) * d.Nslots + p) * VPR + v] = __ldg(x + r * VPR + v);
    }
    // padding slots of this rank's heads
    const long long prow = (long long)B * d.heads * d.Nslots;
    for (long long r = warp * RPW + sub; r < prow; r += nwarps * RPW) {
        const long long bh = r / d.Nslots;
        const long long p = r - bh * d.Nslots;
        const int hg = rank * d.heads + (int)(bh % d.heads);
        int t, h, w;
        if (!vsa_slot_coords_any(d, __ldg(layout + hg), p, t, h, w)) peer(dst, rank)[r * VPR + v] = make_uint4(0u, 0u, 0u, 0u);
    }
    __threadfence_system();
}

// Rank `rank`'s output o [B][heads][n_slots][D] -> the token owners' shards
// dst[r] [B][n_r][world*heads][D].
template <int D>
__global__ void __launch_bounds__(256) ulysses_unpermute_kernel(vsa_dims d, const int32_t* __restrict__ layout,
                                                                int B, int rank, int world,
                                                                const uint4* __restrict__ o, PeerPtrs dst)
{
    constexpr int VPR = D * 2 / 16;
    constexpr int RPW = 32 / VPR;
    const int lane = threadIdx.x & 31;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int sub = lane / VPR, v = lane % VPR;
    const int htot = world * d.heads;
    const long long rows = (long long)B * d.heads * d.N;
    for (long long r = warp * RPW + sub; r < rows; r += nwarps * RPW) {
        const long long bh = r / d.N;
        const long long n = r - bh * d.N;
        const int hl = (int)(bh % d.heads);
        const long long b = bh / d.heads;
        const int hg = rank * d.heads + hl;
        const long long p = token_slot(d, __ldg(layout + hg), n);
        // owner of token n: the last rank whose shard starts at or before n
        int own = (int)(n * world / d.N);
        while (own + 1 < world && shard_off(d.N, world, own + 1) <= n) ++own;
        while (own > 0 && shard_off(d.N, world, own) > n) --own;
        const long long off = shard_off(d.N, world, own);
        const long long n_own = shard_off(d.N, world, own + 1) - off;
        peer(dst, own)[((b * n_own + (n - off)) * htot + hg) * VPR + v] = __ldg(o + (bh * d.Nslots + p) * VPR + v);
    }
    __threadfence_system();
}

int sm_count_u()
{
    static int cached = 0;
    if (!cached) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&cached, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) cached = 148;
    }
    return cached;
}

int launch_exchange(bool forward, vsa_plan_t plan, const void* src, int B, int D, int rank, int world,
                    const int32_t* layout, void* const* dst, void* stream)
{
    if (!plan || B < 0 || world < 1 || world > kMaxWorld || rank < 0 || rank >= world) return VSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
    if (B == 0) return VSA_OK;
    if (!src || !layout || !dst) return VSA_ERR_INVALID_ARG;
    const vsa_dims& d = plan->d;
    if (d.N < world) return VSA_ERR_INVALID_ARG;
    PeerPtrs pp;
    for (int g = 0; g < kMaxWorld; ++g) pp.p[g] = nullptr;
    for (int g = 0; g < world; ++g) {
        if (!dst[g]) return VSA_ERR_INVALID_ARG;
        if (!vsa_aligned16(dst[g])) return VSA_ERR_ALIGNMENT;
        pp.p[g] = (uint4*)dst[g];
    }
    if (!vsa_aligned16(src) || ((uintptr_t)layout & 3u)) return VSA_ERR_ALIGNMENT;
    const long long rows = forward ? (long long)B * (d.N / world + 1) * world * d.heads : (long long)B * d.heads * d.N;
    const int threads = 256;
    const long long want = (rows * (D * 2 / 16) + threads - 1) / threads;
    const long long cap = (long long)sm_count_u() * 8;
    const unsigned grid = (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
    cudaStream_t s = (cudaStream_t)stream;
    if (forward) {
        if (D == 128)
            ulysses_permute_kernel<128><<<grid, threads, 0, s>>>(d, layout, B, rank, world, (const uint4*)src, pp);
        else
            ulysses_permute_kernel<64><<<grid, threads, 0, s>>>(d, layout, B, rank, world, (const uint4*)src, pp);
    } else {
        if (D == 128)
            ulysses_unpermute_kernel<128><<<grid, threads, 0, s>>>(d, layout, B, rank, world, (const uint4*)src, pp);
        else
            ulysses_unpermute_kernel<64><<<grid, threads, 0, s>>>(d, layout, B, rank, world, (const uint4*)src, pp);
    }
    return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace

extern "C" int vsa_ulysses_permute(vsa_plan_t plan, const void* x, int B, int D, int rank, int world,
                                   const int32_t* head_layout, void* const* dst, void* stream)
{
    return launch_exchange(true, plan, x, B, D, rank, world, head_layout, dst, stream);
}

extern "C" int vsa_ulysses_unpermute(vsa_plan_t plan, const void* o, int B, int D, int rank, int world,
                                     const int32_t* head_layout, void* const* dst, void* stream)
{
    return launch_exchange(false, plan, o, B, D, rank, world, head_layout, dst, stream);
}

// Token permutation between the natural (t,h,w) order and each head's layout:
// the tile-major order of 3D units with zero padding ("Video diffusion
// long-sequence attention and sparsity", section 7.2: the permutation is one
// [N, d] gather; "Parameterized Stripe Attention", key design 2: hierarchical
// layout with 3D padding), or the frame-0-first position-major order of
// temporal heads ("Sparse VideoGen: accelerating video diffusion attention on
// TPU", "arranging tokens for efficient temporal access").  HBM-bound copies: the
// plan's lookup tables give each slot's token (and each token's slot) in both
// orders, and every row of D bf16 values moves as 16-byte
// vectors, a warp covers 2 rows (D = 128) or 4 rows (D = 64) per step, and
// the grid is a multiple of the SM count with a grid-stride loop.
#include <cuda_runtime.h>

#include "vsa_internal.h"

namespace {

template <int D>
__global__ void __launch_bounds__(256) permute_kernel(vsa_dims d, const vsa_mask_spec* __restrict__ specs,
                                                      const int32_t* __restrict__ s2t, long long rows,
                                                      const uint4* __restrict__ in, uint4* __restrict__ out)
{
    constexpr int VPR = D * 2 / 16;   // 16-byte vectors per row
    constexpr int RPW = 32 / VPR;     // rows per warp step
    const int lane = threadIdx.x & 31;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int sub = lane / VPR, v = lane % VPR;
    for (long long r = warp * RPW + sub; r < rows; r += nwarps * RPW) {
        const long long bh = r / d.Nslots;
        const long long p = r - bh * d.Nslots;
        const int layout = __ldg(&specs[bh % d.heads].layout);
        const int n = __ldg(s2t + layout * d.Nslots + p);
        out[r * VPR + v] = n >= 0 ? __ldg(in + (bh * d.N + n) * VPR + v) : make_uint4(0u, 0u, 0u, 0u);
    }
}

template <int D>
__global__ void __launch_bounds__(256) unpermute_kernel(vsa_dims d, const vsa_mask_spec* __restrict__ specs,
                                                        const int32_t* __restrict__ t2s, long long rows,
                                                        const uint4* __restrict__ in, uint4* __restrict__ out)
{
    constexpr int VPR = D * 2 / 16;
    constexpr int RPW = 32 / VPR;
    const int lane = threadIdx.x & 31;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int sub = lane / VPR, v = lane % VPR;
    const long long stride = nwarps * RPW;
    // two rows per thread in flight: both loads are issued before the stores
    for (long long r0 = warp * RPW + sub; r0 < rows; r0 += 2 * stride) {
        uint4 val[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const long long r = r0 + u * stride;
            if (r < rows) {
                const long long bh = r / d.N;
                const long long n = r - bh * d.N;
                const int layout = __ldg(&specs[bh % d.heads].layout);
                const long long p = __ldg(t2s + layout * d.N + n);
                val[u] = __ldg(in + (bh * d.Nslots + p) * VPR + v);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const long long r = r0 + u * stride;
            if (r < rows) out[r * VPR + v] = val[u];
        }
    }
}

// q, k and v in one pass: one slot -> token lookup per row serves the three
// tensors, and each thread keeps six 16-byte loads (two rows of each tensor)
// in flight before its stores.
template <int D>
__global__ void __launch_bounds__(256) permute3_kernel(vsa_dims d, const vsa_mask_spec* __restrict__ specs,
                                                       const int32_t* __restrict__ s2t,
                                                       long long rows, const uint4* __restrict__ q,
                                                       const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                       uint4* __restrict__ qo, uint4* __restrict__ ko,
                                                       uint4* __restrict__ vo)
{
    constexpr int VPR = D * 2 / 16;
    constexpr int RPW = 32 / VPR;
    const int lane = threadIdx.x & 31;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int sub = lane / VPR, c = lane % VPR;
    const long long stride = nwarps * RPW;
    for (long long r0 = warp * RPW + sub; r0 < rows; r0 += 2 * stride) {
        long long src[2];
        bool real[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const long long r = r0 + u * stride;
            real[u] = false;
            src[u] = 0;
            if (r < rows) {
                const long long bh = r / d.Nslots;
                const long long p = r - bh * d.Nslots;
                const int layout = __ldg(&specs[bh % d.heads].layout);
                const int n = __ldg(s2t + layout * d.Nslots + p);
                if (n >= 0) {
                    real[u] = true;
                    src[u] = (bh * d.N + n) * VPR + c;
                }
            }
        }
        uint4 a[2], b[2], e[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            a[u] = real[u] ? __ldg(q + src[u]) : z;
            b[u] = real[u] ? __ldg(k + src[u]) : z;
            e[u] = real[u] ? __ldg(v + src[u]) : z;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const long long r = r0 + u * stride;
            if (r < rows) {
                qo[r * VPR + c] = a[u];
                ko[r * VPR + c] = b[u];
                vo[r * VPR + c] = e[u];
            }
        }
    }
}

int sm_count()
{
    static int cached = 0;
    if (!cached) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&cached, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            cached = 148;
    }
    return cached;
}

int launch(bool forward, vsa_plan_t plan, const void* in, void* out, int B, int D, void* stream)
{
    if (!plan || B < 0) return VSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
    if (B == 0) return VSA_OK;
    if (!in || !out) return VSA_ERR_INVALID_ARG;
    if (!vsa_aligned16(in) || !vsa_aligned16(out)) return VSA_ERR_ALIGNMENT;
    const vsa_dims& d = plan->d;
    const long long rows = (long long)B * d.heads * (forward ? d.Nslots : d.N);
    const long long in_rows = (long long)B * d.heads * (forward ? d.N : d.Nslots);
    const size_t row_bytes = (size_t)D * 2;
    const char* ib = (const char*)in;
    const char* ob = (const char*)out;
    if (ib < ob + rows * row_bytes && ob < ib + in_rows * row_bytes) return VSA_ERR_INVALID_ARG;
    const int threads = 256;
    const long long want = (rows * (D * 2 / 16) + threads - 1) / threads;
    const long long cap = (long long)sm_count() * 8;
    const unsigned grid = (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
    cudaStream_t s = (cudaStream_t)stream;
    if (forward) {
        if (D == 128) permute_kernel<128><<<grid, threads, 0, s>>>(d, plan->d_specs, plan->d_slot2tok, rows, (const uint4*)in, (uint4*)out);
        else permute_kernel<64><<<grid, threads, 0, s>>>(d, plan->d_specs, plan->d_slot2tok, rows, (const uint4*)in, (uint4*)out);
    } else {
        if (D == 128) unpermute_kernel<128><<<grid, threads, 0, s>>>(d, plan->d_specs, plan->d_tok2slot, rows, (const uint4*)in, (uint4*)out);
        else unpermute_kernel<64><<<grid, threads, 0, s>>>(d, plan->d_specs, plan->d_tok2slot, rows, (const uint4*)in, (uint4*)out);
    }
    return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace

extern "C" int vsa_permute(vsa_plan_t plan, const void* in, void* out, int B, int D, void* stream)
{
    return launch(true, plan, in, out, B, D, stream);
}

extern "C" int vsa_unpermute(vsa_plan_t plan, const void* in, void* out, int B, int D, void* stream)
{
    return launch(false, plan, in, out, B, D, stream);
}

extern "C" int vsa_permute_qkv(vsa_plan_t plan, const void* q, const void* k, const void* v, void* q_out,
                               void* k_out, void* v_out, int B, int D, void* stream)
{
    if (!plan || B < 0) return VSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
    if (B == 0) return VSA_OK;
    const void* ins[3] = {q, k, v};
    void* outs[3] = {q_out, k_out, v_out};
    const vsa_dims& d = plan->d;
    const long long rows = (long long)B * d.heads * d.Nslots;
    const long long in_rows = (long long)B * d.heads * d.N;
    const size_t row_bytes = (size_t)D * 2;
    for (int i = 0; i < 3; ++i) {
        if (!ins[i] || !outs[i]) return VSA_ERR_INVALID_ARG;
        if (!vsa_aligned16(ins[i]) || !vsa_aligned16(outs[i])) return VSA_ERR_ALIGNMENT;
    }
    // no output may overlap an input or another output
    for (int i = 0; i < 3; ++i)
        for (int j = 0; j < 3; ++j) {
            const char* ib = (const char*)ins[j];
            const char* ob = (const char*)outs[i];
            if (ib < ob + rows * row_bytes && ob < ib + in_rows * row_bytes) return VSA_ERR_INVALID_ARG;
            if (i != j) {
                const char* o2 = (const char*)outs[j];
                if (o2 < ob + rows * row_bytes && ob < o2 + rows * row_bytes) return VSA_ERR_INVALID_ARG;
            }
        }
    const int threads = 256;
    const long long want = (rows * (D * 2 / 16) / 2 + threads - 1) / threads;
    const long long cap = (long long)sm_count() * 8;
    const unsigned grid = (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
    cudaStream_t s = (cudaStream_t)stream;
    if (D == 128)
        permute3_kernel<128><<<grid, threads, 0, s>>>(d, plan->d_specs, plan->d_slot2tok, rows, (const uint4*)q, (const uint4*)k,
                                                      (const uint4*)v, (uint4*)q_out, (uint4*)k_out, (uint4*)v_out);
    else
        permute3_kernel<64><<<grid, threads, 0, s>>>(d, plan->d_specs, plan->d_slot2tok, rows, (const uint4*)q, (const uint4*)k,
                                                     (const uint4*)v, (uint4*)q_out, (uint4*)k_out, (uint4*)v_out);
    return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

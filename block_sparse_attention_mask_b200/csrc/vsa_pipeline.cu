// Host-buffer attention with the copies overlapped: the (batch, head) pairs
// are cut into chunks of a few heads; chunk c's host-to-device copies, its
// plan rebuild + permute + attention + unpermute, and its device-to-host
// copies run on three streams, so that while chunk c computes, chunk c+1's
// inputs are in flight over PCIe and chunk c-1's outputs come back.  Two
// sets of device staging buffers alternate between chunks; events order
// every reuse.  The kernels are the plan's own: each chunk of heads has its
// own plan (the specs of those heads), and its tensors are contiguous slices
// of the [B][heads][...] host arrays.
//
// Chunks run in decreasing order of executed tile steps.  Every chunk of a
// full size moves the same bytes over PCIe, so with copy-in and compute as a
// two-stage flow shop, heaviest compute first is Johnson's rule: the chunks
// whose compute outlasts their copy go while later copies are still coming,
// and the chunk left to compute after the last copy is the lightest.
#include <cuda_runtime.h>

#include <cstring>
#include <new>

#include "vsa_internal.h"

namespace {

constexpr int kSets = 2;

struct Staging {
    void *q, *k, *v;          // natural [nh][N][D]
    void *qp, *kp, *vp, *op;  // tile-major [nh][n_slots][D]
    void* o;                  // natural [nh][N][D]
    float* lse;               // [nh][n_slots]
    cudaEvent_t in_free, out_ready, out_free, in_ready;
};

}  // namespace

struct vsa_pipeline_s {
    int device;
    int B, D, heads, chunk, nchunks_h;
    long long N, Nslots;
    vsa_plan_t* plans;        // one per head chunk
    int* chunk_heads;         // heads in each head chunk
    int* order;               // head chunks in issue order
    Staging set[kSets];
    cudaStream_t s_h2d, s_comp, s_d2h;
    cudaEvent_t start, done;
};

namespace {

void destroy_pipeline(vsa_pipeline_s* p)
{
    if (!p) return;
    for (int i = 0; i < kSets; ++i) {
        Staging& st = p->set[i];
        cudaFree(st.q);
        cudaFree(st.k);
        cudaFree(st.v);
        cudaFree(st.qp);
        cudaFree(st.kp);
        cudaFree(st.vp);
        cudaFree(st.op);
        cudaFree(st.o);
        cudaFree(st.lse);
        if (st.in_free) cudaEventDestroy(st.in_free);
        if (st.out_ready) cudaEventDestroy(st.out_ready);
        if (st.out_free) cudaEventDestroy(st.out_free);
        if (st.in_ready) cudaEventDestroy(st.in_ready);
    }
    if (p->plans)
        for (int c = 0; c < p->nchunks_h; ++c)
            if (p->plans[c]) vsa_plan_destroy(p->plans[c]);
    delete[] p->plans;
    delete[] p->chunk_heads;
    delete[] p->order;
    if (p->s_h2d) cudaStreamDestroy(p->s_h2d);
    if (p->s_comp) cudaStreamDestroy(p->s_comp);
    if (p->s_d2h) cudaStreamDestroy(p->s_d2h);
    if (p->start) cudaEventDestroy(p->start);
    if (p->done) cudaEventDestroy(p->done);
    delete p;
}

}  // namespace

extern "C" int vsa_pipeline_create(const vsa_mask_spec* specs, int num_heads, int T, int H, int W, int bt, int bh,
                                   int bw, int q_tile, int kv_tile, int B, int D, int chunk_heads,
                                   vsa_pipeline_t* out)
{
    if (!out) return VSA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!specs || num_heads < 1 || B < 1 || chunk_heads < 1) return VSA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return VSA_ERR_UNSUPPORTED;
    vsa_pipeline_s* p = new (std::nothrow) vsa_pipeline_s;
    if (!p) return VSA_ERR_OOM;
    memset(p, 0, sizeof *p);
    p->B = B;
    p->D = D;
    p->heads = num_heads;
    p->chunk = chunk_heads < num_heads ? chunk_heads : num_heads;
    p->nchunks_h = (num_heads + p->chunk - 1) / p->chunk;
    if (cudaGetDevice(&p->device) != cudaSuccess) {
        delete p;
        return VSA_ERR_CUDA;
    }
    p->plans = new (std::nothrow) vsa_plan_t[p->nchunks_h]();
    p->chunk_heads = new (std::nothrow) int[p->nchunks_h]();
    p->order = new (std::nothrow) int[p->nchunks_h]();
    long long* work = new (std::nothrow) long long[p->nchunks_h]();
    int64_t* steps = new (std::nothrow) int64_t[p->chunk]();
    if (!p->plans || !p->chunk_heads || !p->order || !work || !steps) {
        delete[] work;
        delete[] steps;
        destroy_pipeline(p);
        return VSA_ERR_OOM;
    }
    for (int c = 0; c < p->nchunks_h; ++c) {
        const int h0 = c * p->chunk;
        const int nh = (h0 + p->chunk <= num_heads) ? p->chunk : num_heads - h0;
        p->chunk_heads[c] = nh;
        int r = vsa_plan_create(specs + h0, nh, T, H, W, bt, bh, bw, q_tile, kv_tile, nullptr, &p->plans[c]);
        if (r == VSA_OK) r = vsa_plan_exec_steps(p->plans[c], steps, (size_t)nh, nullptr);
        if (r != VSA_OK) {
            delete[] work;
            delete[] steps;
            destroy_pipeline(p);
            return r;
        }
        for (int i = 0; i < nh; ++i) work[c] += steps[i];
        // insertion by decreasing work; equal work keeps head order
        int at = c;
        while (at > 0 && work[p->order[at - 1]] < work[c]) {
            p->order[at] = p->order[at - 1];
            --at;
        }
        p->order[at] = c;
    }
    delete[] work;
    delete[] steps;
    p->N = p->plans[0]->d.N;
    p->Nslots = p->plans[0]->d.Nslots;
    const size_t nat = (size_t)p->chunk * p->N * D * 2, tm = (size_t)p->chunk * p->Nslots * D * 2;
    bool ok = cudaStreamCreateWithFlags(&p->s_h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p->s_comp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p->s_d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p->start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&p->done, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < kSets; ++i) {
        Staging& st = p->set[i];
        ok = cudaMalloc(&st.q, nat) == cudaSuccess && cudaMalloc(&st.k, nat) == cudaSuccess &&
             cudaMalloc(&st.v, nat) == cudaSuccess && cudaMalloc(&st.qp, tm) == cudaSuccess &&
             cudaMalloc(&st.kp, tm) == cudaSuccess && cudaMalloc(&st.vp, tm) == cudaSuccess &&
             cudaMalloc(&st.op, tm) == cudaSuccess && cudaMalloc(&st.o, nat) == cudaSuccess &&
             cudaMalloc(&st.lse, (size_t)p->chunk * p->Nslots * sizeof(float)) == cudaSuccess &&
             cudaEventCreateWithFlags(&st.in_free, cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&st.out_ready, cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&st.out_free, cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&st.in_ready, cudaEventDisableTiming) == cudaSuccess;
    }
    if (!ok) {
        cudaGetLastError();
        destroy_pipeline(p);
        return VSA_ERR_OOM;
    }
    // the staging sets start free: record every event once
    for (int i = 0; i < kSets; ++i) {
        cudaEventRecord(p->set[i].in_free, p->s_comp);
        cudaEventRecord(p->set[i].out_free, p->s_d2h);
    }
    if (cudaStreamSynchronize(p->s_comp) != cudaSuccess || cudaStreamSynchronize(p->s_d2h) != cudaSuccess) {
        destroy_pipeline(p);
        return VSA_ERR_CUDA;
    }
    *out = p;
    return VSA_OK;
}

extern "C" int vsa_pipeline_run(vsa_pipeline_t p, const void* q_host, const void* k_host, const void* v_host,
                                void* o_host, float* lse_host, float scale, void* stream)
{
    if (!p || !q_host || !k_host || !v_host || !o_host || !lse_host) return VSA_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || !(scale < 1e30f)) return VSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const int D = p->D;
    const size_t row = (size_t)D * 2;
    // the caller's earlier work on `stream` comes first
    VSA_CUDA_TRY(cudaEventRecord(p->start, s));
    VSA_CUDA_TRY(cudaStreamWaitEvent(p->s_h2d, p->start, 0));
    VSA_CUDA_TRY(cudaStreamWaitEvent(p->s_comp, p->start, 0));
    VSA_CUDA_TRY(cudaStreamWaitEvent(p->s_d2h, p->start, 0));
    int c = 0;
    for (int b = 0; b < p->B; ++b)
        for (int i = 0; i < p->nchunks_h; ++i, ++c) {
            const int hc = p->order[i];
            Staging& st = p->set[c % kSets];
            vsa_plan_t plan = p->plans[hc];
            const int nh = p->chunk_heads[hc];
            const int h0 = hc * p->chunk;
            const size_t nat = (size_t)nh * p->N * row;
            const size_t off_nat = ((size_t)b * p->heads + h0) * p->N * row;
            const size_t off_lse = ((size_t)b * p->heads + h0) * p->Nslots;
            // inputs: once the chunk before the previous one has permuted its own
            VSA_CUDA_TRY(cudaStreamWaitEvent(p->s_h2d, st.in_free, 0));
            VSA_CUDA_TRY(cudaMemcpyAsync(st.q, (const char*)q_host + off_nat, nat, cudaMemcpyHostToDevice, p->s_h2d));
            VSA_CUDA_TRY(cudaMemcpyAsync(st.k, (const char*)k_host + off_nat, nat, cudaMemcpyHostToDevice, p->s_h2d));
            VSA_CUDA_TRY(cudaMemcpyAsync(st.v, (const char*)v_host + off_nat, nat, cudaMemcpyHostToDevice, p->s_h2d));
            VSA_CUDA_TRY(cudaEventRecord(st.in_ready, p->s_h2d));
            // compute: inputs landed and the output staging of this set drained
            VSA_CUDA_TRY(cudaStreamWaitEvent(p->s_comp, st.in_ready, 0));
            VSA_CUDA_TRY(cudaStreamWaitEvent(p->s_comp, st.out_free, 0));
            int r = b == 0 ? vsa_plan_build(plan, p->s_comp) : VSA_OK;   // a plan serves every batch
            if (r == VSA_OK) r = vsa_permute_qkv(plan, st.q, st.k, st.v, st.qp, st.kp, st.vp, 1, D, p->s_comp);
            if (r != VSA_OK) return r;
            VSA_CUDA_TRY(cudaEventRecord(st.in_free, p->s_comp));
            r = vsa_sparse_attn_fwd(st.qp, st.kp, st.vp, st.op, st.lse, plan, 1, D, scale, p->s_comp);
            if (r == VSA_OK) r = vsa_unpermute(plan, st.op, st.o, 1, D, p->s_comp);
            if (r != VSA_OK) return r;
            VSA_CUDA_TRY(cudaEventRecord(st.out_ready, p->s_comp));
            // outputs back to the host
            VSA_CUDA_TRY(cudaStreamWaitEvent(p->s_d2h, st.out_ready, 0));
            VSA_CUDA_TRY(cudaMemcpyAsync((char*)o_host + off_nat, st.o, nat, cudaMemcpyDeviceToHost, p->s_d2h));
            VSA_CUDA_TRY(cudaMemcpyAsync(lse_host + off_lse, st.lse, (size_t)nh * p->Nslots * sizeof(float),
                                         cudaMemcpyDeviceToHost, p->s_d2h));
            VSA_CUDA_TRY(cudaEventRecord(st.out_free, p->s_d2h));
        }
    // `stream` resumes once every copy back is done (and every kernel before it)
    VSA_CUDA_TRY(cudaEventRecord(p->done, p->s_d2h));
    VSA_CUDA_TRY(cudaStreamWaitEvent(s, p->done, 0));
    return VSA_OK;
}

extern "C" int vsa_pipeline_check_status(vsa_pipeline_t p, void* stream)
{
    if (!p) return VSA_ERR_INVALID_ARG;
    int worst = VSA_OK;
    for (int c = 0; c < p->nchunks_h; ++c) {
        const int r = vsa_check_status(p->plans[c], stream);
        if (r != VSA_OK && worst == VSA_OK) worst = r;
    }
    return worst;
}

extern "C" int vsa_pipeline_destroy(vsa_pipeline_t p)
{
    if (!p) return VSA_ERR_INVALID_ARG;
    int prev = -1;
    const int dev = p->device;
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
    const cudaError_t e = cudaDeviceSynchronize();
    destroy_pipeline(p);
    if (prev >= 0 && prev != dev) cudaSetDevice(prev);
    return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// Tile-map builder for callers that cannot allocate device memory.
//
// vsa_plan_create allocates the plan's buffers with cudaMalloc.  Some callers
// cannot do that: a host framework that owns every byte of device memory
// through its own pool (a direct cudaMalloc would bypass its accounting and can
// fail once the pool has reserved the memory), or a latency-bound serving loop
// that must not pay for cudaMalloc's implicit device synchronisation.  This
// entry point builds the same int8 tile map into a buffer the caller already
// owns.  Its only working memory (the mask specs and the per-head stripe
// offset tables) lives in one file-scope device array, so it allocates nothing.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "vsa_internal.h"

namespace {

// Scratch layout: [specs: VSA_NOALLOC_MAX_HEADS x vsa_mask_spec, padded to 4 KiB]
//                 [stripe offset tables: num_heads x sbits_words x 4 bytes]
constexpr size_t kSpecBytes = 4096;
static_assert(VSA_NOALLOC_MAX_HEADS * sizeof(vsa_mask_spec) <= kSpecBytes, "spec area too small");

// Held by every GPU that loads the library, until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[VSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

struct SpecPack {
    vsa_mask_spec s[VSA_NOALLOC_MAX_HEADS];
};

// The specs travel as a kernel parameter, so no host-to-device copy is needed.
__global__ void store_specs_kernel(const __grid_constant__ SpecPack pack, int n, vsa_mask_spec* dst)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) dst[i] = pack.s[i];
}

// Device address of the scratch array on the current device.  Host code only
// sees a host-side stand-in under the array's name, so the address is taken
// once per device with cudaGetSymbolAddress while that device is current.
int scratch_address(void** out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return VSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return VSA_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return VSA_OK;
}

}  // namespace

extern "C" int vsa_tile_map_noalloc(const vsa_mask_spec* specs, int num_heads, int T, int H, int W, int bt,
                                    int bh, int bw, int q_tile, int kv_tile, int8_t* map_out,
                                    size_t map_bytes, void* stream)
{
    if (!specs || !map_out || num_heads < 1) return VSA_ERR_INVALID_ARG;
    if (num_heads > VSA_NOALLOC_MAX_HEADS) return VSA_ERR_UNSUPPORTED;
    int has_stripe = 0;
    for (int h = 0; h < num_heads; ++h) {
        const int r = vsa_check_spec(&specs[h]);
        if (r != VSA_OK) return r;
        has_stripe |= specs[h].kind == VSA_MASK_STRIPE;
    }
    vsa_dims d;
    {
        const int r = vsa_dims_for(num_heads, T, H, W, bt, bh, bw, q_tile, kv_tile, has_stripe, &d);
        if (r != VSA_OK) return r;
    }
    const size_t need_map = (size_t)num_heads * d.nQ * d.nK;
    if (map_bytes < need_map) return VSA_ERR_INVALID_ARG;
    const size_t need_scratch = kSpecBytes + (size_t)num_heads * d.sbits_words * sizeof(uint32_t);
    if (need_scratch > VSA_NOALLOC_SCRATCH_BYTES) return VSA_ERR_UNSUPPORTED;

    // map_out must be device (or managed) memory of the current device: a host
    // pointer or another GPU's memory would fault the kernel, so it is refused
    // here (cudaPointerGetAttributes allocates nothing)
    {
        int dev = -1;
        if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
        cudaPointerAttributes pa;
        memset(&pa, 0, sizeof pa);
        if (cudaPointerGetAttributes(&pa, map_out) != cudaSuccess) {
            cudaGetLastError();
            return VSA_ERR_INVALID_ARG;
        }
        if ((pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged) || pa.device != dev)
            return VSA_ERR_INVALID_ARG;
    }
    void* base = nullptr;
    {
        const int r = scratch_address(&base);
        if (r != VSA_OK) return r;
    }
    vsa_mask_spec* d_specs = (vsa_mask_spec*)base;
    uint32_t* d_sbits = has_stripe ? (uint32_t*)((unsigned char*)base + kSpecBytes) : nullptr;

    SpecPack pack;
    memset(&pack, 0, sizeof pack);
    memcpy(pack.s, specs, sizeof(vsa_mask_spec) * num_heads);
    cudaStream_t s = (cudaStream_t)stream;
    store_specs_kernel<<<1, VSA_NOALLOC_MAX_HEADS, 0, s>>>(pack, num_heads, d_specs);
    if (cudaGetLastError() != cudaSuccess) return VSA_ERR_CUDA;
    if (has_stripe) {
        // every word of every head's table is rewritten, so the previous
        // call's contents never leak into this one
        const int r = vsa_launch_stripe_bits(d, d_specs, d_sbits, s);
        if (r != VSA_OK) return r;
    }
    return vsa_launch_tile_map(d, d_specs, d_sbits, map_out, s);
}

// noalloc.cu -- fa_fwd_kvcache_noalloc: KV-cache decode that needs no caller workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// code running inside a CUDA-graph capture that must not grow the pool, plugins
// and inference runtimes that hand a kernel only the tensors they own, or C
// programs with no allocator of their own.  This entry point runs the same
// split-KV decode as fa_fwd_kvcache, but keeps the per-split partial outputs
// and log-sum-exps in a fixed array compiled into the library.
//
// The array is a file-scope __device__ buffer of kNoAllocScratchBytes (16 MiB):
// every GPU that loads the library holds it until the process exits.  All
// calls share it, so two calls that overlap on the GPU (different streams, or
// different host threads) race on its contents; serialise them.  The partials
// of one call are all written before they are read by the same call, so
// nothing in the array has to start at zero and nothing is cleared.
#include "../../include/fa.h"
#include "internal.h"

namespace fa {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of g_noalloc_scratch per device.  The host-side symbol is only
// a stand-in for the device array and must never be handed to a kernel.
void* g_scratch_ptr[64] = {};

int scratch_for_current_device(const Device& dev, void** out) {
    if (dev.id < 0 || dev.id >= 64) return FA_ERR_CUDA;
    if (g_scratch_ptr[dev.id] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
        g_scratch_ptr[dev.id] = p;
    }
    *out = g_scratch_ptr[dev.id];
    return FA_OK;
}
}  // namespace

}  // namespace fa

using namespace fa;

extern "C" size_t fa_fwd_kvcache_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" int fa_fwd_kvcache_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* cache_seqlens, void* out, float* lse, int B, int Hq, int Hkv,
                                      int Sq, int cache_capacity, int D, float softmax_scale, int causal,
                                      int num_splits, fa_stream_t stream) {
    (void)causal;  // one query row sees every valid key under the bottom-right causal rule
    if (!q || !k_cache || !v_cache || !cache_seqlens || !out) return FA_ERR_INVALID_ARG;
    if (B <= 0 || cache_capacity <= 0 || num_splits < 0 || Sq != 1) return FA_ERR_INVALID_ARG;
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || !(softmax_scale > 0.f)) return FA_ERR_INVALID_ARG;
    if ((D != 64 && D != 128) || Hq / Hkv > 8) return FA_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * cache_capacity > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(q) || !a16(k_cache) || !a16(v_cache) || !a16(out) || (lse && !a16(lse))) return FA_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) return FA_ERR_ALIGNMENT;

    // Split size: the usual choice, made coarser (auto mode only) until the partials fit the fixed array.
    int chunk = decode_chunk_size(B, Hkv, cache_capacity, num_splits, 148);
    while (decode_workspace_bytes(B, Hq, Hkv, cache_capacity, D, chunk) > kNoAllocScratchBytes) {
        if (num_splits > 0 || chunk >= cache_capacity) return FA_ERR_WORKSPACE;   // beyond the fixed maximum
        chunk = chunk * 2 > cache_capacity ? (cache_capacity + 63) / 64 * 64 : chunk * 2;
    }

    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    void* scratch = nullptr;
    const int st = scratch_for_current_device(dev, &scratch);
    if (st != FA_OK) return st;

    Decode d;
    d.q = q;
    d.k_cache = k_cache;
    d.v_cache = v_cache;
    d.seqlens = cache_seqlens;
    d.out = out;
    d.lse = lse;
    d.B = B;
    d.Hq = Hq;
    d.Hkv = Hkv;
    d.cap = cache_capacity;
    d.D = D;
    d.scale = softmax_scale;
    d.chunk = chunk;
    d.max_chunks = (cache_capacity + chunk - 1) / chunk;
    const size_t rows = static_cast<size_t>(B) * Hkv * d.max_chunks * (Hq / Hkv);
    d.part_o = static_cast<float*>(scratch);
    d.part_lse = reinterpret_cast<float*>(static_cast<char*>(scratch) + ((rows * D * 4 + 255) & ~size_t(255)));
    return launch_decode(d, dev, static_cast<cudaStream_t>(stream));
}

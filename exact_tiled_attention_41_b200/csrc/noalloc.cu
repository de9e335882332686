// noalloc.cu -- fa_fwd_kvcache_noalloc: KV-cache decode that needs no caller workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// plugins and inference runtimes that plan all device memory ahead of time and
// hand a kernel only the tensors they own, or C programs with no allocator of
// their own, so a per-call workspace has nowhere to come from.  This entry point runs the same
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
// Device address of g_noalloc_scratch per device, looked up by the first call on that device
// and kept for the life of the process (a cudaDeviceReset after that is not supported).  The
// host-side symbol is only a stand-in for the device array and must never be handed to a kernel.
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
    KvCall c = {};
    c.q = q;
    c.k_cache = const_cast<void*>(k_cache);
    c.v_cache = const_cast<void*>(v_cache);
    c.cache_seqlens = cache_seqlens;
    c.cache_batch = B;
    c.cache_capacity = cache_capacity;
    c.out = out;
    c.lse = lse;
    c.B = B;
    c.Hq = Hq;
    c.Hkv = Hkv;
    c.Sq = Sq;
    c.D = D;
    c.scale = softmax_scale;
    c.causal = causal;
    c.window_left = -1;
    c.window_right = -1;
    c.num_splits = num_splits;
    const int st0 = kvcache_validate(c, true);
    if (st0 != FA_OK) return st0;

    // Split size: the usual choice; in automatic mode, when its partials do not fit the fixed array, the
    // largest smaller split count that fits (each count split exactly as num_splits = n splits it).
    const int cap = kvcache_chunk_limit(c);
    int chunk = kvcache_chunk(c, 148);
    if (kvcache_workspace_bytes(c, chunk) > kNoAllocScratchBytes) {
        if (num_splits > 0) return FA_ERR_WORKSPACE;                   // an explicit split is not changed
        KvCall cn = c;
        for (int n = (cap + chunk - 1) / chunk - 1;; --n) {
            if (n < 1) return FA_ERR_WORKSPACE;                        // one split per row does not fit either
            cn.num_splits = n;
            chunk = kvcache_chunk(cn, 148);
            if (kvcache_workspace_bytes(c, chunk) <= kNoAllocScratchBytes) break;
        }
    }

    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    void* scratch = nullptr;
    const int st = scratch_for_current_device(dev, &scratch);
    if (st != FA_OK) return st;
    return kvcache_launch(c, chunk, scratch, dev, static_cast<cudaStream_t>(stream));
}

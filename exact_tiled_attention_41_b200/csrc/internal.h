// internal.h -- launch descriptors shared by the C-ABI layer (api.cu) and the
// kernel files.  Host-side only types; no torch, no STL containers.
#pragma once

#include <cuda_runtime.h>

#include <utility>
#include <stddef.h>
#include <stdint.h>

namespace fa {

// A batch of independent attention problems.  Dense batches are the special
// case cu_q = cu_k = NULL with sequence b occupying tokens b*Sq .. b*Sq+Sq-1
// (queries) and b*Sk .. b*Sk+Sk-1 (keys).
struct Problem {
    const void* q;       // [Tq, Hq, D]  bf16
    const void* k;       // [Tk, Hkv, D] bf16
    const void* v;       // [Tk, Hkv, D] bf16
    const int32_t* cu_q; // device [num_seqs + 1] or NULL
    const int32_t* cu_k;
    int num_seqs;
    int Sq, Sk;          // dense lengths, or the maxima for varlen
    int Tq, Tk;          // total tokens
    int Hq, Hkv, D;
    float scale;
    // Sliding window (README, flash_attn_func docstring): query i keeps the keys j with
    // i + Lk - Lq - wl <= j <= i + Lk - Lq + wr; -1 leaves that side unbounded.
    // A causal mask is wr = 0 (with or without a window on the left).
    int wl, wr;
    // LSE addressing: index = b * lse_sB + h * lse_sH + tok_start * lse_sT + row
    long long lse_sB, lse_sH;
    int lse_sT;
};

struct Device {
    int id;
    int num_sms;
    int* status;                 // device status word
    unsigned long long timeout_ns;
};

int get_device(Device* dev);     // fills for the current device; returns FA status

// optional CUDA-event timing around a main-kernel launch (see fa_profile_begin)
void prof_before(int kernel_id, cudaStream_t s);
void prof_after(int kernel_id, cudaStream_t s);

// Launch `kern` on `stream` with programmatic stream serialization: its CTAs may be scheduled before the
// previous kernel on the stream has finished and run until their grid_dep_wait(), which returns once
// that kernel has completed.  (With an event recorded in between, the launch is serialized as usual.)
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

int launch_fwd(const Problem& pr, void* out, float* lse, int* counter, const Device& dev, cudaStream_t stream);

size_t bwd_workspace_bytes(long long Tq, int Hq, int D);
int* bwd_unit_counter(void* workspace, long long Tq, int Hq, int D);
int bwd_chunk_groups(int num_groups, int units_per_group, int group_q_heads, int max_len, int D, int num_sms);
// head dim 256: main backward kernel + dQ convert (after the shared preprocess); with_dq = false
// leaves dq alone (the deterministic backward computes it with launch_bwd_dq)
int launch_bwd256_main(const Problem& pr, const void* dout, const float* lse2, const float* delta, float* dq_acc,
                       void* dq, void* dk, void* dv, bool with_dq, const Device& dev, cudaStream_t stream);
// deterministic dQ: query-tile-stationary pass writing bf16 dq from LSE2 / Delta of the preprocess
int launch_bwd_dq(const Problem& pr, const void* dout, const float* lse2, const float* delta, void* dq,
                  const Device& dev, cudaStream_t stream);
// deterministic: dQ from a separate query-tile-stationary pass instead of float32 reduce-adds
int launch_bwd(const Problem& pr, const void* out, const void* dout, const float* lse, void* dq, void* dk,
               void* dv, void* workspace, bool deterministic, const Device& dev, cudaStream_t stream);

// One flash_attn_with_kvcache call as the C ABI receives it (README, flash_attn_with_kvcache docstring).
struct KvCall {
    const void* q;                   // [B, Sq, Hq, D]
    void* k_cache;                   // contiguous [cache_batch, cache_capacity, Hkv, D];
    void* v_cache;                   // paged [cache_batch = num_blocks, cache_capacity = page_block_size, Hkv, D]
    const int32_t* cache_seqlens;    // device [B]: keys already in the cache
    const void* k_new;               // [B, seqlen_new, Hkv, D] appended at cache_seqlens, or NULL
    const void* v_new;
    int seqlen_new;
    const int32_t* cache_batch_idx;  // device [B] or NULL (contiguous caches only)
    const int32_t* block_table;      // device [B, max_blocks_per_seq] or NULL
    int max_blocks_per_seq;
    int cache_batch, cache_capacity;
    void* out;                       // [B, Sq, Hq, D]
    float* lse;                      // [B, Hq, Sq] or NULL
    int B, Hq, Hkv, Sq, D;
    float scale;
    int causal, window_left, window_right, num_splits;
};

int kvcache_validate(const KvCall& c, bool pointers);         // FA status, no CUDA calls
int kvcache_chunk(const KvCall& c, int num_sms);              // keys per split (multiple of 64)
int kvcache_chunk_limit(const KvCall& c);                     // keys one sequence can hold
size_t kvcache_workspace_bytes(const KvCall& c, int chunk);   // float32 partial outputs and LSEs
int kvcache_launch(const KvCall& c, int chunk, void* workspace, const Device& dev, cudaStream_t stream);

int launch_wait_selftest(unsigned long long timeout_ns, const Device& dev, cudaStream_t stream);
int launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t stream);
int launch_umma_selftest(const void* a, const void* b, float* c, int mode, const Device& dev, cudaStream_t stream);

// cuTensorMapEncodeTiled, fetched through the runtime so the library needs no -lcuda.
bool make_map_3d_bf16(void* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                      uint64_t stride2_bytes, uint32_t box0, uint32_t box1, uint32_t box2);
bool make_map_2d_bf16(void* map, const void* base, uint64_t d0, uint64_t d1, uint64_t stride1_bytes, uint32_t box0,
                      uint32_t box1);

}  // namespace fa

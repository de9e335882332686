// api.cu -- the C ABI declared in include/fa.h: argument validation, workspace
// sizing, tensor-map creation and dispatch to the kernels.  Validation happens
// before any CUDA call, so invalid arguments are reported without a GPU.
#include "../../include/fa.h"
#include "internal.h"

#include <cuda.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

namespace fa {

__device__ int g_status_word;

static unsigned long long g_timeout_ns = 2000000000ull;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

bool make_map_3d_bf16(void* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                      uint64_t stride2_bytes, uint32_t box0, uint32_t box1, uint32_t box2) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {box0, box1, box2};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d_bf16(void* map, const void* base, uint64_t d0, uint64_t d1, uint64_t stride1_bytes, uint32_t box0,
                      uint32_t box1) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {d0, d1};
    cuuint64_t strides[1] = {stride1_bytes};
    cuuint32_t box[2] = {box0, box1};
    cuuint32_t estr[2] = {1, 1};
    return fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int get_device(Device* d) {
    static int sms[64] = {};
    static int* status[64] = {};
    int id = 0;
    if (cudaGetDevice(&id) != cudaSuccess || id < 0 || id >= 64) return FA_ERR_CUDA;
    if (sms[id] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, id) != cudaSuccess || n <= 0) return FA_ERR_CUDA;
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return FA_ERR_CUDA;
        status[id] = static_cast<int*>(ptr);
        sms[id] = n;
    }
    d->id = id;
    d->num_sms = sms[id];
    d->status = status[id];
    d->timeout_ns = g_timeout_ns;
    return FA_OK;
}

}  // namespace fa

using namespace fa;

namespace {
// The whole backward of one call (preprocess, main kernel, dQ convert or dQ pass) between one pair
// of profiling events (id FA_KERNEL_BWD_ALL).
int launch_bwd_timed(const Problem& pr, const void* out, const void* dout, const float* lse, void* dq, void* dk,
                     void* dv, void* workspace, bool deterministic, const Device& dev, cudaStream_t stream) {
    prof_before(4, stream);
    const int st = launch_bwd(pr, out, dout, lse, dq, dk, dv, workspace, deterministic, dev, stream);
    prof_after(4, stream);
    return st;
}
}  // namespace

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
static bool supported_d(int D) { return D == 64 || D == 128 || D == 256; }

static int check_heads(int Hq, int Hkv, int D, float scale) {
    if (Hq <= 0 || Hkv <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return FA_ERR_INVALID_ARG;
    if (!supported_d(D)) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

// Sequence lengths are bounded by 2^30 so that row +- window arithmetic stays inside int32 in the kernels.
static const int kMaxSeqlen = 1 << 30;

// Window sides as the kernels take them: -1 = unbounded; a causal mask caps the right side at 0
// (the keys kept are those both rules keep).  Any negative side counts as unbounded, and so does a
// side of 2^30 or more: with j - (i + Sk - Sq) in [1 - Sk, Sq - 1] it never excludes a key.
static void window_sides(int causal, int window_left, int window_right, int* wl, int* wr) {
    *wl = (window_left < 0 || window_left >= kMaxSeqlen) ? -1 : window_left;
    *wr = (window_right < 0 || window_right >= kMaxSeqlen) ? -1 : window_right;
    if (causal) *wr = 0;
}

static int check_tokens(long long tokens, int H, int D) {
    // element indices are formed in 64-bit, token coordinates of tile loads in int32
    if (tokens > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    if (tokens * H * D > (1LL << 40)) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

extern "C" {

const char* fa_status_string(int s) {
    switch (s) {
        case FA_OK: return "ok";
        case FA_ERR_INVALID_ARG: return "invalid argument";
        case FA_ERR_UNSUPPORTED: return "unsupported configuration";
        case FA_ERR_ALIGNMENT: return "misaligned pointer";
        case FA_ERR_WORKSPACE: return "workspace too small";
        case FA_ERR_CUDA: return "CUDA error";
        case FA_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

unsigned long long fa_set_wait_timeout_ns(unsigned long long ns) {
    const unsigned long long prev = g_timeout_ns;
    g_timeout_ns = ns == 0 ? 2000000000ull : ns;
    return prev;
}

int fa_get_device_status(fa_stream_t stream) {
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaMemcpyAsync(&host, dev.status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemsetAsync(dev.status, 0, sizeof(int), s) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
    return host;
}

// ----------------------------------------------------------------------- dense forward
// The forward's workspace is optional: 256 bytes for the unit counter of its dynamic schedule.
constexpr size_t kFwdWorkspace = 256;
size_t fa_fwd_workspace_size(int, int, int, int, int, int) { return kFwdWorkspace; }

// NULL: the static schedule (nothing to check); otherwise the counter, with the usual workspace rules.
static int fwd_counter(void* workspace, size_t workspace_bytes, int** counter) {
    *counter = nullptr;
    if (workspace == nullptr) return FA_OK;
    if (!aligned256(workspace)) return FA_ERR_ALIGNMENT;
    if (workspace_bytes < kFwdWorkspace) return FA_ERR_WORKSPACE;
    *counter = static_cast<int*>(workspace);
    return FA_OK;
}

static int validate_dense(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                          float scale) {
    if (q == nullptr || k == nullptr || v == nullptr) return FA_ERR_INVALID_ARG;
    if (B <= 0 || Sq <= 0 || Sk <= 0) return FA_ERR_INVALID_ARG;
    if (Sq > kMaxSeqlen || Sk > kMaxSeqlen) return FA_ERR_UNSUPPORTED;
    int st = check_heads(Hq, Hkv, D, scale);
    if (st != FA_OK) return st;
    if ((st = check_tokens(static_cast<long long>(B) * Sq, Hq, D)) != FA_OK) return st;
    if ((st = check_tokens(static_cast<long long>(B) * Sk, Hkv, D)) != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return FA_ERR_ALIGNMENT;
    return FA_OK;
}

static Problem dense_problem(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int Sq, int Sk,
                             int D, float scale, int causal, int window_left, int window_right) {
    Problem pr;
    pr.q = q;
    pr.k = k;
    pr.v = v;
    pr.cu_q = nullptr;
    pr.cu_k = nullptr;
    pr.num_seqs = B;
    pr.Sq = Sq;
    pr.Sk = Sk;
    pr.Tq = B * Sq;
    pr.Tk = B * Sk;
    pr.Hq = Hq;
    pr.Hkv = Hkv;
    pr.D = D;
    pr.scale = scale;
    window_sides(causal, window_left, window_right, &pr.wl, &pr.wr);
    pr.lse_sB = static_cast<long long>(Hq) * Sq;
    pr.lse_sH = Sq;
    pr.lse_sT = 0;
    return pr;
}

int fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int Sq, int Sk,
           int D, float softmax_scale, int causal, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    return fa_fwd_ex(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, softmax_scale, causal, -1, -1, workspace,
                     workspace_bytes, stream);
}

int fa_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int Sq,
              int Sk, int D, float softmax_scale, int causal, int window_left, int window_right, void* workspace,
              size_t workspace_bytes, fa_stream_t stream) {
    int st = validate_dense(q, k, v, B, Hq, Hkv, Sq, Sk, D, softmax_scale);
    if (st != FA_OK) return st;
    if (out == nullptr || lse == nullptr) return FA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(lse)) return FA_ERR_ALIGNMENT;
    int* counter = nullptr;
    if ((st = fwd_counter(workspace, workspace_bytes, &counter)) != FA_OK) return st;
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    Problem pr = dense_problem(q, k, v, B, Hq, Hkv, Sq, Sk, D, softmax_scale, causal, window_left, window_right);
    return launch_fwd(pr, out, lse, counter, dev, static_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------- dense backward
size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D) {
    (void)Hkv;
    (void)Sk;
    if (B <= 0 || Hq <= 0 || Sq <= 0 || D <= 0) return 0;
    return bwd_workspace_bytes(static_cast<long long>(B) * Sq, Hq, D);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse, void* dq,
           void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int D, float softmax_scale, int causal,
           void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    return fa_bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D, softmax_scale, causal, -1, -1, 0,
                     workspace, workspace_bytes, stream);
}

int fa_bwd_ex(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
              void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int D, float softmax_scale,
              int causal, int window_left, int window_right, int deterministic, void* workspace,
              size_t workspace_bytes, fa_stream_t stream) {
    int st = validate_dense(q, k, v, B, Hq, Hkv, Sq, Sk, D, softmax_scale);
    if (st != FA_OK) return st;
    if (!out || !dout || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(dout) || !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_ALIGNMENT;
    if (!aligned256(workspace)) return FA_ERR_ALIGNMENT;
    if (workspace_bytes < fa_bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D)) return FA_ERR_WORKSPACE;
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    Problem pr = dense_problem(q, k, v, B, Hq, Hkv, Sq, Sk, D, softmax_scale, causal, window_left, window_right);
    return launch_bwd_timed(pr, out, dout, lse, dq, dk, dv, workspace, deterministic != 0, dev,
                            static_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------- varlen
static int validate_varlen(const void* q, const void* k, const void* v, const int32_t* cu_q, const int32_t* cu_k,
                           int num_seqs, int max_q, int max_k, int total_q, int total_k, int Hq, int Hkv, int D,
                           float scale) {
    if (!q || !k || !v || !cu_q || !cu_k) return FA_ERR_INVALID_ARG;
    if (num_seqs <= 0 || max_q <= 0 || max_k <= 0 || total_q <= 0 || total_k <= 0) return FA_ERR_INVALID_ARG;
    if (max_q > kMaxSeqlen || max_k > kMaxSeqlen) return FA_ERR_UNSUPPORTED;
    int st = check_heads(Hq, Hkv, D, scale);
    if (st != FA_OK) return st;
    if ((st = check_tokens(total_q, Hq, D)) != FA_OK) return st;
    if ((st = check_tokens(total_k, Hkv, D)) != FA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return FA_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(cu_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_k) & 3u)) return FA_ERR_ALIGNMENT;
    return FA_OK;
}

static Problem varlen_problem(const void* q, const void* k, const void* v, const int32_t* cu_q, const int32_t* cu_k,
                              int num_seqs, int max_q, int max_k, int total_q, int total_k, int Hq, int Hkv, int D,
                              float scale, int causal, int window_left, int window_right) {
    Problem pr;
    pr.q = q;
    pr.k = k;
    pr.v = v;
    pr.cu_q = cu_q;
    pr.cu_k = cu_k;
    pr.num_seqs = num_seqs;
    pr.Sq = max_q;
    pr.Sk = max_k;
    pr.Tq = total_q;
    pr.Tk = total_k;
    pr.Hq = Hq;
    pr.Hkv = Hkv;
    pr.D = D;
    pr.scale = scale;
    window_sides(causal, window_left, window_right, &pr.wl, &pr.wr);
    pr.lse_sB = 0;
    pr.lse_sH = total_q;
    pr.lse_sT = 1;
    return pr;
}

size_t fa_varlen_fwd_workspace_size(int, int, int, int, int, int) { return kFwdWorkspace; }

int fa_varlen_fwd(const void* q, const void* k, const void* v, void* out, float* lse, const int32_t* cu_seqlens_q,
                  const int32_t* cu_seqlens_k, int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q,
                  int total_k, int Hq, int Hkv, int D, float softmax_scale, int causal, void* workspace,
                  size_t workspace_bytes, fa_stream_t stream) {
    return fa_varlen_fwd_ex(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, max_seqlen_k,
                            total_q, total_k, Hq, Hkv, D, softmax_scale, causal, -1, -1, workspace, workspace_bytes,
                            stream);
}

int fa_varlen_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse, const int32_t* cu_seqlens_q,
                     const int32_t* cu_seqlens_k, int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q,
                     int total_k, int Hq, int Hkv, int D, float softmax_scale, int causal, int window_left,
                     int window_right, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    int st = validate_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, max_seqlen_k, total_q, total_k,
                             Hq, Hkv, D, softmax_scale);
    if (st != FA_OK) return st;
    if (!out || !lse) return FA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(lse)) return FA_ERR_ALIGNMENT;
    int* counter = nullptr;
    if ((st = fwd_counter(workspace, workspace_bytes, &counter)) != FA_OK) return st;
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    Problem pr = varlen_problem(q, k, v, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, max_seqlen_k, total_q,
                                total_k, Hq, Hkv, D, softmax_scale, causal, window_left, window_right);
    return launch_fwd(pr, out, lse, counter, dev, static_cast<cudaStream_t>(stream));
}

size_t fa_varlen_bwd_workspace_size(int num_seqs, int total_q, int total_k, int Hq, int Hkv, int D) {
    (void)num_seqs;
    (void)total_k;
    (void)Hkv;
    if (total_q <= 0 || Hq <= 0 || D <= 0) return 0;
    return bwd_workspace_bytes(total_q, Hq, D);
}

int fa_varlen_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int num_seqs,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int D,
                  float softmax_scale, int causal, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    return fa_varlen_bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q,
                            max_seqlen_k, total_q, total_k, Hq, Hkv, D, softmax_scale, causal, -1, -1, 0, workspace,
                            workspace_bytes, stream);
}

int fa_varlen_bwd_ex(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
                     void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                     int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv,
                     int D, float softmax_scale, int causal, int window_left, int window_right, int deterministic,
                     void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    int st = validate_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, max_seqlen_k, total_q, total_k,
                             Hq, Hkv, D, softmax_scale);
    if (st != FA_OK) return st;
    if (!out || !dout || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(dout) || !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_ALIGNMENT;
    if (!aligned256(workspace)) return FA_ERR_ALIGNMENT;
    if (workspace_bytes < fa_varlen_bwd_workspace_size(num_seqs, total_q, total_k, Hq, Hkv, D)) return FA_ERR_WORKSPACE;
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    Problem pr = varlen_problem(q, k, v, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, max_seqlen_k, total_q,
                                total_k, Hq, Hkv, D, softmax_scale, causal, window_left, window_right);
    return launch_bwd_timed(pr, out, dout, lse, dq, dk, dv, workspace, deterministic != 0, dev,
                            static_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------- KV-cache decode
// A contiguous cache of B rows; `paged_tag` stands in for the block table when only shapes are checked.
static KvCall plain_kv_call(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_seqlens,
                            void* out, float* lse, int B, int Hq, int Hkv, int Sq, int cache_capacity, int D,
                            float softmax_scale, int causal, int num_splits) {
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
    return c;
}

static int run_kv_call(const KvCall& c, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    int st = kvcache_validate(c, true);
    if (st != FA_OK) return st;
    if (!workspace) return FA_ERR_INVALID_ARG;
    if (!aligned256(workspace)) return FA_ERR_ALIGNMENT;
    const int chunk = kvcache_chunk(c, 148);
    if (workspace_bytes < kvcache_workspace_bytes(c, chunk)) return FA_ERR_WORKSPACE;
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    return kvcache_launch(c, chunk, workspace, dev, static_cast<cudaStream_t>(stream));
}

size_t fa_fwd_kvcache_workspace_size(int B, int Hq, int Hkv, int Sq, int cache_capacity, int D, int num_splits) {
    KvCall c = plain_kv_call(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, Hq, Hkv, Sq, cache_capacity, D,
                             1.0f, 0, num_splits);
    if (kvcache_validate(c, false) != FA_OK) return 0;
    return kvcache_workspace_bytes(c, kvcache_chunk(c, 148));
}

int fa_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_seqlens, void* out,
                   float* lse, int B, int Hq, int Hkv, int Sq, int cache_capacity, int D, float softmax_scale,
                   int causal, int num_splits, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    const KvCall c = plain_kv_call(q, k_cache, v_cache, cache_seqlens, out, lse, B, Hq, Hkv, Sq, cache_capacity, D,
                                   softmax_scale, causal, num_splits);
    return run_kv_call(c, workspace, workspace_bytes, stream);
}

size_t fa_fwd_kvcache_ex_workspace_size(int B, int Hq, int Hkv, int Sq, int D, int cache_capacity,
                                        int max_blocks_per_seq, int num_splits) {
    KvCall c = plain_kv_call(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, Hq, Hkv, Sq, cache_capacity, D,
                             1.0f, 0, num_splits);
    if (max_blocks_per_seq < 0) return 0;
    static const int32_t paged_tag = 0;
    if (max_blocks_per_seq > 0) {
        c.block_table = &paged_tag;   // only its presence matters for the sizes
        c.max_blocks_per_seq = max_blocks_per_seq;
    }
    if (kvcache_validate(c, false) != FA_OK) return 0;
    return kvcache_workspace_bytes(c, kvcache_chunk(c, 148));
}

int fa_fwd_kvcache_ex(const void* q, void* k_cache, void* v_cache, const int32_t* cache_seqlens, const void* k_new,
                      const void* v_new, int seqlen_new, const int32_t* cache_batch_idx, const int32_t* block_table,
                      int max_blocks_per_seq, int cache_batch, int cache_capacity, void* out, float* lse, int B,
                      int Hq, int Hkv, int Sq, int D, float softmax_scale, int causal, int window_left,
                      int window_right, int num_splits, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
    KvCall c = plain_kv_call(q, k_cache, v_cache, cache_seqlens, out, lse, B, Hq, Hkv, Sq, cache_capacity, D,
                             softmax_scale, causal, num_splits);
    c.k_new = k_new;
    c.v_new = v_new;
    c.seqlen_new = seqlen_new;
    c.cache_batch_idx = cache_batch_idx;
    c.block_table = block_table;
    c.max_blocks_per_seq = max_blocks_per_seq;
    c.cache_batch = cache_batch;
    c.window_left = window_left;
    c.window_right = window_right;
    return run_kv_call(c, workspace, workspace_bytes, stream);
}

// ----------------------------------------------------------------------- diagnostics
int fa_debug_wait_timeout_selftest(unsigned long long timeout_ns, fa_stream_t stream) {
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    return launch_wait_selftest(timeout_ns, dev, static_cast<cudaStream_t>(stream));
}

int fa_debug_exp2_selftest(const float* x, float* y, int n, fa_stream_t stream) {
    if (!x || !y || n <= 0 || (n & 1)) return FA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return FA_ERR_ALIGNMENT;
    return launch_exp2_selftest(x, y, n, static_cast<cudaStream_t>(stream)) == 0 ? FA_OK : FA_ERR_CUDA;
}

int fa_debug_umma_selftest(const void* a, const void* b, float* c, int mode, fa_stream_t stream) {
    if (!a || !b || !c || mode < 0 || mode > 2) return FA_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(c)) return FA_ERR_ALIGNMENT;
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    return launch_umma_selftest(a, b, c, mode, dev, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

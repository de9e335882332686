// merge.cu -- merge attention results computed over disjoint key sets.
//
// For key blocks c with normalised outputs O_c and log-sum-exps LSE_c of the
// same queries, attention over the union of the blocks is
//   LSE = ln sum_c exp(LSE_c),   O = sum_c exp(LSE_c - LSE) O_c
// (flash-attention README, changelog 2.2: the split-KV decode combines its
// pieces this way in a separate kernel; kernels-community/flash-attn2 Hub
// card: the low-level ops return the LSE that makes such a merge possible).
// Blocks with LSE = -inf hold no key; if every block is empty the row's output
// is 0 and its LSE -inf.  One warp per (b, s, h) row; each lane keeps D/32
// accumulators in registers and writes only after reading every part, so the
// output may be the same buffer as one of the parts.
#include "../../include/fa.h"
#include "internal.h"
#include "sm100.cuh"

#include <math.h>

namespace fa {

template <int D, bool PARTS_F32, bool OUT_F32>
__global__ void __launch_bounds__(256) merge_lse_kernel(const void* o_parts, const float* lse_parts, int C,
                                                         long long rows, int S, int H, void* out, float* lse) {
    constexpr int PER = D / 32;   // elements per lane, contiguous
    const int lane = threadIdx.x & 31;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; row < rows;
         row += nwarps) {
        // row = (b * S + s) * H + h; the LSE of (b, h, s) sits at (b * H + h) * S + s
        const long long bs = row / H;
        const int h = static_cast<int>(row % H);
        const long long b = bs / S;
        const int s = static_cast<int>(bs % S);
        const long long li = (b * H + h) * S + s;
        const long long part_stride_lse = rows;   // [C][B][H][S]
        float mx = -INFINITY;
        for (int c = 0; c < C; ++c) mx = fmaxf(mx, __ldg(lse_parts + c * part_stride_lse + li));
        float acc[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = 0.f;
        float wsum = 0.f;
        for (int c = 0; c < C; ++c) {
            const float lc = __ldg(lse_parts + c * part_stride_lse + li);
            const float f = (lc == -INFINITY) ? 0.f : expf(lc - mx);
            wsum += f;
            const size_t base = (static_cast<size_t>(c) * rows + row) * D + lane * PER;
            if constexpr (PARTS_F32) {
                const float* src = static_cast<const float*>(o_parts) + base;
#pragma unroll
                for (int e = 0; e < PER; ++e) acc[e] = fmaf(f, src[e], acc[e]);
            } else {
                const __nv_bfloat162* src = reinterpret_cast<const __nv_bfloat162*>(
                    static_cast<const __nv_bfloat16*>(o_parts) + base);
#pragma unroll
                for (int e = 0; e < PER / 2; ++e) {
                    const float2 v = __bfloat1622float2(src[e]);
                    acc[2 * e] = fmaf(f, v.x, acc[2 * e]);
                    acc[2 * e + 1] = fmaf(f, v.y, acc[2 * e + 1]);
                }
            }
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        const size_t ob = static_cast<size_t>(row) * D + lane * PER;
        if constexpr (OUT_F32) {
            float* dst = static_cast<float*>(out) + ob;
#pragma unroll
            for (int e = 0; e < PER; ++e) dst[e] = acc[e] * inv;
        } else {
            uint32_t* dst = reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(out) + ob);
#pragma unroll
            for (int e = 0; e < PER / 2; ++e) dst[e] = pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
        }
        if (lse != nullptr && lane == 0) lse[li] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
    }
}

template <int D>
static int run_merge(const void* o_parts, const float* lse_parts, int C, long long rows, int S, int H, bool parts_f32,
                     void* out, float* lse, bool out_f32, const Device& dev, cudaStream_t stream) {
    long long blocks = (rows + 7) / 8;
    const long long cap = static_cast<long long>(dev.num_sms) * 16;
    if (blocks > cap) blocks = cap;
    const dim3 grid(static_cast<unsigned>(blocks));
    if (parts_f32) {
        if (out_f32) merge_lse_kernel<D, true, true><<<grid, 256, 0, stream>>>(o_parts, lse_parts, C, rows, S, H, out, lse);
        else merge_lse_kernel<D, true, false><<<grid, 256, 0, stream>>>(o_parts, lse_parts, C, rows, S, H, out, lse);
    } else {
        if (out_f32) merge_lse_kernel<D, false, true><<<grid, 256, 0, stream>>>(o_parts, lse_parts, C, rows, S, H, out, lse);
        else merge_lse_kernel<D, false, false><<<grid, 256, 0, stream>>>(o_parts, lse_parts, C, rows, S, H, out, lse);
    }
    return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa

using namespace fa;

extern "C" int fa_merge_lse(const void* o_parts, const float* lse_parts, int num_parts, int B, int S, int H, int D,
                            int parts_fp32, void* out, float* lse, int out_fp32, fa_stream_t stream) {
    if (!o_parts || !lse_parts || !out) return FA_ERR_INVALID_ARG;
    if (num_parts <= 0 || B <= 0 || S <= 0 || H <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256) return FA_ERR_UNSUPPORTED;
    const long long rows = static_cast<long long>(B) * S * H;
    if (rows * D * num_parts > (1LL << 40)) return FA_ERR_UNSUPPORTED;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(o_parts) || !a16(out) || !a16(lse_parts) || (lse && !a16(lse))) return FA_ERR_ALIGNMENT;
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool pf = parts_fp32 != 0, of = out_fp32 != 0;
    switch (D) {
        case 64: return run_merge<64>(o_parts, lse_parts, num_parts, rows, S, H, pf, out, lse, of, dev, s);
        case 128: return run_merge<128>(o_parts, lse_parts, num_parts, rows, S, H, pf, out, lse, of, dev, s);
        default: return run_merge<256>(o_parts, lse_parts, num_parts, rows, S, H, pf, out, lse, of, dev, s);
    }
}

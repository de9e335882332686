// merge.cu -- merge attention results computed over disjoint key sets.
//
// For key blocks c with normalised outputs O_c and log-sum-exps LSE_c of the
// same queries, attention over the union of the blocks is
//   LSE = ln sum_c exp(LSE_c),   O = sum_c exp(LSE_c - LSE) O_c
// (flash-attention README, changelog 2.2: the split-KV decode combines its
// pieces this way in a separate kernel; kernels-community/flash-attn2 Hub
// card: the low-level ops return the LSE that makes such a merge possible).
// Blocks with LSE = -inf hold no key; if every block is empty the row's output
// is 0 and its LSE -inf.  A warp merges two (b, s, h) rows at a time; each lane
// keeps D/32 accumulators per row in registers and writes only after reading
// every part of its rows, so the output may be the same buffer as one of the
// parts.
#include "../../include/fa.h"
#include "internal.h"
#include "sm100.cuh"

#include <math.h>

namespace fa {

// The part weights exp(LSE_c - max) are taken as exp2 of a scaled difference on the multi-function
// unit (the per-row scalar work would otherwise outweigh the memory traffic of the row).
constexpr float kLog2e = 1.4426950408889634f;

// D / 32 = 2, 4 or 8 contiguous elements per lane.  bf16 parts stay packed (two per word) until they
// are accumulated, so the loads of many rows can be in flight with few registers.
template <int D, bool PARTS_F32>
struct PartRow {
    static constexpr int PER = D / 32;
    static constexpr int WORDS = PARTS_F32 ? PER : PER / 2;
    uint32_t w[WORDS];
    __device__ __forceinline__ void load(const void* o_parts, size_t base) {
        if constexpr (PARTS_F32) {
            const float* src = static_cast<const float*>(o_parts) + base;
            if constexpr (PER == 2) {
                const uint2 x = __ldg(reinterpret_cast<const uint2*>(src));
                w[0] = x.x;
                w[1] = x.y;
            } else {
#pragma unroll
                for (int e = 0; e < PER / 4; ++e) {
                    const uint4 x = __ldg(reinterpret_cast<const uint4*>(src) + e);
                    w[4 * e] = x.x;
                    w[4 * e + 1] = x.y;
                    w[4 * e + 2] = x.z;
                    w[4 * e + 3] = x.w;
                }
            }
        } else {
            const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(o_parts) + base;
            if constexpr (PER == 2) {
                w[0] = __ldg(reinterpret_cast<const unsigned int*>(src));
            } else if constexpr (PER == 4) {
                const uint2 x = __ldg(reinterpret_cast<const uint2*>(src));
                w[0] = x.x;
                w[1] = x.y;
            } else {
                const uint4 x = __ldg(reinterpret_cast<const uint4*>(src));
                w[0] = x.x;
                w[1] = x.y;
                w[2] = x.z;
                w[3] = x.w;
            }
        }
    }
    __device__ __forceinline__ float get(int e) const {
        if constexpr (PARTS_F32) {
            return __uint_as_float(w[e]);
        } else {
            const uint32_t x = w[e >> 1];
            return __uint_as_float((e & 1) ? (x & 0xffff0000u) : (x << 16));   // bf16 -> f32 exactly
        }
    }
};

// Each warp merges RPW rows at a time in one pass over the parts: a chunk of up to four parts has its
// LSEs and rows loaded together, then the running maximum, weight sum and accumulators are rescaled
// (exactly as an online softmax) and the chunk is added.
// Work split: block k takes (b, h) = k % (B H) and positions s of stride (number of blocks / (B H));
// consecutive blocks are neighbouring heads of the same tokens, so blocks resident at the same time
// read neighbouring 256-byte pieces of the same rows.  No division on the per-row path; LSE loads of
// consecutive positions are contiguous.  At most 64 registers, so four blocks (32 warps) per SM keep
// enough loads in flight.
template <int D, bool PARTS_F32, bool OUT_F32, int RPW>
__global__ void __launch_bounds__(256, 4) merge_lse_kernel(const void* o_parts, const float* lse_parts, int C,
                                                         long long rows, int B, int S, int H, void* out, float* lse) {
    constexpr int PER = D / 32;   // elements per lane, contiguous
    constexpr int CU = 4;         // parts per chunk
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int BH = B * H;
    const int per_bh = gridDim.x / BH;    // blocks sharing one (b, h); the grid holds per_bh * BH blocks
    const int bh = blockIdx.x % BH, sx = blockIdx.x / BH;
    const int b = bh / H, h = bh % H;
    const long long lbase = static_cast<long long>(bh) * S;              // LSE of (b, h, s) at lbase + s
    for (int s0 = (sx * 8 + warp) * RPW; s0 < S; s0 += per_bh * 8 * RPW) {
        long long row[RPW];
        float m[RPW], wsum[RPW], acc[RPW][PER];
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int s = min(s0 + i, S - 1);                            // a position past S repeats S-1
            row[i] = (static_cast<long long>(b) * S + s) * H + h;        // O row of (b, s, h)
            m[i] = -INFINITY;
            wsum[i] = 0.f;
#pragma unroll
            for (int e = 0; e < PER; ++e) acc[i][e] = 0.f;
        }
        for (int c0 = 0; c0 < C; c0 += CU) {
            float lc[RPW][CU];
            PartRow<D, PARTS_F32> v[RPW][CU];
#pragma unroll
            for (int i = 0; i < RPW; ++i) {
                const int s = min(s0 + i, S - 1);
#pragma unroll
                for (int u = 0; u < CU; ++u) {
                    const int c = min(c0 + u, C - 1);   // a part past the end is reloaded, weight 0
                    lc[i][u] = c0 + u < C ? __ldg(lse_parts + c * rows + lbase + s) : -INFINITY;
                    v[i][u].load(o_parts, (static_cast<size_t>(c) * rows + row[i]) * D + lane * PER);
                }
            }
#pragma unroll
            for (int i = 0; i < RPW; ++i) {
                float mc = m[i];
#pragma unroll
                for (int u = 0; u < CU; ++u) mc = fmaxf(mc, lc[i][u]);
                const float sc = (m[i] == -INFINITY) ? 0.f : ex2_approx((m[i] - mc) * kLog2e);
                wsum[i] *= sc;
#pragma unroll
                for (int e = 0; e < PER; ++e) acc[i][e] *= sc;
#pragma unroll
                for (int u = 0; u < CU; ++u) {
                    const float f = (lc[i][u] == -INFINITY) ? 0.f : ex2_approx((lc[i][u] - mc) * kLog2e);
                    wsum[i] += f;
#pragma unroll
                    for (int e = 0; e < PER; ++e) acc[i][e] = fmaf(f, v[i][u].get(e), acc[i][e]);
                }
                m[i] = mc;
            }
        }
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            if (s0 + i >= S) break;
            const float inv = wsum[i] > 0.f ? 1.f / wsum[i] : 0.f;
            const size_t ob = static_cast<size_t>(row[i]) * D + lane * PER;
            if constexpr (OUT_F32) {
                float* dst = static_cast<float*>(out) + ob;
                if constexpr (PER == 2) {
                    *reinterpret_cast<float2*>(dst) = make_float2(acc[i][0] * inv, acc[i][1] * inv);
                } else {
#pragma unroll
                    for (int e = 0; e < PER / 4; ++e)
                        reinterpret_cast<float4*>(dst)[e] =
                            make_float4(acc[i][4 * e] * inv, acc[i][4 * e + 1] * inv, acc[i][4 * e + 2] * inv,
                                        acc[i][4 * e + 3] * inv);
                }
            } else {
                uint32_t w[PER / 2];
#pragma unroll
                for (int e = 0; e < PER / 2; ++e) w[e] = pack_bf16x2(acc[i][2 * e] * inv, acc[i][2 * e + 1] * inv);
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(out) + ob;
                if constexpr (PER == 2) *reinterpret_cast<uint32_t*>(dst) = w[0];
                else if constexpr (PER == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
                else *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (lse != nullptr && lane == 0)
                lse[lbase + s0 + i] = wsum[i] > 0.f ? m[i] + __logf(wsum[i]) : -INFINITY;
        }
    }
}

template <int D>
static int run_merge(const void* o_parts, const float* lse_parts, int C, int B, int S, int H, bool parts_f32,
                     void* out, float* lse, bool out_f32, const Device& dev, cudaStream_t stream) {
    constexpr int RPW = 2;   // rows per warp per pass
    const long long rows = static_cast<long long>(B) * S * H;
    const long long BH = static_cast<long long>(B) * H;
    // about 16 blocks of 8 warps per SM; a whole number of blocks per (b, h) when there are enough
    long long per_bh = (static_cast<long long>(dev.num_sms) * 16 + BH - 1) / BH;
    const long long need = (S + 8 * RPW - 1) / (8 * RPW);
    if (per_bh > need) per_bh = need;
    if (per_bh < 1) per_bh = 1;
    if (per_bh * BH > 0x7fffffffLL) per_bh = 1;   // B * H itself is at most 2^31 - 1 (checked by the caller)
    const dim3 grid(static_cast<unsigned>(per_bh * BH));
    if (parts_f32) {
        if (out_f32) merge_lse_kernel<D, true, true, RPW><<<grid, 256, 0, stream>>>(o_parts, lse_parts, C, rows, B, S, H, out, lse);
        else merge_lse_kernel<D, true, false, RPW><<<grid, 256, 0, stream>>>(o_parts, lse_parts, C, rows, B, S, H, out, lse);
    } else {
        if (out_f32) merge_lse_kernel<D, false, true, RPW><<<grid, 256, 0, stream>>>(o_parts, lse_parts, C, rows, B, S, H, out, lse);
        else merge_lse_kernel<D, false, false, RPW><<<grid, 256, 0, stream>>>(o_parts, lse_parts, C, rows, B, S, H, out, lse);
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
    if (rows * D * num_parts > (1LL << 40) || S > (1 << 30) || static_cast<long long>(B) * H > 0x7fffffffLL)
        return FA_ERR_UNSUPPORTED;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(o_parts) || !a16(out) || !a16(lse_parts) || (lse && !a16(lse))) return FA_ERR_ALIGNMENT;
    Device dev;
    if (get_device(&dev) != FA_OK) return FA_ERR_CUDA;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool pf = parts_fp32 != 0, of = out_fp32 != 0;
    switch (D) {
        case 64: return run_merge<64>(o_parts, lse_parts, num_parts, B, S, H, pf, out, lse, of, dev, s);
        case 128: return run_merge<128>(o_parts, lse_parts, num_parts, B, S, H, pf, out, lse, of, dev, s);
        default: return run_merge<256>(o_parts, lse_parts, num_parts, B, S, H, pf, out, lse, of, dev, s);
    }
}

// decode.cu -- single-query attention against a contiguous KV cache, split over
// the cache length (flash-attention README, changelog 2.2: for query length 1
// the bottleneck is loading the KV cache, so the load is split across thread
// blocks and a separate kernel combines the results; flash_attn_with_kvcache
// docstring: cache (batch, capacity, nheads_k, headdim), cache_seqlens per row).
//
// Split kernel: one CTA per (chunk of `chunk` keys, KV head, batch row).  A
// producer warp streams 64-key K/V tiles through a 3-stage TMA ring (128-byte
// swizzle); four consumer warps each take 16 keys of every tile and serve all
// G = Hq/Hkv query heads of the KV head from that single read, with bf16
// mma.sync (16 x 8 x 16) for QK^T and PV -- the arithmetic is small next to the
// bytes, so the tensor-core instruction only has to keep up with HBM.  Each warp
// keeps its own running max / sum / output; the four are merged in shared
// memory and the chunk's normalised output and LSE are written in fp32.
// Combine kernel: LSE = ln sum_c exp(LSE_c), O = sum_c exp(LSE_c - LSE) O_c.
// Keys at or beyond cache_seqlens[b] are masked, and their V rows are zeroed
// in shared memory before use so that whatever the cache holds there (the
// tests fill it with NaN) cannot reach the result.
#include "internal.h"
#include "sm100.cuh"

#include <math.h>

namespace fa {

struct DecodeParams {
    const __nv_bfloat16* q;
    const int32_t* seqlens;
    float* part_o;
    float* part_lse;
    int Hq, Hkv, G, cap, chunk, max_chunks;
    float scale_log2;
    unsigned long long timeout_ns;
    int* status;
};

constexpr int kDecTile = 64;       // keys per pipeline stage
constexpr int kDecStages = 3;
constexpr int kDecConsumers = 4;   // warps; 16 keys each per stage

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of (row, 16-byte chunk) inside a [rows][64 bf16] tile written by TMA with 128-byte swizzle
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__((kDecConsumers + 1) * 32, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ DecodeParams p) {
    constexpr int NBOX = D / 64;
    constexpr uint32_t TILE_BYTES = kDecTile * D * 2;        // one of K or V
    constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;
    constexpr int KSTEPS = D / 16;
    constexpr int NT_D = D / 8;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecStages * STAGE_BYTES);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kDecStages);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kDecStages);

    const int chunk_id = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int L = min(max(__ldg(p.seqlens + b), 0), p.cap);   // lengths beyond the capacity are clamped
    const int k0 = chunk_id * p.chunk;
    if (k0 >= L) return;                              // this split holds no valid key
    const int nk = min(p.chunk, L - k0);
    const int ns = (nk + kDecTile - 1) / kDecTile;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(bars + s, 1);
            mbar_init(bars + kDecStages + s, kDecConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const Watch w{abort_flag, p.status, p.timeout_ns};

    if (warp == kDecConsumers) {
        if (lane == 0) {
            const int y0 = b * p.cap + k0;
            for (int s = 0; s < ns; ++s) {
                const int slot = s % kDecStages;
                if (s >= kDecStages && !mbar_wait(empty0 + 8 * slot, ((s / kDecStages) - 1) & 1, w)) break;
                mbar_arrive_expect_tx(full0 + 8 * slot, STAGE_BYTES);
                uint8_t* sk = smem + slot * STAGE_BYTES;
#pragma unroll
                for (int c = 0; c < NBOX; ++c) {
                    tma_load_2d(smem_u32(sk + c * kDecTile * 128), &tmK, full0 + 8 * slot, hk * D + c * 64,
                                y0 + s * kDecTile);
                    tma_load_2d(smem_u32(sk + TILE_BYTES + c * kDecTile * 128), &tmV, full0 + 8 * slot,
                                hk * D + c * 64, y0 + s * kDecTile);
                }
            }
        }
        __syncwarp();
        return;   // the producer does not take part in the merge below
    }

    // ---------------------------------------------------------------- consumers
    const float c2 = p.scale_log2;
    const int qr = lane >> 2;          // fragment row (query head within the group), and qr + 8
    const int qc = (lane & 3) * 2;     // fragment column pair
    // Q as the A operand (rows = query heads of this KV head; rows >= G are zero)
    uint32_t qa[KSTEPS][4];
    {
        const __nv_bfloat16* qbase = p.q + (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(hk) * p.G) * D;
        const bool r0 = qr < p.G, r1 = qr + 8 < p.G;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int d0 = kk * 16 + qc;
            qa[kk][0] = r0 ? *reinterpret_cast<const uint32_t*>(qbase + qr * D + d0) : 0u;
            qa[kk][1] = r1 ? *reinterpret_cast<const uint32_t*>(qbase + (qr + 8) * D + d0) : 0u;
            qa[kk][2] = r0 ? *reinterpret_cast<const uint32_t*>(qbase + qr * D + d0 + 8) : 0u;
            qa[kk][3] = r1 ? *reinterpret_cast<const uint32_t*>(qbase + (qr + 8) * D + d0 + 8) : 0u;
        }
    }
    float o[NT_D][4];
#pragma unroll
    for (int j = 0; j < NT_D; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows qr and qr + 8
    const int kw = warp * 16;          // this warp's keys inside a tile
    bool ok = true;

    for (int s = 0; s < ns; ++s) {
        const int slot = s % kDecStages;
        if (!mbar_wait(full0 + 8 * slot, (s / kDecStages) & 1, w)) { ok = false; break; }
        const uint32_t sk = smem_u32(smem + slot * STAGE_BYTES);
        const uint32_t sv = sk + TILE_BYTES;
        const int kt = k0 + s * kDecTile + kw;    // cache index of this warp's first key
        // ---- S = Q K^T for 16 keys (two n-tiles of 8)
        float sc[2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t) sc[t][0] = sc[t][1] = sc[t][2] = sc[t][3] = 0.f;
        {
            const int mi = lane >> 3, ri = lane & 7;
            const int key = kw + 8 * (mi >> 1) + ri;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const int chunk = 2 * kk + (mi & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sk + (chunk >> 3) * kDecTile * 128 + sw128(key, chunk & 7), b0, b1, b2, b3);
                mma_bf16_16816(sc[0], qa[kk], b0, b1);
                mma_bf16_16816(sc[1], qa[kk], b2, b3);
            }
        }
        // ---- mask keys beyond the cache length
        const bool tail = kt + 16 > L;
        if (tail) {
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (kt + 8 * t + qc + (e & 1) >= L) sc[t][e] = -INFINITY;
            // zero V rows of keys >= L in this warp's 16-row slice
            for (int idx = lane; idx < 16 * NBOX * 8; idx += 32) {
                const int rr = idx / (NBOX * 8), rem = idx % (NBOX * 8);
                if (kt + rr >= L) {
                    uint8_t* dst = smem + slot * STAGE_BYTES + TILE_BYTES + (rem >> 3) * kDecTile * 128 +
                                   (kw + rr) * 128 + (rem & 7) * 16;
                    *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
                }
            }
            __syncwarp();
        }
        // ---- online softmax (rows qr: e = 0, 1; rows qr + 8: e = 2, 3)
        float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = (m0 == -INFINITY) ? 0.f : ex2_approx((m0 - mn0) * c2);
        const float al1 = (m1 == -INFINITY) ? 0.f : ex2_approx((m1 - mn1) * c2);
        const float ms0 = (mn0 == -INFINITY) ? 0.f : mn0 * c2;
        const float ms1 = (mn1 == -INFINITY) ? 0.f : mn1 * c2;
        m0 = mn0;
        m1 = mn1;
        float pr[2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            pr[t][0] = ex2_approx(fmaf(sc[t][0], c2, -ms0));
            pr[t][1] = ex2_approx(fmaf(sc[t][1], c2, -ms0));
            pr[t][2] = ex2_approx(fmaf(sc[t][2], c2, -ms1));
            pr[t][3] = ex2_approx(fmaf(sc[t][3], c2, -ms1));
        }
        l0 = l0 * al0 + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
        l1 = l1 * al1 + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
        uint32_t pa[4];
        pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
        pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
        pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
        pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
        // ---- O = O * alpha + P V
        {
            const int mi = lane >> 3, ri = lane & 7;
            const int key = kw + 8 * (mi & 1) + ri;
#pragma unroll
            for (int jj = 0; jj < NT_D / 2; ++jj) {
                const int chunk = 2 * jj + (mi >> 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(sv + (chunk >> 3) * kDecTile * 128 + sw128(key, chunk & 7), b0, b1, b2, b3);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float* oo = o[2 * jj + h];
                    oo[0] *= al0;
                    oo[1] *= al0;
                    oo[2] *= al1;
                    oo[3] *= al1;
                }
                mma_bf16_16816(o[2 * jj], pa, b0, b1);
                mma_bf16_16816(o[2 * jj + 1], pa, b2, b3);
            }
        }
        if (tail) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * slot);
    }

    // ---------------------------------------------------------------- merge the four warps
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    // all consumers are past their last stage before the stage memory is reused
    asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumers * 32) : "memory");
    if (!__all_sync(0xffffffffu, ok) || w.aborted()) return;
    float* sO = reinterpret_cast<float*>(smem);                          // [4 warps][16 rows][D]
    float* sM = sO + kDecConsumers * 16 * D;                             // [4][16]
    float* sL = sM + kDecConsumers * 16;
    {
        float* ow = sO + warp * 16 * D;
#pragma unroll
        for (int j = 0; j < NT_D; ++j) {
            ow[qr * D + 8 * j + qc] = o[j][0];
            ow[qr * D + 8 * j + qc + 1] = o[j][1];
            ow[(qr + 8) * D + 8 * j + qc] = o[j][2];
            ow[(qr + 8) * D + 8 * j + qc + 1] = o[j][3];
        }
        if ((lane & 3) == 0) {
            sM[warp * 16 + qr] = m0;
            sM[warp * 16 + qr + 8] = m1;
            sL[warp * 16 + qr] = l0;
            sL[warp * 16 + qr + 8] = l1;
        }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumers * 32) : "memory");
    const size_t row0 = ((static_cast<size_t>(b) * p.Hkv + hk) * p.max_chunks + chunk_id) * p.G;
    for (int idx = threadIdx.x; idx < p.G * D; idx += kDecConsumers * 32) {
        const int r = idx / D, d = idx % D;
        float mx = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kDecConsumers; ++ww) mx = fmaxf(mx, sM[ww * 16 + r]);
        float lsum = 0.f, acc = 0.f;
#pragma unroll
        for (int ww = 0; ww < kDecConsumers; ++ww) {
            const float mw = sM[ww * 16 + r];
            const float f = (mw == -INFINITY) ? 0.f : exp2f((mw - mx) * c2);
            lsum += f * sL[ww * 16 + r];
            acc += f * sO[(ww * 16 + r) * D + d];
        }
        p.part_o[(row0 + r) * D + d] = lsum > 0.f ? acc / lsum : 0.f;
        if (d == 0)
            p.part_lse[row0 + r] = lsum > 0.f ? (mx * c2 + log2f(lsum)) * 0.69314718055994530942f : -INFINITY;
    }
}

// One warp per (batch row, query head): merge the splits of that row.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const int32_t* seqlens, const float* part_o,
                                                             const float* part_lse, __nv_bfloat16* out, float* lse,
                                                             int B, int Hq, int Hkv, int G, int cap, int chunk,
                                                             int max_chunks) {
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= B * Hq) return;
    const int b = gw / Hq, hq = gw % Hq, hk = hq / G, r = hq % G;
    const int L = min(max(__ldg(seqlens + b), 0), cap);
    const int n = L > 0 ? (L + chunk - 1) / chunk : 0;
    const size_t base = (static_cast<size_t>(b) * Hkv + hk) * max_chunks;
    float mx = -INFINITY;
    for (int c = 0; c < n; ++c) mx = fmaxf(mx, part_lse[(base + c) * G + r]);
    constexpr int PER = D / 32;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    float wsum = 0.f;
    for (int c = 0; c < n; ++c) {
        const float lc = part_lse[(base + c) * G + r];
        const float f = (lc == -INFINITY) ? 0.f : expf(lc - mx);
        wsum += f;
        const float* src = part_o + ((base + c) * G + r) * D + lane * PER;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += f * src[e];
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    __nv_bfloat16* dst = out + (static_cast<size_t>(b) * Hq + hq) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
    if (lse != nullptr && lane == 0) lse[static_cast<size_t>(b) * Hq + hq] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

int decode_chunk_size(int B, int Hkv, int cap, int num_splits, int num_sms) {
    long long ch;
    if (num_splits > 0) {
        ch = (static_cast<long long>(cap) + num_splits - 1) / num_splits;
    } else {
        // aim for ~8 splits per CTA slot (2 CTAs per SM), assuming caches half full on average
        ch = static_cast<long long>(B) * Hkv * cap / (2LL * 8 * 2 * num_sms);
        if (ch > 1024) ch = 1024;
        if (ch < 256) ch = 256;
    }
    ch = (ch + kDecTile - 1) / kDecTile * kDecTile;
    if (ch < kDecTile) ch = kDecTile;
    if (ch > cap) ch = (cap + kDecTile - 1) / kDecTile * kDecTile;
    return static_cast<int>(ch);
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int cap, int D, int chunk) {
    const size_t max_chunks = (cap + chunk - 1) / chunk;
    const size_t rows = static_cast<size_t>(B) * Hkv * max_chunks * (Hq / Hkv);
    return ((rows * D * 4 + 255) & ~size_t(255)) + rows * 4;
}

template <int D>
static int run_decode(const Decode& d, const Device& dev, cudaStream_t stream) {
    alignas(64) CUtensorMap mk, mv;
    const uint64_t row_bytes = static_cast<uint64_t>(d.Hkv) * D * 2;
    const uint64_t rows = static_cast<uint64_t>(d.B) * d.cap;
    if (!make_map_2d_bf16(&mk, d.k_cache, static_cast<uint64_t>(d.Hkv) * D, rows, row_bytes, 64, kDecTile)) return 5;
    if (!make_map_2d_bf16(&mv, d.v_cache, static_cast<uint64_t>(d.Hkv) * D, rows, row_bytes, 64, kDecTile)) return 5;
    DecodeParams p;
    p.q = static_cast<const __nv_bfloat16*>(d.q);
    p.seqlens = d.seqlens;
    p.part_o = d.part_o;
    p.part_lse = d.part_lse;
    p.Hq = d.Hq;
    p.Hkv = d.Hkv;
    p.G = d.Hq / d.Hkv;
    p.cap = d.cap;
    p.chunk = d.chunk;
    p.max_chunks = d.max_chunks;
    p.scale_log2 = d.scale * 1.4426950408889634f;
    p.timeout_ns = dev.timeout_ns;
    p.status = dev.status;
    constexpr size_t stage_bytes = 2 * kDecTile * D * 2;
    constexpr size_t merge_bytes = (kDecConsumers * 16 * D + 2 * kDecConsumers * 16) * 4;
    static_assert(merge_bytes <= kDecStages * stage_bytes, "merge buffer reuses the stage memory");
    const size_t smem = 1024 + kDecStages * stage_bytes + 2 * kDecStages * 8 + 16;
    static bool set[64] = {};
    auto kern = decode_split_kernel<D>;
    if (!set[dev.id & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess)
            return 5;
        set[dev.id & 63] = true;
    }
    dim3 grid(d.max_chunks, d.Hkv, d.B);
    prof_before(2, stream);
    kern<<<grid, (kDecConsumers + 1) * 32, smem, stream>>>(mk, mv, p);
    prof_after(2, stream);
    if (cudaPeekAtLastError() != cudaSuccess) return 5;
    const int warps = d.B * d.Hq;
    decode_combine_kernel<D><<<(warps + 3) / 4, 128, 0, stream>>>(d.seqlens, d.part_o, d.part_lse,
                                                                  static_cast<__nv_bfloat16*>(d.out), d.lse, d.B, d.Hq,
                                                                  d.Hkv, p.G, d.cap, d.chunk, d.max_chunks);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 5;
}

int launch_decode(const Decode& d, const Device& dev, cudaStream_t stream) {
    switch (d.D) {
        case 64: return run_decode<64>(d, dev, stream);
        case 128: return run_decode<128>(d, dev, stream);
        default: return 2;
    }
}

}  // namespace fa

// decode.cu -- new queries against a KV cache, split over the cache length
// (flash-attention README, changelog 2.2: for short queries the bottleneck is
// loading the KV cache, so the load is split across thread blocks and a
// separate kernel combines the results; flash_attn_with_kvcache docstring:
// cache (batch, capacity, nheads_k, headdim) or pages (num_blocks,
// page_block_size, nheads_k, headdim) through block_table, cache_seqlens per
// row, optional k / v appended in place at cache_seqlens, cache_batch_idx,
// bottom-right causal mask, sliding window).
//
// Append kernel (only when k / v are given): one warp per new (row, token,
// KV head) copies the key and value rows into the cache at logical position
// cache_seqlens[b] + token, through the block table for paged caches.
//
// Split kernel: one CTA per (chunk of `chunk` keys, KV head x block of 16
// query rows, batch row).  The query rows of a KV head are its G = Hq/Hkv query
// heads times the Sq new tokens (row r = token * G + head-in-group); a block of
// 16 of them is the M dimension of bf16 mma.sync (16 x 8 x 16) for QK^T and PV
// -- the arithmetic is small next to the bytes, so the tensor-core instruction
// only has to keep up with HBM.  A producer warp streams 64-key K/V tiles
// through a 3-stage TMA ring (128-byte swizzle; a tile never crosses a page,
// whose size is a multiple of 256); four consumer warps each take 16 keys of
// every tile.  Each warp keeps its own running max / sum / output; the four are
// merged in shared memory and the chunk's normalised output and LSE are
// written in fp32.  Keys outside a row's causal / window range are masked; a
// chunk no row of the block can see writes an empty partial (LSE = -inf).
// Combine kernel: LSE = ln sum_c exp(LSE_c), O = sum_c exp(LSE_c - LSE) O_c.
// Keys at or beyond the sequence length are masked, and their V rows are zeroed
// in shared memory before use so that whatever the cache holds there (the
// tests fill it with NaN) cannot reach the result.
#include "../../include/fa.h"
#include "internal.h"
#include "sm100.cuh"

#include <math.h>

namespace fa {

struct DecodeParams {
    const __nv_bfloat16* q;
    const int32_t* seqlens;
    const int32_t* batch_idx;     // contiguous caches: cache row of each sequence, or NULL
    const int32_t* block_table;   // paged caches: [B][max_blocks], or NULL
    float* part_o;                // [B][Hkv][max_chunks][R][D]
    float* part_lse;              // [B][Hkv][max_chunks][R]
    int Hq, Hkv, G, Sq, R, row_blocks;
    int kmax;                     // keys one sequence can hold
    int chunk, max_chunks;
    int max_blocks, page;         // page = 0: contiguous cache
    int cache_batch;              // batch rows (contiguous) or blocks (paged) of the cache tensor
    int rows_total;               // physical cache rows: a tile at this row is out of the map (zero fill)
    int seq_add;                  // keys appended by this call
    int wl, wr;                   // window sides, -1 = unbounded; causal is wr = 0
    float scale_log2;
    unsigned long long timeout_ns;
    int* status;
};

constexpr int kDecTile = 64;       // keys per pipeline stage
constexpr int kDecStages = 3;
constexpr int kDecConsumers = 4;   // warps; 16 keys each per stage

// Keys sequence b attends to (cached + appended, at most kmax), and its cache batch row.  A
// contiguous-cache row index outside the cache makes the sequence empty and records an error.
__device__ __forceinline__ int dec_len(const DecodeParams& p, int b, int* bc_out, bool report) {
    int bc = b;
    if (p.page == 0 && p.batch_idx != nullptr) bc = __ldg(p.batch_idx + b);
    *bc_out = bc;
    if (p.page == 0 && (bc < 0 || bc >= p.cache_batch)) {
        if (report) atomicCAS(p.status, 0, FA_ERR_INVALID_ARG);
        return 0;
    }
    return min(max(__ldg(p.seqlens + b), 0) + p.seq_add, p.kmax);
}

// physical cache row of logical key `key` (a multiple of the tile) of sequence b; -1 if the block table
// names a block outside the cache
__device__ __forceinline__ int dec_phys_row(const DecodeParams& p, int b, int bc, int key) {
    if (p.page > 0) {
        const int blk = __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks + key / p.page);
        return (blk >= 0 && blk < p.cache_batch) ? blk * p.page + key % p.page : -1;
    }
    return bc * p.kmax + key;
}

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

// Two CTAs per SM up to D = 128 (3 stages of 2 x 64 keys x D); at D = 256 a stage is 64 KB and the
// output fragments alone take 128 registers per thread, so one CTA per SM (the 3-stage ring still
// keeps 128 KB of K/V in flight per SM).
template <int D>
constexpr int dec_min_blocks() { return D == 256 ? 1 : 2; }

template <int D>
__global__ void __launch_bounds__((kDecConsumers + 1) * 32, dec_min_blocks<D>())
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
    // launched with programmatic serialization: everything the previous kernel on the stream wrote (the
    // appended cache rows, the lengths, the previous call's use of the partials) is settled after this
    grid_dep_wait();
    grid_dep_launch();

    const int chunk_id = blockIdx.x, b = blockIdx.z;
    const int hk = blockIdx.y / p.row_blocks, rb = blockIdx.y % p.row_blocks;
    int bc;
    const int L = dec_len(p, b, &bc, threadIdx.x == 0 && chunk_id == 0 && blockIdx.y == 0);
    const int k0 = chunk_id * p.chunk;
    if (k0 >= L) return;                              // the combine reads chunks below L only
    const int r0 = rb * 16, nrows = min(16, p.R - r0);
    const size_t row0 = ((static_cast<size_t>(b) * p.Hkv + hk) * p.max_chunks + chunk_id) * p.R + r0;
    // keys visible to some row of this block (rows r0 .. r0+nrows-1 are tokens s_lo .. s_hi)
    const int off = L - p.Sq;
    const int s_lo = r0 / p.G, s_hi = (r0 + nrows - 1) / p.G;
    int lo_any = 0, hi_any = L - 1, lo_all = 0, hi_all = L - 1;
    if (p.wl >= 0) {
        lo_any = max(0, s_lo + off - p.wl);
        lo_all = max(0, s_hi + off - p.wl);
    }
    if (p.wr >= 0) {
        hi_any = min(L - 1, s_hi + off + p.wr);
        hi_all = min(L - 1, s_lo + off + p.wr);
    }
    const int kstart = k0 + max(0, (lo_any - k0) / kDecTile) * kDecTile;
    const int kend = min(k0 + p.chunk, hi_any + 1);   // exclusive
    if (kend <= kstart) {
        // no row of the block sees a key of this split: an empty partial
        for (int idx = threadIdx.x; idx < nrows * D; idx += blockDim.x) {
            p.part_o[row0 * D + idx] = 0.f;
            if (idx % D == 0) p.part_lse[row0 + idx / D] = -INFINITY;
        }
        return;
    }
    const int ns = (kend - kstart + kDecTile - 1) / kDecTile;
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
            bool bad = false;
            for (int s = 0; s < ns; ++s) {
                const int slot = s % kDecStages;
                if (s >= kDecStages && !mbar_wait(empty0 + 8 * slot, ((s / kDecStages) - 1) & 1, w)) break;
                int y = dec_phys_row(p, b, bc, kstart + s * kDecTile);
                if (y < 0) {
                    bad = true;
                    y = p.rows_total;     // outside the map: the tile reads as zeros
                }
                mbar_arrive_expect_tx(full0 + 8 * slot, STAGE_BYTES);
                uint8_t* sk = smem + slot * STAGE_BYTES;
#pragma unroll
                for (int c = 0; c < NBOX; ++c) {
                    tma_load_2d(smem_u32(sk + c * kDecTile * 128), &tmK, full0 + 8 * slot, hk * D + c * 64, y);
                    tma_load_2d(smem_u32(sk + TILE_BYTES + c * kDecTile * 128), &tmV, full0 + 8 * slot,
                                hk * D + c * 64, y);
                }
            }
            if (bad) atomicCAS(p.status, 0, FA_ERR_INVALID_ARG);
        }
        __syncwarp();
        return;   // the producer does not take part in the merge below
    }

    // ---------------------------------------------------------------- consumers
    const float c2 = p.scale_log2;
    const int qr = lane >> 2;          // fragment rows qr and qr + 8 of the block
    const int qc = (lane & 3) * 2;     // fragment column pair
    const int ra = r0 + qr, rbr = r0 + qr + 8;
    // per-row key ranges (rows past R are padding: their results are never stored)
    auto row_lo = [&](int r) { return p.wl >= 0 ? max(0, r / p.G + off - p.wl) : 0; };
    auto row_hi = [&](int r) { return p.wr >= 0 ? min(L - 1, r / p.G + off + p.wr) : L - 1; };
    const int lo_a = row_lo(ra), hi_a = row_hi(ra), lo_b = row_lo(rbr), hi_b = row_hi(rbr);
    // Q as the A operand: row r is query head hk * G + r % G of token r / G; rows past R are zero
    uint32_t qa[KSTEPS][4];
    {
        const bool va = ra < p.R, vb = rbr < p.R;
        const __nv_bfloat16* qa_row =
            p.q + ((static_cast<size_t>(b) * p.Sq + (va ? ra / p.G : 0)) * p.Hq + hk * p.G + (va ? ra % p.G : 0)) * D;
        const __nv_bfloat16* qb_row =
            p.q + ((static_cast<size_t>(b) * p.Sq + (vb ? rbr / p.G : 0)) * p.Hq + hk * p.G + (vb ? rbr % p.G : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int d0 = kk * 16 + qc;
            qa[kk][0] = va ? *reinterpret_cast<const uint32_t*>(qa_row + d0) : 0u;
            qa[kk][1] = vb ? *reinterpret_cast<const uint32_t*>(qb_row + d0) : 0u;
            qa[kk][2] = va ? *reinterpret_cast<const uint32_t*>(qa_row + d0 + 8) : 0u;
            qa[kk][3] = vb ? *reinterpret_cast<const uint32_t*>(qb_row + d0 + 8) : 0u;
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
        const int kt = kstart + s * kDecTile + kw;    // logical index of this warp's first key
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
        // ---- mask keys outside each row's range (which includes keys >= L)
        if (kt + 15 > hi_all || kt < lo_all) {
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = kt + 8 * t + qc + (e & 1);
                    const bool keep = e < 2 ? (key >= lo_a && key <= hi_a) : (key >= lo_b && key <= hi_b);
                    if (!keep) sc[t][e] = -INFINITY;
                }
        }
        const bool tail = kt + 16 > L;
        if (tail) {
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
    for (int idx = threadIdx.x; idx < nrows * D; idx += kDecConsumers * 32) {
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

// One warp per (batch row, token, query head): merge the splits of that row.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ DecodeParams p,
                                                             __nv_bfloat16* out, float* lse, int B) {
    grid_dep_wait();   // the split kernel's partials
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= B * p.Sq * p.Hq) return;
    const int b = gw / (p.Sq * p.Hq), rem = gw % (p.Sq * p.Hq);
    const int s = rem / p.Hq, hq = rem % p.Hq;
    const int hk = hq / p.G, r = s * p.G + hq % p.G;
    int bc;
    const int L = dec_len(p, b, &bc, false);
    const int n = L > 0 ? (L + p.chunk - 1) / p.chunk : 0;
    const size_t base = (static_cast<size_t>(b) * p.Hkv + hk) * p.max_chunks;
    float mx = -INFINITY;
    for (int c = 0; c < n; ++c) mx = fmaxf(mx, p.part_lse[(base + c) * p.R + r]);
    constexpr int PER = D / 32;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    float wsum = 0.f;
    for (int c = 0; c < n; ++c) {
        const float lc = p.part_lse[(base + c) * p.R + r];
        const float f = (lc == -INFINITY) ? 0.f : expf(lc - mx);
        wsum += f;
        const float* src = p.part_o + ((base + c) * p.R + r) * D + lane * PER;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += f * src[e];
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    __nv_bfloat16* dst = out + ((static_cast<size_t>(b) * p.Sq + s) * p.Hq + hq) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
    if (lse != nullptr && lane == 0)
        lse[(static_cast<size_t>(b) * p.Hq + hq) * p.Sq + s] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

// One warp per (batch row, new token, KV head): write k_new / v_new into the cache at logical row
// cache_seqlens[b] + token.  Rows past what a sequence can hold are not written (and not attended).
template <int D>
__global__ void __launch_bounds__(256) kv_append_kernel(const __grid_constant__ DecodeParams p,
                                                        __nv_bfloat16* k_cache, __nv_bfloat16* v_cache,
                                                        const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                                        int B, int Sn) {
    grid_dep_launch();   // the split kernel may be scheduled; it waits for this grid before reading
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= static_cast<long long>(B) * Sn * p.Hkv) return;
    const int hk = static_cast<int>(gw % p.Hkv);
    const int s = static_cast<int>((gw / p.Hkv) % Sn);
    const int b = static_cast<int>(gw / (static_cast<long long>(p.Hkv) * Sn));
    int bc = b;
    if (p.page == 0 && p.batch_idx != nullptr) bc = __ldg(p.batch_idx + b);
    if (p.page == 0 && (bc < 0 || bc >= p.cache_batch)) return;   // reported by the split kernel
    const int pos = max(__ldg(p.seqlens + b), 0) + s;
    if (pos >= p.kmax) return;
    int phys;
    if (p.page > 0) {
        const int blk = __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks + pos / p.page);
        if (blk < 0 || blk >= p.cache_batch) {
            if (lane == 0) atomicCAS(p.status, 0, FA_ERR_INVALID_ARG);
            return;
        }
        phys = blk * p.page + pos % p.page;
    } else {
        phys = bc * p.kmax + pos;
    }
    constexpr int V4 = D / 8;   // 16-byte pieces per row
    if (lane < V4) {
        const size_t src = ((static_cast<size_t>(b) * Sn + s) * p.Hkv + hk) * D;
        const size_t dst = (static_cast<size_t>(phys) * p.Hkv + hk) * D;
        reinterpret_cast<uint4*>(k_cache + dst)[lane] = reinterpret_cast<const uint4*>(k_new + src)[lane];
        reinterpret_cast<uint4*>(v_cache + dst)[lane] = reinterpret_cast<const uint4*>(v_new + src)[lane];
    }
}

// ------------------------------------------------------------------------------------------ host side

int kvcache_chunk_limit(const KvCall& c) {
    return c.block_table != nullptr ? c.max_blocks_per_seq * c.cache_capacity : c.cache_capacity;
}

static int rows_per_kv_head(const KvCall& c) { return (c.Hq / c.Hkv) * c.Sq; }

int kvcache_validate(const KvCall& c, bool pointers) {
    if (pointers && (!c.q || !c.k_cache || !c.v_cache || !c.cache_seqlens || !c.out)) return FA_ERR_INVALID_ARG;
    if (c.B <= 0 || c.Sq <= 0 || c.cache_capacity <= 0 || c.cache_batch <= 0 || c.num_splits < 0)
        return FA_ERR_INVALID_ARG;
    if (c.Hq <= 0 || c.Hkv <= 0 || c.Hq % c.Hkv != 0) return FA_ERR_INVALID_ARG;
    if (!(c.scale > 0.f) || !isfinite(c.scale)) return FA_ERR_INVALID_ARG;
    if (c.D != 64 && c.D != 128 && c.D != 256) return FA_ERR_UNSUPPORTED;
    if (pointers) {
        if ((c.k_new == nullptr) != (c.v_new == nullptr)) return FA_ERR_INVALID_ARG;
        if ((c.seqlen_new > 0) != (c.k_new != nullptr)) return FA_ERR_INVALID_ARG;
    }
    if (c.seqlen_new < 0) return FA_ERR_INVALID_ARG;
    if (c.block_table != nullptr) {
        // README: page_block_size must be a multiple of 256
        if (c.cache_capacity % 256 != 0 || c.max_blocks_per_seq <= 0) return FA_ERR_INVALID_ARG;
        if (c.cache_batch_idx != nullptr) return FA_ERR_INVALID_ARG;   // batch index applies to contiguous caches
    }
    const long long kmax = c.block_table != nullptr ? static_cast<long long>(c.max_blocks_per_seq) * c.cache_capacity
                                                    : c.cache_capacity;
    if (kmax > (1LL << 30)) return FA_ERR_UNSUPPORTED;
    const long long rows_total = static_cast<long long>(c.cache_batch) * c.cache_capacity;
    if (rows_total >= 0x7fffffffLL || rows_total * c.Hkv * c.D > (1LL << 40)) return FA_ERR_UNSUPPORTED;
    if (static_cast<long long>(c.B) * c.Sq * c.Hq * c.D > (1LL << 40)) return FA_ERR_UNSUPPORTED;
    const long long grid_y = static_cast<long long>(c.Hkv) * ((rows_per_kv_head(c) + 15) / 16);
    if (grid_y > 65535 || c.B > 65535) return FA_ERR_UNSUPPORTED;
    if (!pointers) return FA_OK;
    auto a16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
    auto a4 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; };
    if (!a16(c.q) || !a16(c.k_cache) || !a16(c.v_cache) || !a16(c.out)) return FA_ERR_ALIGNMENT;
    if ((c.lse && !a16(c.lse)) || (c.k_new && (!a16(c.k_new) || !a16(c.v_new)))) return FA_ERR_ALIGNMENT;
    if (!a4(c.cache_seqlens) || (c.block_table && !a4(c.block_table)) || (c.cache_batch_idx && !a4(c.cache_batch_idx)))
        return FA_ERR_ALIGNMENT;
    return FA_OK;
}

int kvcache_chunk(const KvCall& c, int num_sms) {
    const int cap = kvcache_chunk_limit(c);
    const long long parallel = static_cast<long long>(c.B) * c.Hkv * ((rows_per_kv_head(c) + 15) / 16);
    long long ch;
    if (c.num_splits > 0) {
        ch = (static_cast<long long>(cap) + c.num_splits - 1) / c.num_splits;
    } else {
        // aim for about 6 waves of split CTAs (2 per SM), assuming caches half full on average, with at
        // least 512 keys per split: shorter splits spend a large share of their time starting up (B200, 64
        // rows x 8 KV heads of 1-2K keys: 256-key splits 4.0 TB/s, 512-key 4.9), while on long caches fewer,
        // longer splits cut the partial-output traffic (64 rows x 8 KV heads of 1-16K keys, 1 / 4 new tokens:
        // 16 splits of 1024 keys 6.38 / 5.54 TB/s, 8 splits 6.66 / 6.17, 6 splits 6.72 / 6.35)
        ch = parallel * cap / (2LL * 6 * 2 * num_sms);
        if (ch < 512) ch = 512;
    }
    ch = (ch + kDecTile - 1) / kDecTile * kDecTile;
    if (ch < kDecTile) ch = kDecTile;
    if (ch > cap) ch = (static_cast<long long>(cap) + kDecTile - 1) / kDecTile * kDecTile;
    return static_cast<int>(ch);
}

size_t kvcache_workspace_bytes(const KvCall& c, int chunk) {
    const size_t max_chunks = (static_cast<size_t>(kvcache_chunk_limit(c)) + chunk - 1) / chunk;
    const size_t rows = static_cast<size_t>(c.B) * c.Hkv * max_chunks * rows_per_kv_head(c);
    return ((rows * c.D * 4 + 255) & ~size_t(255)) + rows * 4;
}

template <int D>
static int run_decode(const KvCall& c, int chunk, void* workspace, const Device& dev, cudaStream_t stream) {
    const int kmax = kvcache_chunk_limit(c);
    DecodeParams p;
    p.q = static_cast<const __nv_bfloat16*>(c.q);
    p.seqlens = c.cache_seqlens;
    p.batch_idx = c.block_table != nullptr ? nullptr : c.cache_batch_idx;
    p.block_table = c.block_table;
    p.Hq = c.Hq;
    p.Hkv = c.Hkv;
    p.G = c.Hq / c.Hkv;
    p.Sq = c.Sq;
    p.R = p.G * c.Sq;
    p.row_blocks = (p.R + 15) / 16;
    p.kmax = kmax;
    p.chunk = chunk;
    p.max_chunks = (kmax + chunk - 1) / chunk;
    p.max_blocks = c.max_blocks_per_seq;
    p.page = c.block_table != nullptr ? c.cache_capacity : 0;
    p.cache_batch = c.cache_batch;
    p.rows_total = c.cache_batch * c.cache_capacity;
    p.seq_add = c.seqlen_new;
    p.wl = (c.window_left < 0 || c.window_left >= (1 << 30)) ? -1 : c.window_left;
    p.wr = (c.window_right < 0 || c.window_right >= (1 << 30)) ? -1 : c.window_right;
    if (c.causal) p.wr = 0;
    p.scale_log2 = c.scale * 1.4426950408889634f;
    p.timeout_ns = dev.timeout_ns;
    p.status = dev.status;
    const size_t rows = static_cast<size_t>(c.B) * c.Hkv * p.max_chunks * p.R;
    p.part_o = static_cast<float*>(workspace);
    p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((rows * D * 4 + 255) & ~size_t(255)));

    if (c.seqlen_new > 0) {
        const long long warps = static_cast<long long>(c.B) * c.seqlen_new * c.Hkv;
        const long long blocks = (warps + 7) / 8;
        if (blocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
        kv_append_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            p, static_cast<__nv_bfloat16*>(c.k_cache), static_cast<__nv_bfloat16*>(c.v_cache),
            static_cast<const __nv_bfloat16*>(c.k_new), static_cast<const __nv_bfloat16*>(c.v_new), c.B, c.seqlen_new);
        if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
    }

    alignas(64) CUtensorMap mk, mv;
    const uint64_t row_bytes = static_cast<uint64_t>(c.Hkv) * D * 2;
    if (!make_map_2d_bf16(&mk, c.k_cache, static_cast<uint64_t>(c.Hkv) * D, p.rows_total, row_bytes, 64, kDecTile))
        return FA_ERR_CUDA;
    if (!make_map_2d_bf16(&mv, c.v_cache, static_cast<uint64_t>(c.Hkv) * D, p.rows_total, row_bytes, 64, kDecTile))
        return FA_ERR_CUDA;
    constexpr size_t stage_bytes = 2 * kDecTile * D * 2;
    constexpr size_t merge_bytes = (kDecConsumers * 16 * D + 2 * kDecConsumers * 16) * 4;
    static_assert(merge_bytes <= kDecStages * stage_bytes, "merge buffer reuses the stage memory");
    const size_t smem = 1024 + kDecStages * stage_bytes + 2 * kDecStages * 8 + 16;
    static bool set[64] = {};
    auto kern = decode_split_kernel<D>;
    if (!set[dev.id & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess)
            return FA_ERR_CUDA;
        set[dev.id & 63] = true;
    }
    dim3 grid(p.max_chunks, c.Hkv * p.row_blocks, c.B);
    prof_before(2, stream);
    if (launch_dependent(kern, grid, dim3((kDecConsumers + 1) * 32), smem, stream, mk, mv, p) != cudaSuccess)
        return FA_ERR_CUDA;
    prof_after(2, stream);
    const long long warps = static_cast<long long>(c.B) * c.Sq * c.Hq;
    if (launch_dependent(decode_combine_kernel<D>, dim3(static_cast<unsigned>((warps + 3) / 4)), dim3(128), 0, stream,
                         p, static_cast<__nv_bfloat16*>(c.out), c.lse, c.B) != cudaSuccess)
        return FA_ERR_CUDA;
    return FA_OK;
}

int kvcache_launch(const KvCall& c, int chunk, void* workspace, const Device& dev, cudaStream_t stream) {
    switch (c.D) {
        case 64: return run_decode<64>(c, chunk, workspace, dev, stream);
        case 128: return run_decode<128>(c, chunk, workspace, dev, stream);
        case 256: return run_decode<256>(c, chunk, workspace, dev, stream);
        default: return FA_ERR_UNSUPPORTED;
    }
}

}  // namespace fa

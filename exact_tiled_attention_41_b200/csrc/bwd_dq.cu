// bwd_dq.cu -- dQ of the deterministic backward on sm_100a.
//
// flash-attention README, flash_attn_func docstring: the backward has a
// deterministic variant (slower, more memory; the forward is always
// deterministic).  The default backward accumulates dQ with float32 reduce-adds
// from key-tile-stationary CTAs, whose order varies between runs.  With the
// deterministic option the main kernel leaves dQ out and this kernel computes
// it query-tile stationary: one CTA holds a 128-row tile of Q and dO and walks
// its KV tiles in increasing order,
//   S_j = Q K_j^T,  dP_j = dO V_j^T,  P_j = exp2(S_j scale log2(e) - LSE2),
//   dS_j = P_j (dP_j - Delta),  dQ = scale sum_j dS_j K_j,
// summing into one tensor-memory accumulator, so every run adds the same
// numbers in the same order.  LSE2 (= LSE log2(e), +inf for a row without keys)
// and Delta = rowsum(dO O) come from the backward's preprocess.
//
// Roles (12 warps, one persistent CTA per SM):
//   warps 0-7  two compute warpgroups, thread = query row; warpgroup g owns key
//              columns [g BK/2, (g+1) BK/2) of S_j and dP_j.  It reads its dP_j
//              half first (so dP_{j+1} can be computed), then S_j in 32-column
//              chunks, and writes dS_j as bf16 pairs into the low columns of its
//              own S half (columns it has already read); epilogue: its half of
//              the dQ columns, scaled and rounded to bf16, straight to dq.
//   warp 8     TMA producer: Q, dO once per unit; K and V through rings of KST and VST
//              stages.  K must have >= 2 stages: K_j is still read by dQ_j after S_{j+1}
//              has been issued; V is only read by dP_j.
//   warp 9     tensor memory and every tcgen05 MMA.  Per KV tile j:
//              S_j into S buffer j%2; dP_j once the compute warps hold dP_{j-1};
//              dQ += dS_{j-1} K_{j-1} once dS_{j-1} is written (A from tensor memory).
//   warps 10-11 idle.
//   tensor memory: S0 [0,BK) | S1 [BK,2BK) | dP [2BK,3BK) | dQ [3BK,3BK+D)
#include "internal.h"
#include "sm100.cuh"

#include <math.h>

namespace fa {

struct DqParams {
    __nv_bfloat16* dq;
    const float* lse2;      // [Hq][Tq]
    const float* delta;     // [Hq][Tq]
    const int32_t* cu_q;
    const int32_t* cu_k;
    int num_seqs, Sq, Sk, Tq, Tk, Hq, Hkv, group;
    int m_blocks, num_units;
    float scale, scale_log2;
    int wl, wr;             // window sides, -1 = unbounded; a causal mask is wr = 0
    unsigned long long timeout_ns;
    int* status;
};

struct DqUnit {
    int b, h, q_start, k_start, Lq, Lk, q0, kv0, n_kv;
    bool skip;
};

template <int BK>
__device__ __forceinline__ DqUnit decode_dq_unit(const DqParams& p, int u) {
    DqUnit t;
    const int per_m = p.num_seqs * p.Hq;
    const int m = p.m_blocks - 1 - u / per_m;   // under a causal mask the last query tiles see the most keys
    const int r = u % per_m;
    t.b = r / p.Hq;
    t.h = r % p.Hq;
    if (p.cu_q != nullptr) {
        t.q_start = max(__ldg(p.cu_q + t.b), 0);
        t.k_start = max(__ldg(p.cu_k + t.b), 0);
        t.Lq = max(min(min(__ldg(p.cu_q + t.b + 1) - t.q_start, p.Tq - t.q_start), 1 << 30), 0);
        t.Lk = max(min(min(__ldg(p.cu_k + t.b + 1) - t.k_start, p.Tk - t.k_start), 1 << 30), 0);
    } else {
        t.q_start = t.b * p.Sq;
        t.Lq = p.Sq;
        t.k_start = t.b * p.Sk;
        t.Lk = p.Sk;
    }
    t.q0 = m * 128;
    t.skip = t.q0 >= t.Lq;
    t.kv0 = 0;
    t.n_kv = 0;
    if (!t.skip) {
        // keys reachable from rows q0 .. row_end-1 (lengths <= 2^30, window sides < 2^30: int32 is exact)
        const int row_end = min(t.q0 + 128, t.Lq);
        const int off = t.Lk - t.Lq;
        int lo = 0, hi = t.Lk - 1;
        if (p.wl >= 0) lo = max(lo, t.q0 + off - p.wl);
        if (p.wr >= 0) hi = min(hi, row_end - 1 + off + p.wr);
        if (hi >= lo) {
            t.kv0 = lo / BK;
            t.n_kv = hi / BK + 1 - t.kv0;
        }
    }
    return t;
}

template <int D, int BK, int KST, int VST>
struct DqCfg {
    static constexpr int BM = 128;
    static constexpr int NCHUNK = D / 64;
    static constexpr int HALF = BK / 2;                   // key columns per compute warpgroup
    static constexpr uint32_t T_BYTES = BM * D * 2;       // a Q or dO tile
    static constexpr uint32_t KV_BYTES = BK * D * 2;
    // q_full, q_empty, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST],
    // s_full[2], dp_full, dp_free, ds_full[2], dq_full, dq_empty
    static constexpr int B1 = 2 + 2 * KST + 2 * VST;
    static constexpr int NUM_BARS = B1 + 8;
    // 2 KB per compute warp to write the dQ rows 8 at a time, where shared memory has room for it
    static constexpr bool STAGE = 1024 + 2 * T_BYTES + (KST + VST) * KV_BYTES + 8 * 2048 + NUM_BARS * 8 + 16 <= 232448;
    static constexpr uint32_t STG_BYTES = STAGE ? 8 * 2048 : 0;
    static constexpr size_t SMEM = 1024 + 2 * T_BYTES + (KST + VST) * KV_BYTES + STG_BYTES + NUM_BARS * 8 + 16;
    static_assert(KST >= 2 && VST >= 1, "K_j is read by dQ_j after S_{j+1} is issued");
    static constexpr int THREADS = 384;
    static constexpr uint32_t S_COL(int s) { return s * BK; }
    static constexpr uint32_t DP_COL = 2 * BK, DQ_COL = 3 * BK;
    static_assert(3 * BK + D <= 512, "tensor memory budget");
    static_assert(HALF % 32 == 0 && D % 64 == 0, "tile shape");
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <int D, int BK, int KST, int VST>
__global__ void __launch_bounds__(384, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const __grid_constant__ DqParams p) {
    using C = DqCfg<D, BK, KST, VST>;
    constexpr int BM = C::BM;
    constexpr int HALF = C::HALF;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sDO = sQ + C::T_BYTES;
    uint8_t* sK = sDO + C::T_BYTES;
    uint8_t* sV = sK + KST * C::KV_BYTES;
    uint8_t* sStg = sV + VST * C::KV_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sStg + C::STG_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const uint32_t b0 = smem_u32(bars);
    const uint32_t q_full = b0, q_empty = b0 + 8;
    auto k_full = [&](int s) { return b0 + 8u * (2 + s); };
    auto k_empty = [&](int s) { return b0 + 8u * (2 + KST + s); };
    auto v_full = [&](int s) { return b0 + 8u * (2 + 2 * KST + s); };
    auto v_empty = [&](int s) { return b0 + 8u * (2 + 2 * KST + VST + s); };
    const uint32_t b1 = b0 + 8u * C::B1;
    auto s_full = [&](int s) { return b1 + 8u * s; };
    const uint32_t dp_full = b1 + 16, dp_free = b1 + 24;
    auto ds_full = [&](int s) { return b1 + 32 + 8u * s; };
    const uint32_t dq_full = b1 + 48, dq_empty = b1 + 56;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr int PRODUCER = 8, MMA = 9;

    if (threadIdx.x == 0) {
        mbar_init(bars + 0, 1);
        mbar_init(bars + 1, 1);
        for (int s = 0; s < 2 * KST + 2 * VST; ++s) mbar_init(bars + 2 + s, 1);
        mbar_init(bars + C::B1 + 0, 1);     // s_full[0]
        mbar_init(bars + C::B1 + 1, 1);     // s_full[1]
        mbar_init(bars + C::B1 + 2, 1);     // dp_full
        mbar_init(bars + C::B1 + 3, 256);   // dp_free: every compute thread holds its dP values
        mbar_init(bars + C::B1 + 4, 256);   // ds_full[0]
        mbar_init(bars + C::B1 + 5, 256);   // ds_full[1]
        mbar_init(bars + C::B1 + 6, 1);     // dq_full
        mbar_init(bars + C::B1 + 7, 256);   // dq_empty
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == PRODUCER && lane == 0) {
        tma_prefetch_map(&tmQ);
        tma_prefetch_map(&tmDO);
        tma_prefetch_map(&tmK);
        tma_prefetch_map(&tmV);
    }
    if (warp == MMA) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Watch w{abort_flag, p.status, p.timeout_ns};

    if (warp == PRODUCER) {
        if (lane == 0) {
            uint32_t kv_it = 0, q_it = 0;
            bool ok = true;
            for (int k = 0, u = snake_unit(0, p.num_units); u >= 0 && ok; u = snake_unit(++k, p.num_units)) {
                if (u >= p.num_units) continue;
                const DqUnit t = decode_dq_unit<BK>(p, u);
                if (t.skip || t.n_kv == 0) continue;
                const int hk = t.h / p.group;
                if (q_it > 0 && !mbar_wait(q_empty, (q_it - 1) & 1, w)) break;
                mbar_arrive_expect_tx(q_full, 2 * C::T_BYTES);
#pragma unroll
                for (int c = 0; c < C::NCHUNK; ++c) {
                    tma_load_3d(smem_u32(sQ + c * BM * 128), &tmQ, q_full, c * 64, t.h, t.q_start + t.q0);
                    tma_load_3d(smem_u32(sDO + c * BM * 128), &tmDO, q_full, c * 64, t.h, t.q_start + t.q0);
                }
                ++q_it;
                for (int j = 0; j < t.n_kv; ++j, ++kv_it) {
                    const int st = kv_it % KST, sv = kv_it % VST;
                    const uint32_t n = kv_it / KST, nv = kv_it / VST;
                    const int krow = t.k_start + (t.kv0 + j) * BK;
                    if (n > 0 && !mbar_wait(k_empty(st), (n - 1) & 1, w)) { ok = false; break; }
                    mbar_arrive_expect_tx(k_full(st), C::KV_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c)
                        tma_load_3d(smem_u32(sK + st * C::KV_BYTES + c * BK * 128), &tmK, k_full(st), c * 64, hk, krow);
                    if (nv > 0 && !mbar_wait(v_empty(sv), (nv - 1) & 1, w)) { ok = false; break; }
                    mbar_arrive_expect_tx(v_full(sv), C::KV_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c)
                        tma_load_3d(smem_u32(sV + sv * C::KV_BYTES + c * BK * 128), &tmV, v_full(sv), c * 64, hk, krow);
                }
            }
        }
        __syncwarp();
    } else if (warp == MMA) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BK, false, false);   // S, dP: both K-major
            constexpr uint32_t idesc_dq = idesc_bf16_f32(BM, D, false, true);    // dQ: K tile N-major
            // [128 x D] tile times a [BK x D] tile transposed, into tensor-memory column dcol; descriptor
            // low words advanced by constant offsets >> 4 (one add per operand per MMA)
            auto issue_ss = [&](uint32_t dcol, const uint8_t* a, const uint8_t* b) {
                const uint32_t ad = sdesc_lo(smem_u32(a), 16), bd = sdesc_lo(smem_u32(b), 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss_lo(tmem + dcol, ad + (((kk >> 2) * BM * 128 + (kk & 3) * 32) >> 4),
                               bd + (((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4), idesc_s, kk > 0 ? 1u : 0u);
            };
            // dQ (+)= dS K: dS for keys [16 kk, 16 kk + 16) sits in the S half of the warpgroup that owns
            // those keys, at (key offset inside the half) / 2 packed columns from the half's start
            auto issue_dq = [&](int sb, int st, bool acc) {
                const uint32_t kd = sdesc_lo(smem_u32(sK + st * C::KV_BYTES), BK * 128);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const int k0 = kk * 16;
                    const uint32_t acol = C::S_COL(sb) + (k0 / HALF) * HALF + (k0 % HALF) / 2;
                    umma_ts_lo(tmem + C::DQ_COL, tmem + acol, kd + ((kk * 16 * 128) >> 4), idesc_dq,
                               (acc || kk > 0) ? 1u : 0u);
                }
            };
            uint32_t kv_it = 0, q_it = 0, gt = 0, unit_it = 0;
            bool ok = true;
            for (int k = 0, u = snake_unit(0, p.num_units); u >= 0 && ok; u = snake_unit(++k, p.num_units)) {
                if (u >= p.num_units) continue;
                const DqUnit t = decode_dq_unit<BK>(p, u);
                if (t.skip || t.n_kv == 0) continue;
                if (!mbar_wait(q_full, q_it & 1, w)) break;
                ++q_it;
                bool first_dq = true;
                // dQ of global tile g (its S buffer g % 2, its KV stage st)
                auto dq_step = [&](uint32_t g, int st, bool acc) -> bool {
                    if (!mbar_wait(ds_full(g & 1), (g >> 1) & 1, w)) return false;
                    if (first_dq) {
                        // the previous unit's dQ must have been read out before it is overwritten
                        if (unit_it > 0 && !mbar_wait(dq_empty, (unit_it - 1) & 1, w)) return false;
                        first_dq = false;
                    }
                    tc_fence_after();
                    issue_dq(g & 1, st, acc);
                    umma_commit(k_empty(st));
                    return true;
                };
                for (int j = 0; j < t.n_kv && ok; ++j) {
                    const uint32_t g = gt + j;
                    const uint32_t it = kv_it + j;
                    const int st = it % KST, sv = it % VST;
                    if (!mbar_wait(k_full(st), (it / KST) & 1, w)) { ok = false; break; }
                    tc_fence_after();
                    issue_ss(C::S_COL(g & 1), sQ, sK + st * C::KV_BYTES);
                    umma_commit(s_full(g & 1));
                    if (!mbar_wait(v_full(sv), (it / VST) & 1, w)) { ok = false; break; }
                    if (g > 0 && !mbar_wait(dp_free, (g - 1) & 1, w)) { ok = false; break; }
                    tc_fence_after();
                    issue_ss(C::DP_COL, sDO, sV + sv * C::KV_BYTES);
                    umma_commit(dp_full);
                    umma_commit(v_empty(sv));
                    if (j + 1 == t.n_kv) umma_commit(q_empty);   // Q and dO are read by S and dP only
                    if (j > 0 && !dq_step(g - 1, (it - 1) % KST, j > 1)) { ok = false; break; }
                }
                if (!ok) break;
                const uint32_t it_last = kv_it + t.n_kv - 1;
                if (!dq_step(gt + t.n_kv - 1, it_last % KST, t.n_kv > 1)) break;
                umma_commit(dq_full);
                kv_it += t.n_kv;
                gt += t.n_kv;
                ++unit_it;
            }
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------- compute warpgroups (thread = query row)
        const int gw = warp >> 2;                  // key columns [gw HALF, gw HALF + HALF) of each tile
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lb = tmem_lane_base(wq);
        const float c2 = p.scale_log2;
        const float2 c2v = make_float2(c2, c2);
        uint32_t gt = 0, unit_it = 0;
        bool ok = true;
        for (int k = 0, u = snake_unit(0, p.num_units); u >= 0 && ok; u = snake_unit(++k, p.num_units)) {
            if (u >= p.num_units) continue;
            const DqUnit t = decode_dq_unit<BK>(p, u);
            if (t.skip) continue;
            const int row = t.q0 + r;
            const bool valid = row < t.Lq;
            __nv_bfloat16* dst = p.dq + (static_cast<size_t>(t.q_start + row) * p.Hq + t.h) * D + gw * (D / 2);
            if (t.n_kv == 0) {
                if (valid) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    for (int c = 0; c < D / 16; ++c) reinterpret_cast<uint4*>(dst)[c] = z;
                }
                continue;
            }
            const size_t si = static_cast<size_t>(t.h) * p.Tq + t.q_start + row;
            const float nl = valid ? -__ldg(p.lse2 + si) : -INFINITY;   // rows past the sequence: P = 0
            const float nd = valid ? -__ldg(p.delta + si) : 0.f;
            const float2 nl2 = make_float2(nl, nl), nd2 = make_float2(nd, nd);
            int key_lo = 0, key_hi = t.Lk - 1;
            if (p.wl >= 0) key_lo = max(0, row + (t.Lk - t.Lq) - p.wl);
            if (p.wr >= 0) key_hi = min(key_hi, row + (t.Lk - t.Lq) + p.wr);
            for (int j = 0; j < t.n_kv; ++j) {
                const uint32_t g = gt + j;
                const uint32_t tS = tmem + lb + C::S_COL(g & 1) + gw * HALF;
                bool got = mbar_wait(s_full(g & 1), (g >> 1) & 1, w);
                got = got && mbar_wait(dp_full, g & 1, w);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                uint32_t dp[HALF / 32][32];
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc) tmem_ld32(tmem + lb + C::DP_COL + gw * HALF + cc * 32, dp[cc]);
                tmem_ld_wait_tie(dp[0]);
#pragma unroll
                for (int cc = 1; cc < HALF / 32; ++cc) reg_tie(dp[cc]);
                tc_fence_before();
                mbar_arrive(dp_free);
                const int kbase = (t.kv0 + j) * BK + gw * HALF;   // key index of this thread's first column
                const bool any_mask = __any_sync(0xffffffffu, kbase + HALF - 1 > key_hi || kbase < key_lo);
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc) {
                    uint32_t sv[32];
                    tmem_ld32(tS + cc * 32, sv);
                    tmem_ld_wait_tie(sv);
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float2 x = ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2v, nl2);
                        float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                        if (any_mask) {
                            const int kj = kbase + cc * 32 + e;
                            pr.x = (kj >= key_lo && kj <= key_hi) ? pr.x : 0.f;
                            pr.y = (kj + 1 >= key_lo && kj + 1 <= key_hi) ? pr.y : 0.f;
                        }
                        const float2 dv = fadd2(make_float2(__uint_as_float(dp[cc][e]), __uint_as_float(dp[cc][e + 1])), nd2);
                        const float2 ds = fmul2(pr, dv);
                        pk[e / 2] = pack_bf16x2(ds.x, ds.y);
                    }
                    // packed columns [16 cc, 16 cc + 16) of the half: S columns already read
                    tmem_st16(tS + cc * 16, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(ds_full(g & 1));
            }
            if (!ok) break;
            gt += t.n_kv;
            // ------------------------------------------------ epilogue: dq = bf16(scale * dQ), this warpgroup's half
            if (!mbar_wait(dq_full, unit_it & 1, w)) { ok = false; break; }
            ++unit_it;
            tc_fence_after();
            const float2 sc = make_float2(p.scale, p.scale);
#pragma unroll 1
            for (int cc = 0; cc < D / 64; ++cc) {
                uint32_t ra[32];
                tmem_ld32(tmem + lb + C::DQ_COL + gw * (D / 2) + cc * 32, ra);
                tmem_ld_wait_tie(ra);
                if constexpr (C::STAGE) {
                    uint8_t* stg = sStg + warp * 2048;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 v = fmul2(make_float2(__uint_as_float(ra[8 * q + 2 * e]), __uint_as_float(ra[8 * q + 2 * e + 1])), sc);
                            pk[e] = pack_bf16x2(v.x, v.y);
                        }
                        stg_put(stg, q, pk[0], pk[1], pk[2], pk[3]);
                    }
                    stg_flush(stg, reinterpret_cast<uint8_t*>(dst + cc * 32), static_cast<long long>(p.Hq) * D * 2,
                              min(max(t.Lq - (t.q0 + wq * 32), 0), 32));
                } else {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 v = fmul2(make_float2(__uint_as_float(ra[2 * e]), __uint_as_float(ra[2 * e + 1])), sc);
                        pk[e] = pack_bf16x2(v.x, v.y);
                    }
                    if (valid) {
                        uint4* o4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e) o4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(dq_empty);
        }
    }

    __syncthreads();
    if (*abort_flag) {
        // give tensor-core and TMA work already issued time to land before freeing
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) {
        }
    }
    if (warp == MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, int BK, int KST, int VST>
static int run_dq(const Problem& pr, const void* dout, const float* lse2, const float* delta, void* dq,
                  const Device& dev, cudaStream_t stream) {
    using C = DqCfg<D, BK, KST, VST>;
    alignas(64) CUtensorMap mq, mdo, mk, mv;
    const uint64_t rq = static_cast<uint64_t>(pr.Hq) * D * 2, rk = static_cast<uint64_t>(pr.Hkv) * D * 2;
    if (!make_map_3d_bf16(&mq, pr.q, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, C::BM)) return 5;
    if (!make_map_3d_bf16(&mdo, dout, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, C::BM)) return 5;
    if (!make_map_3d_bf16(&mk, pr.k, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, BK)) return 5;
    if (!make_map_3d_bf16(&mv, pr.v, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, BK)) return 5;

    DqParams p;
    p.dq = static_cast<__nv_bfloat16*>(dq);
    p.lse2 = lse2;
    p.delta = delta;
    p.cu_q = pr.cu_q;
    p.cu_k = pr.cu_k;
    p.num_seqs = pr.num_seqs;
    p.Sq = pr.Sq;
    p.Sk = pr.Sk;
    p.Tq = pr.Tq;
    p.Tk = pr.Tk;
    p.Hq = pr.Hq;
    p.Hkv = pr.Hkv;
    p.group = pr.Hq / pr.Hkv;
    p.m_blocks = (pr.Sq + C::BM - 1) / C::BM;
    const long long units = static_cast<long long>(p.m_blocks) * pr.num_seqs * pr.Hq;
    if (units > 0x7fffffffLL) return 2;
    p.num_units = static_cast<int>(units);
    p.scale = pr.scale;
    p.scale_log2 = pr.scale * 1.4426950408889634f;
    p.wl = pr.wl;
    p.wr = pr.wr;
    p.timeout_ns = dev.timeout_ns;
    p.status = dev.status;
    if (p.num_units == 0) return 0;

    auto kern = dq_kernel<D, BK, KST, VST>;
    static bool attr_set[64] = {};
    if (!attr_set[dev.id & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM)) !=
            cudaSuccess)
            return 5;
        attr_set[dev.id & 63] = true;
    }
    const int grid = p.num_units < dev.num_sms ? p.num_units : dev.num_sms;
    prof_before(3, stream);
    kern<<<grid, C::THREADS, C::SMEM, stream>>>(mq, mdo, mk, mv, p);
    prof_after(3, stream);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 5;
}

int launch_bwd_dq(const Problem& pr, const void* dout, const float* lse2, const float* delta, void* dq,
                  const Device& dev, cudaStream_t stream) {
    switch (pr.D) {
        case 64: return run_dq<64, 128, 3, 3>(pr, dout, lse2, delta, dq, dev, stream);
        case 128: return run_dq<128, 128, 2, 2>(pr, dout, lse2, delta, dq, dev, stream);
        case 256: return run_dq<256, 64, 2, 1>(pr, dout, lse2, delta, dq, dev, stream);
        default: return 2;
    }
}

}  // namespace fa

// bwd256.cu -- backward main kernel and dQ convert for head dim 256.
//
// Same mathematics as bwd.cu (recompute P from the stored LSE; dV = P^T dO,
// dP = dO V^T, dS = P (dP - Delta), dQ = scale dS K, dK = scale dS^T Q), with a
// tiling that fits tensor memory at D = 256: dV and dK of a 128-key tile would
// take all 512 columns, so each work unit owns one half (128 columns) of the
// head dimension of dV and dK.  The unit still contracts S^T = K Q^T and
// dP^T = V dO^T over the full head dimension (the two halves recompute them),
// and emits the matching half of dQ.  Query tiles are 64 rows so that K, V
// (128 x 256 each), a ring of five 16 KB slots for the Q and dO tiles (see Cfg)
// and dS^T fit shared memory.
//   tensor memory: dV half [0,128) | dK half [128,256) | S^T [256,320) |
//                  dP^T [320,384) | dQ^T half [384,448); after the gradient step each
//                  32-query half's packed P^T and dS^T sit in that half's S^T columns
//   dQ^T = K_half^T dS^T has the head dimension on the 128 lanes, so the dQ
//   warpgroup's atomics cover 32 consecutive head-dim floats per warp and the
//   accumulator is laid out [Hq][Tq][256].
// Roles: warps 0-3 compute (thread = key row), 4-7 dQ (thread = head-dim row),
// 8 producer, 9 MMA issuer, 10-11 idle; registers redistributed with setmaxnreg.
// With DQ = false (the deterministic backward) dQ is left to the query-tile-stationary
// pass of bwd_dq.cu: no dQ product, no reduce-adds, no convert.
#include "internal.h"
#include "sm100.cuh"

#include <math.h>

#ifndef FA_B256_VEC_DQ
#define FA_B256_VEC_DQ 1
#endif

namespace fa {

namespace {

constexpr int D = 256;

struct B256Params {
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* dq_acc;          // [Hq][Tq][256]
    const float* lse2;      // [Hq][Tq]
    const float* delta;     // [Hq][Tq]
    const int32_t* cu_q;
    const int32_t* cu_k;
    int num_seqs, Sq, Sk, Tq, Tk, Hq, Hkv, group;
    int num_units;
    float scale, scale_log2;
    int wl, wr;             // window sides, -1 = unbounded; a causal mask is wr = 0
    int n_blocks, chunk;    // key tiles per sequence; (sequence, KV head) groups per chunk of the unit list
    int* counter;           // unit counter of the dynamic schedule (zeroed by the preprocess kernel)
    unsigned long long timeout_ns;
    int* status;
};

struct U256 {
    int b, hk, hh, q_start, k_start, Lq, Lk, n0, m_start, n_m, n_it;
    bool skip;
};

// Unit u: chunks of p.chunk (sequence, KV head) groups; inside a chunk, key tile by key tile (the
// first tiles have the most work under a causal mask) over the chunk's groups and both head-dim halves.
__device__ __forceinline__ U256 decode_u256(const B256Params& p, int u) {
    U256 t;
    const int groups = p.num_seqs * p.Hkv;
    const int per_chunk = p.chunk * p.n_blocks * 2;
    const int c = u / per_chunk;
    const int g0 = c * p.chunk;
    const int cs = min(p.chunk, groups - g0);
    const int idx = u - c * per_chunk;
    const int n = idx / (2 * cs);       // key tile
    int r = idx % (2 * cs);
    t.hh = r & 1;                       // the two halves of a key tile are taken one after the other
    r = g0 + (r >> 1);
    t.b = r / p.Hkv;
    t.hk = r % p.Hkv;
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
    t.n0 = n * 128;
    t.skip = t.n0 >= t.Lk;
    // query rows that see some key of the tile (key j allowed for row i iff j - off - wr <= i <= j - off + wl)
    // (lengths <= 2^30 and window sides < 2^30 keep every term inside int32)
    const int off = t.Lk - t.Lq;
    int r_lo = 0, r_hi = t.Lq - 1;
    if (p.wr >= 0) r_lo = max(r_lo, t.n0 - off - p.wr);
    if (p.wl >= 0) r_hi = min(r_hi, min(t.n0 + 127, t.Lk - 1) - off + p.wl);
    if (t.skip || r_hi < r_lo) {
        t.m_start = 0;
        t.n_m = 0;
    } else {
        t.m_start = r_lo / 64;
        t.n_m = r_hi / 64 + 1 - t.m_start;
    }
    t.n_it = t.n_m * p.group;
    return t;
}

// Q and dO of a 64-row query tile arrive as four pairs of [64 x 64] boxes (two head-dim chunks each),
// in this order: Q of the other half, dO of the other half, Q of the unit's half, dO of the unit's half.
// The pairs pass through a ring of NSLOT 16 KB slots and each slot is released by the last product that
// reads it (S^T; dP^T; dK; dV), so the next tile's S^T operands and half of its dP^T operands load
// while the current tile's gradient step runs.
struct Cfg {
    static constexpr uint32_t KV_BYTES = 128 * D * 2;    // 64 KB, four [128 x 64] boxes
    static constexpr uint32_t BOX_BYTES = 64 * 64 * 2, PAIR_BYTES = 2 * BOX_BYTES;
    static constexpr uint32_t NSLOT = 5;
    static constexpr uint32_t OFF_K = 0, OFF_V = KV_BYTES, OFF_RING = 2 * KV_BYTES,
                              OFF_DS = OFF_RING + NSLOT * PAIR_BYTES,   // dS^T [128 keys][64 queries], 16 KB
                              OFF_STAT = OFF_DS + 128 * 128,            // [2][-LSE2 x 64 | -Delta x 64]
                              OFF_BAR = OFF_STAT + 2 * 128 * 4;
    // kv_full, kv_empty | slot_full[NSLOT] | slot_empty[NSLOT] | stat_full[2] | stat_empty[2] |
    // s_full, p_full, dq_full, dq_empty, dkv_full, dv_done | unit feed
    static constexpr int BAR_SLOT_FULL = 2, BAR_SLOT_EMPTY = 2 + NSLOT, BAR_STAT_FULL = 2 + 2 * NSLOT,
                         BAR_STAT_EMPTY = BAR_STAT_FULL + 2, BAR_S_FULL = BAR_STAT_EMPTY + 2, BAR_FEED = BAR_S_FULL + 6;
    static constexpr int NUM_BARS = BAR_FEED + 2 * kFeedSlots;
    static constexpr size_t SMEM = OFF_BAR + NUM_BARS * 8 + 16 + 4 * kFeedSlots;
    static_assert(SMEM <= 232448, "shared memory per block");
    static constexpr uint32_t COL_DV = 0, COL_DK = 128, COL_S = 256, COL_DP = 320, COL_DQ = 384;
    // packed P^T of queries [16 kk, 16 kk + 16) (8 columns of bf16 pairs): compute warpgroup kk / 2 wrote
    // them into the first 16 of the 32 S^T columns it read; dS^T of the same queries sits 16 columns later
    static constexpr uint32_t COL_PK(int kk) { return COL_S + 32 * (kk >> 1) + 8 * (kk & 1); }
    // 16 warps: 0-7 two compute warpgroups (query columns 0-31 / 32-63), 8-11 dQ warpgroup, 12 producer,
    // 13 and 14 the two MMA issuers, 15 idle.  Registers: launch at 128 per thread (512 x 128 = 65536); the
    // producer / issuer warpgroup gives 40 per thread to the dQ warpgroup.  The host checks the launch count.
    static constexpr int THREADS = 512, LAUNCH_REGS = 128, COMPUTE_REGS = 128, DQ_REGS = 168, OTHER_REGS = 88;
    static_assert(2 * 128 * COMPUTE_REGS + 128 * DQ_REGS + 128 * OTHER_REGS <= THREADS * LAUNCH_REGS, "register split");
};

// One issuing thread takes about 54 cycles per 16-deep MMA, more than the tensor core needs for the 128 x 64
// products here, so two threads issue: A takes S^T, dQ^T and dK (the Q pairs are its operands), B takes dP^T
// and dV (the dO pairs).  Each releases the ring slots of its own pairs.  S^T of a tile overwrites the
// packed P^T and dS^T of the previous tile (in the S^T columns), read by B's dV and A's own dK, so A waits
// for B's previous dV there (dv_done).
template <bool DQ>
__global__ void __launch_bounds__(512, 1)
    bwd256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ B256Params p) {
    using C = Cfg;
    extern __shared__ __align__(1024) uint8_t smem[];
    float* sStat = reinterpret_cast<float*>(smem + C::OFF_STAT);  // [2][128]: -LSE2 of 64 rows, -Delta of 64 rows
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* feed_slot = reinterpret_cast<int*>(tmem_slot + 4);
    const uint32_t b0 = smem_u32(bars);
    const UnitFeed feed{feed_slot, b0 + 8u * C::BAR_FEED, b0 + 8u * (C::BAR_FEED + kFeedSlots)};
    const uint32_t kv_full = b0, kv_empty = b0 + 8;
    auto slot_full = [&](uint32_t s) { return b0 + 8u * (C::BAR_SLOT_FULL + s); };
    auto slot_empty = [&](uint32_t s) { return b0 + 8u * (C::BAR_SLOT_EMPTY + s); };
    auto stat_full = [&](uint32_t s) { return b0 + 8u * (C::BAR_STAT_FULL + s); };
    auto stat_empty = [&](uint32_t s) { return b0 + 8u * (C::BAR_STAT_EMPTY + s); };
    const uint32_t s_full = b0 + 8u * C::BAR_S_FULL, p_full = s_full + 8, dq_full = s_full + 16,
                   dq_empty = s_full + 24, dkv_full = s_full + 32, dv_done = s_full + 40;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int PRODUCER = 12, MMA_A = 13, MMA_B = 14;

    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0) atomicCAS(p.status, 0, 2);
        return;
    }
    if (threadIdx.x == 0) {
        mbar_init(bars + 0, 1);                                      // kv_full
        mbar_init(bars + 1, 2);                                      // kv_empty: both issuers
        for (int s = 0; s < static_cast<int>(C::NSLOT); ++s) {
            mbar_init(bars + C::BAR_SLOT_FULL + s, 1);               // expect-tx arrival of the pair's loads
            mbar_init(bars + C::BAR_SLOT_EMPTY + s, 1);              // commit of the pair's last reader
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bars + C::BAR_STAT_FULL + s, 32);              // the producer's 32 lanes
            mbar_init(bars + C::BAR_STAT_EMPTY + s, 8);              // one arrival per compute warp
        }
        mbar_init(bars + C::BAR_S_FULL + 0, 2);                      // s_full: S^T (A) and dP^T (B)
        mbar_init(bars + C::BAR_S_FULL + 1, 256);                    // p_full: both compute warpgroups
        mbar_init(bars + C::BAR_S_FULL + 2, 1);                      // dq_full
        mbar_init(bars + C::BAR_S_FULL + 3, 128);                    // dq_empty
        mbar_init(bars + C::BAR_S_FULL + 4, 2);                      // dkv_full: last dK (A) and dV (B)
        mbar_init(bars + C::BAR_S_FULL + 5, 1);                      // dv_done
        for (int s = 0; s < kFeedSlots; ++s) {
            mbar_init(bars + C::BAR_FEED + s, 1);                              // unit published
            mbar_init(bars + C::BAR_FEED + kFeedSlots + s, DQ ? 14 : 10);      // read by the issuers, compute (, dQ) warps
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == PRODUCER && lane == 0) {
        tma_prefetch_map(&tmQ);
        tma_prefetch_map(&tmK);
        tma_prefetch_map(&tmV);
        tma_prefetch_map(&tmDO);
    }
    if (warp == MMA_A) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Watch w{abort_flag, p.status, p.timeout_ns};
    const int G = p.group;

    if (warp >= 12) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::OTHER_REGS));
        if (warp == PRODUCER) {
            uint32_t unit_it = 0, q_it = 0;
            bool ok = true;
            // head-dim chunks c0, c0 + 1 of a 64-row tile of Q or dO into the ring slot of pair number px
            auto load_pair = [&](uint32_t px, const CUtensorMap* map, int c0, int h, int row) -> bool {
                const uint32_t sl = px % C::NSLOT, n = px / C::NSLOT;
                if (n > 0 && !mbar_wait(slot_empty(sl), (n - 1) & 1, w)) return false;
                if (lane == 0) {
                    const uint32_t dst = smem_u32(smem + C::OFF_RING + sl * C::PAIR_BYTES);
                    mbar_arrive_expect_tx(slot_full(sl), C::PAIR_BYTES);
                    tma_load_3d(dst, map, slot_full(sl), c0 * 64, h, row);
                    tma_load_3d(dst + C::BOX_BYTES, map, slot_full(sl), (c0 + 1) * 64, h, row);
                }
                return true;
            };
            for (uint32_t fi = 0; ok; ++fi) {
                int u = 0;
                if (lane == 0 && !feed_put(feed, fi, p.counter, p.num_units, u, w)) u = -2;
                u = __shfl_sync(0xffffffffu, u, 0);
                if (u == -2) { ok = false; break; }
                if (u < 0) break;
                const U256 t = decode_u256(p, u);
                if (t.skip || t.n_it == 0) continue;
                const int oh = 1 - t.hh;
                for (int it = 0; it < t.n_it; ++it, ++q_it) {
                    const int g = it / t.n_m;
                    const int m0 = (t.m_start + it % t.n_m) * 64;
                    const int h = t.hk * G + g;
                    const int row = t.q_start + m0;
                    // the tile's statistics into registers first, so their loads overlap the waits below;
                    // rows past the sequence get -LSE2 = -inf (P = 0) and Delta = 0; stored negated
                    float nl[2], nd[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int rr = m0 + lane * 2 + e;
                        const bool in = rr < t.Lq;
                        const size_t idx = static_cast<size_t>(h) * p.Tq + t.q_start + rr;
                        nl[e] = in ? -__ldg(p.lse2 + idx) : -INFINITY;
                        nd[e] = in ? -__ldg(p.delta + idx) : 0.f;
                    }
                    const uint32_t px = 4u * q_it;
                    if (!load_pair(px, &tmQ, 2 * oh, h, row) || !load_pair(px + 1, &tmDO, 2 * oh, h, row) ||
                        !load_pair(px + 2, &tmQ, 2 * t.hh, h, row)) {
                        ok = false;
                        break;
                    }
                    if (it == 0) {
                        // K and V of the unit, once the previous unit's last products have run
                        if (unit_it > 0 && !mbar_wait(kv_empty, (unit_it - 1) & 1, w)) { ok = false; break; }
                        if (lane == 0) {
                            mbar_arrive_expect_tx(kv_full, 2 * C::KV_BYTES);
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                tma_load_3d(smem_u32(smem + C::OFF_K + c * 128 * 128), &tmK, kv_full, c * 64, t.hk,
                                            t.k_start + t.n0);
                                tma_load_3d(smem_u32(smem + C::OFF_V + c * 128 * 128), &tmV, kv_full, c * 64, t.hk,
                                            t.k_start + t.n0);
                            }
                        }
                        ++unit_it;
                    }
                    if (!load_pair(px + 3, &tmDO, 2 * t.hh, h, row)) { ok = false; break; }
                    const uint32_t sb = q_it & 1;
                    if (q_it >= 2 && !mbar_wait(stat_empty(sb), ((q_it >> 1) - 1) & 1, w)) { ok = false; break; }
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        sStat[sb * 128 + lane * 2 + e] = nl[e];
                        sStat[sb * 128 + 64 + lane * 2 + e] = nd[e];
                    }
                    mbar_arrive(stat_full(sb));
                }
            }
            __syncwarp();
        } else if (warp == MMA_A || warp == MMA_B) {
            if (lane == 0) {
                const bool isA = warp == MMA_A;
                constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);     // S^T, dP^T
                constexpr uint32_t id_g = idesc_bf16_f32(128, 128, false, true);     // dV, dK halves
                constexpr uint32_t id_q = idesc_bf16_f32(128, 64, true, true);       // dQ^T half
                // Descriptor low words, advanced by constant offsets >> 4 (one add per operand per MMA)
                constexpr uint32_t CHUNK16 = (128 * 128) >> 4, BOX16 = C::BOX_BYTES >> 4, PAIR16 = C::PAIR_BYTES >> 4,
                                   K16 = 32 >> 4, ROWS16 = (16 * 128) >> 4;
                // A: K and the Q pairs; B: V and the dO pairs
                const uint32_t dKV = sdesc_lo(smem_u32(smem + (isA ? C::OFF_K : C::OFF_V)), 16);
                const uint32_t dDS = sdesc_lo(smem_u32(smem + C::OFF_DS), 128 * 128);   // dS^T, dQ^T's B (MN-major)
                const uint32_t dRK = sdesc_lo(smem_u32(smem + C::OFF_RING), 16);        // ring pairs, K-major
                const uint32_t dRN = sdesc_lo(smem_u32(smem + C::OFF_RING), C::BOX_BYTES);   // ring pairs, MN-major
                // this issuer's pairs of a tile: A reads Q other (0) and Q own (2); B reads dO other (1), dO own (3)
                const uint32_t k_other = isA ? 0u : 1u, k_own = isA ? 2u : 3u;
                const uint32_t col_s = isA ? C::COL_S : C::COL_DP;                     // S^T or dP^T
                const uint32_t col_g = isA ? C::COL_DK : C::COL_DV;                    // dK or dV
                const uint32_t a_off = isA ? 16u : 0u;                                 // packed dS^T or P^T
                uint32_t unit_it = 0, q_it = 0;
                bool ok = true;
                for (uint32_t fi = 0; ok; ++fi) {
                    int u;
                    if (!feed_get(feed, fi, u, w, false)) { ok = false; break; }
                    if (u < 0) break;
                    const U256 t = decode_u256(p, u);
                    if (t.skip || t.n_it == 0) continue;
                    if (!mbar_wait(kv_full, unit_it & 1, w)) { ok = false; break; }
                    const int oh = 1 - t.hh;
                    const uint32_t xO = dKV + 2 * oh * CHUNK16, xH = dKV + 2 * t.hh * CHUNK16;
                    // K[:, half]^T as dQ^T's A operand (MN-major: the two 64-column boxes of the half, 16 KB apart)
                    const uint32_t kT = sdesc_lo(smem_u32(smem + C::OFF_K + 2 * t.hh * 128 * 128), 128 * 128);
                    for (int it = 0; it < t.n_it; ++it, ++q_it) {
                        const uint32_t px = 4u * q_it;
                        const uint32_t slo = (px + k_other) % C::NSLOT, sho = (px + k_own) % C::NSLOT;
                        const uint32_t po = dRK + slo * PAIR16, ph = dRK + sho * PAIR16, phn = dRN + sho * PAIR16;
                        if (!mbar_wait(slot_full(slo), ((px + k_other) / C::NSLOT) & 1, w)) { ok = false; break; }
                        // the other issuer's product of the previous tile has read what this one overwrites
                        // S^T overwrites the packed P^T / dS^T of the previous tile, read by B's dV (and A's dK)
                        if (isA && q_it > 0 && !mbar_wait(dv_done, (q_it - 1) & 1, w)) { ok = false; break; }
                        if (isA && !mbar_wait(slot_full(sho), ((px + k_own) / C::NSLOT) & 1, w)) { ok = false; break; }
                        tc_fence_after();
                        // S^T = K Q^T (A) or dP^T = V dO^T (B) over the head dim, the other half's chunks first
#pragma unroll
                        for (int i = 0; i < 2; ++i)
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4)
                                umma_ss_lo(tmem + col_s, xO + i * CHUNK16 + k4 * K16, po + i * BOX16 + k4 * K16, id_s,
                                           (i | k4) != 0);
                        if (!isA) {
                            umma_commit(slot_empty(slo));         // dO of the other half: last read by dP^T
                            if (!mbar_wait(slot_full(sho), ((px + k_own) / C::NSLOT) & 1, w)) { ok = false; break; }
                            tc_fence_after();
                        }
#pragma unroll
                        for (int i = 0; i < 2; ++i)
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4)
                                umma_ss_lo(tmem + col_s, xH + i * CHUNK16 + k4 * K16, ph + i * BOX16 + k4 * K16, id_s, 1u);
                        if (isA) umma_commit(slot_empty(slo));    // Q of the other half: last read by S^T
                        umma_commit(s_full);
                        if (!mbar_wait(p_full, q_it & 1, w)) { ok = false; break; }
                        if (DQ && isA && q_it > 0 && !mbar_wait(dq_empty, (q_it - 1) & 1, w)) { ok = false; break; }
                        tc_fence_after();
                        if (DQ && isA) {
                            // dQ^T half = K[:, half]^T dS^T (K-dim = 128 keys)
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                umma_ss_lo(tmem + C::COL_DQ, kT + kk * ROWS16, dDS + kk * ROWS16, id_q, kk > 0);
                            umma_commit(dq_full);
                        }
                        // dK half += dS^T Q[:, half] (A) or dV half += P^T dO[:, half] (B), K-dim = 64 queries
                        const uint32_t first = it > 0 ? 1u : 0u;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_ts_lo(tmem + col_g, tmem + C::COL_PK(kk) + a_off, phn + kk * ROWS16, id_g,
                                       kk > 0 ? 1u : first);
                        umma_commit(slot_empty(sho));             // the own-half pair: last read here
                        if (!isA) umma_commit(dv_done);
                    }
                    if (!ok) break;
                    umma_commit(dkv_full);
                    umma_commit(kv_empty);
                    ++unit_it;
                }
            }
            __syncwarp();
        }
    } else if (warp >= 8) {
        if constexpr (DQ) {
            asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::DQ_REGS));
            // -------------------------------------------------------- dQ warpgroup (thread = head-dim row)
            const int wq = warp - 8;
            const uint32_t lb = tmem_lane_base(wq);
            uint32_t q_it = 0;
            bool ok = true;
            for (uint32_t fi = 0; ok; ++fi) {
                int u;
                if (!feed_get(feed, fi, u, w, true)) { ok = false; break; }
                if (u < 0) break;
                const U256 t = decode_u256(p, u);
                if (t.skip || t.n_it == 0) continue;
                for (int it = 0; it < t.n_it; ++it, ++q_it) {
                    const int g = it / t.n_m;
                    const int m0 = (t.m_start + it % t.n_m) * 64;
                    const int h = t.hk * G + g;
                    if (!mbar_wait(dq_full, q_it & 1, w)) { ok = false; break; }
                    tc_fence_after();
#if FA_B256_VEC_DQ
                    // lanes 4g .. 4g+3 hold head-dim rows 4g .. 4g+3; a 4 x 4 transpose across them (two
                    // butterfly steps) gives lane 4g+j the four head-dim values of query 4b+j, which leave
                    // as one 16-byte reduce-add (8 rows of 128 bytes per warp instruction)
                    const int j4 = lane & 3;
                    float* acc = p.dq_acc + (static_cast<size_t>(h) * p.Tq + t.q_start + m0) * D + t.hh * 128 +
                                 wq * 32 + (lane & ~3);
#pragma unroll 1
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t ra[32];
                        tmem_ld32(tmem + lb + C::COL_DQ + cc * 32, ra);
                        tmem_ld_wait_tie(ra);
#pragma unroll
                        for (int b4 = 0; b4 < 8; ++b4) {
                            float v0 = __uint_as_float(ra[4 * b4]), v1 = __uint_as_float(ra[4 * b4 + 1]),
                                  v2 = __uint_as_float(ra[4 * b4 + 2]), v3 = __uint_as_float(ra[4 * b4 + 3]);
                            {
                                const bool hi = (j4 & 1) != 0;
                                const float y0 = __shfl_xor_sync(0xffffffffu, hi ? v0 : v1, 1);
                                const float y1 = __shfl_xor_sync(0xffffffffu, hi ? v2 : v3, 1);
                                if (hi) { v0 = y0; v2 = y1; } else { v1 = y0; v3 = y1; }
                            }
                            {
                                const bool hi = (j4 & 2) != 0;
                                const float y0 = __shfl_xor_sync(0xffffffffu, hi ? v0 : v2, 2);
                                const float y1 = __shfl_xor_sync(0xffffffffu, hi ? v1 : v3, 2);
                                if (hi) { v0 = y0; v1 = y1; } else { v2 = y0; v3 = y1; }
                            }
                            const int qc = cc * 32 + 4 * b4 + j4;
                            if (m0 + qc < t.Lq)
                                atomicAdd(reinterpret_cast<float4*>(acc + static_cast<size_t>(qc) * D),
                                          make_float4(v0, v1, v2, v3));
                        }
                    }
#else
                    float* acc =
                        p.dq_acc + (static_cast<size_t>(h) * p.Tq + t.q_start + m0) * D + t.hh * 128 + wq * 32 + lane;
#pragma unroll 1
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t ra[32];
                        tmem_ld32(tmem + lb + C::COL_DQ + cc * 32, ra);
                        tmem_ld_wait_tie(ra);
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int qc = cc * 32 + e;
                            if (m0 + qc < t.Lq) atomicAdd(acc + static_cast<size_t>(qc) * D, __uint_as_float(ra[e]));
                        }
                    }
#endif
                    tc_fence_before();
                    mbar_arrive(dq_empty);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ compute warpgroups (thread = key row)
        const int gq = warp >> 2;                  // query columns [32 gq, 32 gq + 32)
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lb = tmem_lane_base(warp & 3);
        const float c2 = p.scale_log2;
        uint32_t unit_it = 0, q_it = 0;
        bool ok = true;
        for (uint32_t fi = 0; ok; ++fi) {
            int u;
            if (!feed_get(feed, fi, u, w, true)) { ok = false; break; }
            if (u < 0) break;
            const U256 t = decode_u256(p, u);
            if (t.skip) continue;
            const int kj = t.n0 + r;
            const bool kvalid = kj < t.Lk;
            const size_t krow = (static_cast<size_t>(t.k_start) + kj) * p.Hkv + t.hk;
            // warpgroup 0 owns dV of the unit's half, warpgroup 1 dK
            __nv_bfloat16* dst = (gq == 0 ? p.dv : p.dk) + krow * D + t.hh * 128;
            if (t.n_it == 0) {
                if (kvalid) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    for (int c = 0; c < 16; ++c) reinterpret_cast<uint4*>(dst)[c] = z;
                }
                continue;
            }
            // this key row is seen by query rows q_lo .. q_hi of the sequence
            int q_lo = -0x40000000, q_hi = 0x40000000;
            if (p.wr >= 0) q_lo = kj - (t.Lk - t.Lq) - p.wr;
            if (p.wl >= 0) q_hi = kj - (t.Lk - t.Lq) + p.wl;
            for (int it = 0; it < t.n_it; ++it, ++q_it) {
                const int m0 = (t.m_start + it % t.n_m) * 64;
                if (!mbar_wait(s_full, q_it & 1, w)) { ok = false; break; }
                const uint32_t sb = q_it & 1;
                if (!mbar_wait(stat_full(sb), (q_it >> 1) & 1, w)) { ok = false; break; }
                const float* nL = sStat + sb * 128 + 32 * gq;      // -LSE2 of this warpgroup's 32 rows
                const float* nD = nL + 64;                         // -Delta
                tc_fence_after();
                uint32_t sa[32], da[32];
                tmem_ld32(tmem + lb + C::COL_S + 32 * gq, sa);
                tmem_ld32(tmem + lb + C::COL_DP + 32 * gq, da);
                tmem_ld_wait_tie(sa);
                reg_tie(da);
                const int qmin = q_lo - m0 - 32 * gq, qmax = q_hi - m0 - 32 * gq;
                const bool any_mask = __any_sync(0xffffffffu, !(kvalid && qmin <= 0 && qmax >= 31));
                const float2 c2v = make_float2(c2, c2);
                uint32_t pp[16], dd[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float2 sv = make_float2(__uint_as_float(sa[e]), __uint_as_float(sa[e + 1]));
                    const float2 dv = make_float2(__uint_as_float(da[e]), __uint_as_float(da[e + 1]));
                    const float2 a = ffma2(sv, c2v, make_float2(nL[e], nL[e + 1]));
                    float2 pr = make_float2(ex2_approx(a.x), ex2_approx(a.y));
                    if (any_mask) {
                        pr.x = (kvalid && e >= qmin && e <= qmax) ? pr.x : 0.f;
                        pr.y = (kvalid && e + 1 >= qmin && e + 1 <= qmax) ? pr.y : 0.f;
                    }
                    const float2 ds = fmul2(pr, fadd2(dv, make_float2(nD[e], nD[e + 1])));
                    pp[e / 2] = pack_bf16x2(pr.x, pr.y);
                    dd[e / 2] = pack_bf16x2(ds.x, ds.y);
                }
                // P^T and dS^T of this warpgroup's 32 queries go back into the 32 S^T columns it has just
                // read (16 each), so neither warpgroup writes columns the other still reads
                tmem_st16(tmem + lb + C::COL_S + 32 * gq, pp);
                tmem_st16(tmem + lb + C::COL_S + 32 * gq + 16, dd);
                uint8_t* ds_row = smem + C::OFF_DS + r * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int cin = gq * 4 + q4;
                    *reinterpret_cast<uint4*>(ds_row + ((cin ^ (r & 7)) << 4)) =
                        make_uint4(dd[4 * q4], dd[4 * q4 + 1], dd[4 * q4 + 2], dd[4 * q4 + 3]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(stat_empty(sb));   // the warp has read the tile's statistics
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(p_full);
            }
            if (!ok) break;
            if (!mbar_wait(dkv_full, unit_it & 1, w)) { ok = false; break; }
            ++unit_it;
            tc_fence_after();
            const uint32_t col = gq == 0 ? C::COL_DV : C::COL_DK;
            const float2 mul2 = gq == 0 ? make_float2(1.f, 1.f) : make_float2(p.scale, p.scale);
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t ra[32];
                tmem_ld32(tmem + lb + col + cc * 32, ra);
                tmem_ld_wait_tie(ra);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 v = fmul2(make_float2(__uint_as_float(ra[2 * e]), __uint_as_float(ra[2 * e + 1])), mul2);
                    pk[e] = pack_bf16x2(v.x, v.y);
                }
                if (kvalid) {
                    uint4* o4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) o4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
            tc_fence_before();
        }
    }

    __syncthreads();
    if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) {
        }
    }
    if (warp == MMA_A) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dQ[tok][h][:] = bf16(scale * dQacc[h][tok][:])
__global__ void __launch_bounds__(256) bwd256_convert_kernel(const float* dq_acc, __nv_bfloat16* dq, int Tq, int Hq,
                                                             float scale) {
    const long long n2 = static_cast<long long>(Tq) * Hq * (D / 2);
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n2;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long e = 2 * i;
        const int d = static_cast<int>(e % D);
        const long long th = e / D;               // tok * Hq + h
        const int h = static_cast<int>(th % Hq);
        const long long tok = th / Hq;
        const float2 v = *reinterpret_cast<const float2*>(dq_acc + (static_cast<size_t>(h) * Tq + tok) * D + d);
        reinterpret_cast<uint32_t*>(dq)[i] = pack_bf16x2(v.x * scale, v.y * scale);
    }
}

}  // namespace

template <bool DQ>
static int run_bwd256(const Problem& pr, const void* dout, const float* lse2, const float* delta, float* dq_acc,
                      void* dq, void* dk, void* dv, const Device& dev, cudaStream_t stream) {
    using C = Cfg;
    alignas(64) CUtensorMap mq, mk, mv, mdo;
    const uint64_t rq = static_cast<uint64_t>(pr.Hq) * D * 2, rk = static_cast<uint64_t>(pr.Hkv) * D * 2;
    if (!make_map_3d_bf16(&mq, pr.q, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, 64)) return 5;
    if (!make_map_3d_bf16(&mdo, dout, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, 64)) return 5;
    if (!make_map_3d_bf16(&mk, pr.k, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, 128)) return 5;
    if (!make_map_3d_bf16(&mv, pr.v, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, 128)) return 5;
    B256Params p;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.dq_acc = dq_acc;
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
    const long long units = static_cast<long long>((pr.Sk + 127) / 128) * pr.num_seqs * pr.Hkv * 2;
    if (units > 0x7fffffffLL) return 2;
    p.num_units = static_cast<int>(units);
    p.scale = pr.scale;
    p.scale_log2 = pr.scale * 1.4426950408889634f;
    p.wl = pr.wl;
    p.wr = pr.wr;
    p.n_blocks = (pr.Sk + 127) / 128;
    p.chunk = bwd_chunk_groups(pr.num_seqs * pr.Hkv, 2 * p.n_blocks, p.group, pr.Sq, D, dev.num_sms);
    p.counter = bwd_unit_counter(dq_acc, pr.Tq, pr.Hq, D);   // dq_acc is the start of the workspace
    p.timeout_ns = dev.timeout_ns;
    p.status = dev.status;
    auto kern = bwd256_kernel<DQ>;
    static bool set[64] = {};
    if (!set[dev.id & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM)) !=
            cudaSuccess)
            return 5;
        cudaFuncAttributes fa_attr;
        if (cudaFuncGetAttributes(&fa_attr, kern) != cudaSuccess || fa_attr.numRegs != C::LAUNCH_REGS) return 2;
        set[dev.id & 63] = true;
    }
    const int grid = p.num_units < dev.num_sms ? p.num_units : dev.num_sms;
    if (grid > 0) {
        prof_before(1, stream);
        kern<<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, mdo, p);
        prof_after(1, stream);
        if (cudaPeekAtLastError() != cudaSuccess) return 5;
    }
    if (!DQ) return 0;
    const long long n2 = static_cast<long long>(pr.Tq) * pr.Hq * (D / 2);
    long long blocks = (n2 + 255) / 256;
    if (blocks > static_cast<long long>(dev.num_sms) * 32) blocks = static_cast<long long>(dev.num_sms) * 32;
    bwd256_convert_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), pr.Tq,
                                                                        pr.Hq, pr.scale);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 5;
}

int launch_bwd256_main(const Problem& pr, const void* dout, const float* lse2, const float* delta, float* dq_acc,
                       void* dq, void* dk, void* dv, bool with_dq, const Device& dev, cudaStream_t stream) {
    return with_dq ? run_bwd256<true>(pr, dout, lse2, delta, dq_acc, dq, dk, dv, dev, stream)
                   : run_bwd256<false>(pr, dout, lse2, delta, dq_acc, dq, dk, dv, dev, stream);
}

}  // namespace fa

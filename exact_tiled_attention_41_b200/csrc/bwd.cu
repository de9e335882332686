// bwd.cu -- backward of exact tiled attention on sm_100a.
//
// The scores are recomputed from Q, K and the forward's LSE instead of being
// stored (flash-attention README: IO-aware tiling with recomputation;
// FlashAttention fork v1.4 notes, section 4: the backward applies the
// exponential against the stored statistics, scale_apply_exp2 with
// Scale_max = false).  With S = scale Q K^T, P = exp(S - LSE):
//   dV = P^T dO,  dP = dO V^T,  Delta_i = rowsum(dO * O)_i,
//   dS = P * (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three launches:
//   1. preprocess: Delta = rowsum(dO * O) in fp32, LSE2 = LSE * log2(e) (+inf for
//      rows with no key, so their P is exactly 0), and a zeroed fp32 dQ accumulator
//      (kept in L2 up to the convert when it is small enough: kBwdL2KeepBytes).
//   2. main kernel, one persistent CTA per SM, KV-tile stationary: a work unit
//      is (sequence, KV head, 128-key tile); it loops over the 128-row query
//      tiles of every query head that reads the KV head (so dK and dV of GQA
//      need no atomics) and only over the query tiles that can see the key
//      tile (causal masks and sliding windows cut the range at both ends).  Roles (16 warps, registers redistributed with setmaxnreg):
//        warps 0-7   two compute warpgroups, thread = key row, each owning 64 of
//                    the 128 query columns: P^T, dS^T from S^T and dP^T in tensor
//                    memory, both written back as bf16 into the warpgroup's own 64
//                    columns of S^T (dS^T also to shared memory), so dP^T's columns
//                    are free for dQ; dV (warpgroup 0) / dK (warpgroup 1) epilogue
//                    (whole key tiles leave through shared memory with TMA stores)
//        warps 8-11  dQ: thread = query row; reads the dQ tile from tensor memory
//                    and adds it to the fp32 accumulator (vector atomics); each half
//                    of the tile is released as soon as it is in registers, so the
//                    next S^T (first half) and dP^T (second half) wait as little as
//                    possible on the reduction traffic
//        warp 12     producer: K, V once per unit; Q, dO tiles (TMA) and the
//                    tile's LSE2 / Delta (plain loads) through a 2-stage ring
//        warp 13     tensor memory and every tcgen05 MMA, in this order per tile:
//                    S^T = K Q^T, then dP^T = V dO^T once the previous dQ read-out
//                    released dP^T's columns (K-major x K-major); dV += P^T dO,
//                    dK += dS^T Q over queries 0-63 as soon as warpgroup 0 is done
//                    (tensor-memory A), while warpgroup 1 still works; then
//                    dQ = dS K, all D columns in one product, into dP^T's columns,
//                    so the dQ read-out overlaps the dV, dK products over queries 64-127
//   3. convert: dQ = bf16(scale * dQacc); the dead accumulator's L2 lines are discarded.
// The deterministic backward runs the main kernel with DQ = false (no dQ product,
// no reduce-adds, warps 8-11 idle) and computes dq in the query-tile-stationary
// pass of bwd_dq.cu instead of steps 2's dQ and 3.
#include "internal.h"
#include "sm100.cuh"

#include <math.h>

#include <type_traits>

#ifndef FA_BWD_FMA_EXP_EVERY
#define FA_BWD_FMA_EXP_EVERY 6
#endif

namespace fa {

// Share of the backward gradient step's exponentials computed on the FMA pipe (exp2_fma2): one pair
// in kBwdFmaExpEvery, 0 = none.
constexpr int kBwdFmaExpEvery = FA_BWD_FMA_EXP_EVERY;

// A dQ accumulator of at most this many bytes (about half of the 126 MB L2) is kept in L2 from the
// preprocess to the convert with the evict_last policy (the dense prefill workload's is 64 MiB: +1.7 % on
// the whole backward; larger ones would push out the Q and dO tiles that the key tiles share).
constexpr size_t kBwdL2KeepBytes = size_t(64) << 20;

#ifndef FA_BWD_PRE_PASSES
#define FA_BWD_PRE_PASSES 1
#endif
constexpr int kPrePasses = FA_BWD_PRE_PASSES;

struct BwdParams {
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* dq_acc;          // [Hq][D/4][Tq][4]
    const float* lse2;      // [Hq][Tq]
    const float* delta;     // [Hq][Tq]
    const int32_t* cu_q;
    const int32_t* cu_k;
    int num_seqs, Sq, Sk, Tq, Tk, Hq, Hkv, group;
    int n_blocks, num_units;
    float scale, scale_log2;
    int wl, wr;             // window sides, -1 = unbounded; a causal mask is wr = 0
    int chunk;              // (sequence, KV head) groups per chunk of the unit list
    int* counter;           // unit counter of the dynamic schedule (zeroed by the preprocess kernel)
    int l2_keep;            // 1: reduce-adds into dQacc with the L2 evict_last policy
    unsigned long long timeout_ns;
    int* status;
};

struct BUnit {
    int b, hk, q_start, k_start, Lq, Lk, n0, m_start, n_m, n_it;
    bool skip;
};

// Unit u: the list is cut into chunks of p.chunk (sequence, KV head) groups; inside a chunk the units
// run key tile by key tile (the first tiles have the most work under a causal mask) over the chunk's
// groups.  With p.chunk = all groups this is the plain heaviest-first order.
__device__ __forceinline__ BUnit decode_bunit(const BwdParams& p, int u) {
    BUnit t;
    const int groups = p.num_seqs * p.Hkv;
    const int per_chunk = p.chunk * p.n_blocks;
    const int c = u / per_chunk;
    const int g0 = c * p.chunk;
    const int cs = min(p.chunk, groups - g0);
    const int idx = u - c * per_chunk;
    const int n = idx / cs;           // key tile
    const int r = g0 + idx % cs;      // group
    t.b = r / p.Hkv;
    t.hk = r % p.Hkv;
    if (p.cu_q != nullptr) {
        t.q_start = __ldg(p.cu_q + t.b);
        t.Lq = __ldg(p.cu_q + t.b + 1) - t.q_start;
        t.k_start = __ldg(p.cu_k + t.b);
        t.Lk = __ldg(p.cu_k + t.b + 1) - t.k_start;
        t.q_start = max(t.q_start, 0);
        t.k_start = max(t.k_start, 0);
        t.Lq = max(min(min(t.Lq, p.Tq - t.q_start), 1 << 30), 0);   // at most 2^30 tokens per sequence
        t.Lk = max(min(min(t.Lk, p.Tk - t.k_start), 1 << 30), 0);
    } else {
        t.q_start = t.b * p.Sq;
        t.Lq = p.Sq;
        t.k_start = t.b * p.Sk;
        t.Lk = p.Sk;
    }
    t.n0 = n * 128;
    t.skip = t.n0 >= t.Lk;
    // query rows that see some key of n0 .. n0+127: key j is allowed for row i iff
    // i + off - wl <= j <= i + off + wr, i.e. j - off - wr <= i <= j - off + wl
    // (lengths <= 2^30 and window sides < 2^30 keep every term inside int32)
    const int off = t.Lk - t.Lq;
    int r_lo = 0, r_hi = t.Lq - 1;
    if (p.wr >= 0) r_lo = max(r_lo, t.n0 - off - p.wr);
    if (p.wl >= 0) r_hi = min(r_hi, min(t.n0 + 127, t.Lk - 1) - off + p.wl);
    if (t.skip || r_hi < r_lo) {
        t.m_start = 0;
        t.n_m = 0;
    } else {
        t.m_start = r_lo / 128;
        t.n_m = r_hi / 128 + 1 - t.m_start;
    }
    t.n_it = t.n_m * p.group;
    return t;
}

template <int D>
struct BwdCfg {
    static constexpr int ST = 2;
    static constexpr int NCHUNK = D / 64;
    static constexpr uint32_t T_BYTES = 128 * D * 2;      // one 128-row tile of K, V, Q or dO
    static constexpr uint32_t DS_BYTES = 128 * 128 * 2;   // dS^T [key][query], two 64-query boxes
    // layout: K | V | Q[ST] | dO[ST] | dS | LSE2[ST][128] | Delta[ST][128] | barriers
    static constexpr uint32_t OFF_K = 0, OFF_V = T_BYTES, OFF_Q = 2 * T_BYTES, OFF_DO = (2 + ST) * T_BYTES,
                              OFF_DS = (2 + 2 * ST) * T_BYTES, OFF_STAT = OFF_DS + DS_BYTES,
                              OFF_BAR = OFF_STAT + 2 * ST * 128 * 4;
    static constexpr int NUM_BARS = 2 + 2 * ST + 10 + 2 * kFeedSlots;
    static constexpr size_t SMEM = OFF_BAR + NUM_BARS * 8 + 16 + 4 * kFeedSlots;
    // tensor memory: dV | dK | S^T | dP^T.  After the gradient step the packed bf16 P^T and dS^T of each
    // 32-query half sit in that half's own 32 columns of S^T; dQ (fp32, D columns) is accumulated over
    // dP^T, whose values the warpgroups have read by then.
    static constexpr uint32_t COL_DV = 0, COL_DK = D, COL_S = 2 * D, COL_DP = 2 * D + 128, COL_DQ = COL_DP;
    // packed P^T / dS^T of queries [16 kk, 16 kk + 16): query half (kk >> 1) of 32 lives in columns
    // [32 (kk >> 1), +32) of S^T, P^T first, dS^T 16 columns later
    static constexpr uint32_t COL_P(int kk) { return COL_S + (kk >> 1) * 32 + (kk & 1) * 8; }
    static constexpr uint32_t COL_DSP(int kk) { return COL_P(kk) + 16; }
    static_assert(2 * D + 256 <= 512, "tensor memory budget");
    static_assert(D == 64 || D == 128, "dQ fits dP^T's 128 columns for D <= 128");
    // 16 warps: 0-7 two compute warpgroups (query columns 0-63 / 64-127), 8-11 dQ warpgroup,
    // 12 producer, 13 MMA issuer, 14-15 idle.  Registers: launch at 128 per thread (512 x 128 = 65536);
    // the producer / MMA warpgroup gives 40 per thread to the dQ warpgroup, which holds a whole dQ row:
    // 2 x 128 x 128 + 128 x 168 + 128 x 88 = 65536.  The host checks the launch count.
    static constexpr int THREADS = 512, LAUNCH_REGS = 128, COMPUTE_REGS = 128, DQ_REGS = 168, OTHER_REGS = 88;
    static_assert(COMPUTE_REGS == LAUNCH_REGS, "the compute warpgroups keep the launch count");
    static_assert(2 * 128 * COMPUTE_REGS + 128 * DQ_REGS + 128 * OTHER_REGS <= THREADS * LAUNCH_REGS, "register split");
};

template <int D, bool DQ>
__global__ void __launch_bounds__(512, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
               const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
               const __grid_constant__ BwdParams p) {
    using C = BwdCfg<D>;
    constexpr int ST = C::ST;
    extern __shared__ __align__(1024) uint8_t smem[];
    float* sLSE = reinterpret_cast<float*>(smem + C::OFF_STAT);          // [ST][128], -LSE2
    float* sDel = sLSE + ST * 128;                                       // [ST][128], -Delta
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* feed_slot = reinterpret_cast<int*>(tmem_slot + 4);
    const uint32_t b0 = smem_u32(bars);
    const UnitFeed feed{feed_slot, b0 + 8u * (2 + 2 * ST + 10), b0 + 8u * (2 + 2 * ST + 10 + kFeedSlots)};
    // K and V of a unit arrive / are released separately: V is last read by the unit's last dP^T,
    // K by its last dQ (or S^T), so the next unit's V and first Q/dO tile load while those finish
    const uint32_t k_full = b0, k_free = b0 + 8;
    auto q_full = [&](int s) { return b0 + 8u * (2 + s); };
    auto q_empty = [&](int s) { return b0 + 8u * (2 + ST + s); };
    // p_full / p_full_hi: compute warpgroup 0 (query columns 0-63) / 1 (64-127) done
    const uint32_t s_full = b0 + 8u * (2 + 2 * ST), p_full = s_full + 8, dq_full = s_full + 16,
                   dq_empty = s_full + 24, dkv_full = s_full + 32, dq_empty_hi = s_full + 40, p_full_hi = s_full + 48,
                   v_full = s_full + 56, v_free = s_full + 64, dv_done = s_full + 72;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int PRODUCER = 12, MMA = 13, MMA_B = 14;

    if ((smem_u32(smem) & 1023u) != 0) {   // the swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicCAS(p.status, 0, 2);
        return;
    }
    if (threadIdx.x == 0) {
        mbar_init(bars + 0, 1);
        mbar_init(bars + 1, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(bars + 2 + s, 33);        // 32 producer lanes (statistics) + the TMA expect-tx arrival
            mbar_init(bars + 2 + ST + s, 2);    // both issuers' last reads of the stage
        }
        mbar_init(bars + 2 + 2 * ST + 0, 2);    // s_full: S^T (issuer A) and dP^T (issuer B)
        mbar_init(bars + 2 + 2 * ST + 1, 128);  // p_full: compute warpgroup 0 (query columns 0-63)
        mbar_init(bars + 2 + 2 * ST + 2, 1);    // dq_full
        mbar_init(bars + 2 + 2 * ST + 3, 128);  // dq_empty: dQ columns in the S^T region read out
        mbar_init(bars + 2 + 2 * ST + 4, 2);    // dkv_full: last dK (A) and dV (B)
        mbar_init(bars + 2 + 2 * ST + 5, 128);  // dq_empty_hi: dQ columns in the dP^T region read out
        mbar_init(bars + 2 + 2 * ST + 6, 128);  // p_full_hi: compute warpgroup 1 (query columns 64-127)
        mbar_init(bars + 2 + 2 * ST + 7, 1);    // v_full
        mbar_init(bars + 2 + 2 * ST + 8, 1);    // v_free
        mbar_init(bars + 2 + 2 * ST + 9, 1);    // dv_done: issuer B's dV of a tile has read P^T
        for (int s = 0; s < kFeedSlots; ++s) {
            mbar_init(bars + 2 + 2 * ST + 10 + s, 1);                            // unit published
            mbar_init(bars + 2 + 2 * ST + 10 + kFeedSlots + s, DQ ? 14 : 10);    // read by the issuers, compute (, dQ) warps
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
    if (warp == MMA) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Watch w{abort_flag, p.status, p.timeout_ns};
    const int G = p.group;
    // the preprocess kernel's outputs (statistics, zeroed accumulator and unit counter) are read from here on
    grid_dep_wait();

    if (warp >= 12) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::OTHER_REGS));
        if (warp == PRODUCER) {
            // -------------------------------------------------------- producer (whole warp)
            uint32_t unit_it = 0, q_it = 0;
            bool ok = true;
            for (uint32_t fi = 0; ok; ++fi) {
                int u = 0;
                if (lane == 0 && !feed_put(feed, fi, p.counter, p.num_units, u, w)) u = -2;
                u = __shfl_sync(0xffffffffu, u, 0);
                if (u == -2) { ok = false; break; }
                if (u < 0) break;
                const BUnit t = decode_bunit(p, u);
                if (t.skip || t.n_it == 0) continue;
                // one query tile's Q and dO (TMA) and statistics (plain loads) into the next ring stage
                auto load_tile = [&](int it) -> bool {
                    const int g = it / t.n_m;
                    const int m0 = (t.m_start + it % t.n_m) * 128;
                    const int h = t.hk * G + g;
                    const int st = q_it % ST;
                    if (q_it >= ST && !mbar_wait(q_empty(st), ((q_it / ST) - 1) & 1, w)) return false;
                    // tile statistics; rows past the sequence get LSE2 = +inf (P = 0) and Delta = 0
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int qi = lane * 4 + e;
                        const int row = m0 + qi;
                        const bool in = row < t.Lq;
                        const size_t idx = static_cast<size_t>(h) * p.Tq + t.q_start + row;
                        // stored negated, so the gradient step adds them (no negation per element)
                        sLSE[st * 128 + qi] = in ? -__ldg(p.lse2 + idx) : -INFINITY;
                        sDel[st * 128 + qi] = in ? -__ldg(p.delta + idx) : 0.f;
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(q_full(st), 2 * C::T_BYTES);
#pragma unroll
                        for (int c = 0; c < C::NCHUNK; ++c) {
                            tma_load_3d(smem_u32(smem + C::OFF_Q + st * C::T_BYTES + c * 128 * 128), &tmQ, q_full(st),
                                        c * 64, h, t.q_start + m0);
                            tma_load_3d(smem_u32(smem + C::OFF_DO + st * C::T_BYTES + c * 128 * 128), &tmDO,
                                        q_full(st), c * 64, h, t.q_start + m0);
                        }
                    }
                    mbar_arrive(q_full(st));
                    ++q_it;
                    return true;
                };
                // V (free once the previous unit's last dP^T has run), the first Q / dO tile, then K
                if (unit_it > 0 && !mbar_wait(v_free, (unit_it - 1) & 1, w)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(v_full, C::T_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c)
                        tma_load_3d(smem_u32(smem + C::OFF_V + c * 128 * 128), &tmV, v_full, c * 64, t.hk,
                                    t.k_start + t.n0);
                }
                if (!load_tile(0)) { ok = false; break; }
                if (unit_it > 0 && !mbar_wait(k_free, (unit_it - 1) & 1, w)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(k_full, C::T_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c)
                        tma_load_3d(smem_u32(smem + C::OFF_K + c * 128 * 128), &tmK, k_full, c * 64, t.hk,
                                    t.k_start + t.n0);
                }
                ++unit_it;
                for (int it = 1; it < t.n_it && ok; ++it)
                    if (!load_tile(it)) ok = false;
            }
            __syncwarp();
        } else if (warp == MMA || warp == MMA_B) {
            // -------------------------------------------------------- MMA issuers
            // One issuing thread needs about 54 cycles per 16-deep MMA, close to the 64 the tensor core
            // needs for these 128 x 128 steps, so the waits between products leave the tensor core idle.  Two
            // threads issue: A takes S^T, dK and dQ (K and Q are its operands), B takes dP^T and dV (V, dO).
            // S^T of a tile overwrites the packed P^T that B's dV of the previous tile reads (dv_done); dP^T
            // overwrites the previous dQ, read out by the dQ warpgroup (dq_empty).
            if (lane == 0) {
                const bool isA = warp == MMA;
                constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);   // S^T, dP^T
                constexpr uint32_t id_tn = idesc_bf16_f32(128, D, false, true);      // dV, dK (A in tensor memory)
                constexpr uint32_t id_dq = idesc_bf16_f32(128, D, true, true);       // dQ, all D columns
                // Descriptor low words, advanced by constant offsets >> 4 (one add per operand per MMA)
                constexpr uint32_t T16 = C::T_BYTES >> 4, ROWS16 = (16 * 128) >> 4;
                // A: K and Q; B: V and dO
                const uint32_t dX0 = sdesc_lo(smem_u32(smem + (isA ? C::OFF_K : C::OFF_V)), 16);      // K-major
                const uint32_t dY0 = sdesc_lo(smem_u32(smem + (isA ? C::OFF_Q : C::OFF_DO)), 16);     // stage 0, K-major
                const uint32_t dY0n = sdesc_lo(smem_u32(smem + (isA ? C::OFF_Q : C::OFF_DO)), 128 * 128);   // MN-major B
                const uint32_t dSn = sdesc_lo(smem_u32(smem + C::OFF_DS), 128 * 128);     // dS, MN-major A of dQ
                const uint32_t dKn = sdesc_lo(smem_u32(smem + C::OFF_K), 128 * 128);      // K, MN-major B of dQ
                const uint32_t col_s = isA ? C::COL_S : C::COL_DP;                         // S^T or dP^T
                const uint32_t col_g = isA ? C::COL_DK : C::COL_DV;                        // dK or dV
                const uint32_t a_off = isA ? 16u : 0u;                                     // packed dS^T / P^T
                auto kchunk = [](int kk) { return static_cast<uint32_t>(((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4); };
                uint32_t unit_it = 0, q_it = 0, g_it = 0;
                bool ok = true;
                for (uint32_t fi = 0; ok; ++fi) {
                    int u;
                    if (!feed_get(feed, fi, u, w, false)) { ok = false; break; }
                    if (u < 0) break;
                    const BUnit t = decode_bunit(p, u);
                    if (t.skip || t.n_it == 0) continue;
                    if (!mbar_wait(isA ? k_full : v_full, unit_it & 1, w)) { ok = false; break; }
                    for (int it = 0; it < t.n_it; ++it, ++q_it, ++g_it) {
                        const bool last = it + 1 == t.n_it;
                        const int st = q_it % ST;
                        if (!mbar_wait(q_full(st), (q_it / ST) & 1, w)) { ok = false; break; }
                        if (isA) {
                            // S^T overwrites the packed P^T that the previous tile's dV read
                            if (g_it > 0 && !mbar_wait(dv_done, (g_it - 1) & 1, w)) { ok = false; break; }
                        } else if (DQ && g_it > 0) {
                            // dP^T goes where the previous tile's dQ was: both halves of it must be read out
                            if (!mbar_wait(dq_empty, (g_it - 1) & 1, w)) { ok = false; break; }
                            if (!mbar_wait(dq_empty_hi, (g_it - 1) & 1, w)) { ok = false; break; }
                        }
                        tc_fence_after();
                        const uint32_t yd = dY0 + st * T16, yn = dY0n + st * T16;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_ss_lo(tmem + col_s, dX0 + kchunk(kk), yd + kchunk(kk), id_kk, kk > 0);
                        umma_commit(s_full);
                        if (isA && !DQ && last) umma_commit(k_free);   // K's last reader without the dQ product
                        if (!isA && last) umma_commit(v_free);         // V's last reader in this unit
                        // once both compute warpgroups are done: dQ first (A), so that its read-out, and with it
                        // the next dP^T, starts early; then dK += dS^T Q (A) and dV += P^T dO (B)
                        if (!mbar_wait(p_full, g_it & 1, w)) { ok = false; break; }
                        if (!mbar_wait(p_full_hi, g_it & 1, w)) { ok = false; break; }
                        tc_fence_after();
                        if (DQ && isA) {
                            // dQ = dS K over dP^T's columns (read out by the dQ warpgroup while dV / dK run)
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)     // K-dim = 128 key rows
                                umma_ss_lo(tmem + C::COL_DQ, dSn + kk * ROWS16, dKn + kk * ROWS16, id_dq, kk > 0);
                            umma_commit(dq_full);
                            if (last) umma_commit(k_free);        // K's last reader in this unit
                        }
                        const uint32_t first = it > 0 ? 1u : 0u;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_ts_lo(tmem + col_g, tmem + C::COL_P(kk) + a_off, yn + kk * ROWS16, id_tn,
                                       kk > 0 ? 1u : first);
                        umma_commit(q_empty(st));
                        if (!isA) umma_commit(dv_done);
                    }
                    if (!ok) break;
                    umma_commit(dkv_full);
                    ++unit_it;
                }
            }
            __syncwarp();
        }
    } else if (warp >= 8) {
        if constexpr (DQ) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::DQ_REGS));
        // ------------------------------------------------------------ dQ warpgroup (thread = query row)
        if constexpr (DQ) {
        const int wq = warp - 8;
        const int r = wq * 32 + lane;
        const uint32_t lb = tmem_lane_base(wq);
        const uint64_t acc_pol = p.l2_keep ? l2_policy_last() : l2_policy_normal();
        uint32_t g_it = 0;
        bool ok = true;
        for (uint32_t fi = 0; ok; ++fi) {
            int u;
            if (!feed_get(feed, fi, u, w, true)) { ok = false; break; }
            if (u < 0) break;
            const BUnit t = decode_bunit(p, u);
            if (t.skip || t.n_it == 0) continue;
            for (int it = 0; it < t.n_it; ++it, ++g_it) {
                const int g = it / t.n_m;
                const int m0 = (t.m_start + it % t.n_m) * 128;
                const int h = t.hk * G + g;
                const bool valid = m0 + r < t.Lq;
                const size_t tok = static_cast<size_t>(t.q_start) + m0 + r;
                if (!mbar_wait(dq_full, g_it & 1, w)) { ok = false; break; }
                tc_fence_after();
                float4* acc = reinterpret_cast<float4*>(p.dq_acc) + static_cast<size_t>(h) * (D / 4) * p.Tq + tok;
                // the whole dQ row in registers at once, so its columns are released before the reduce-adds
                uint32_t ra[D / 32][32];
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tmem + lb + C::COL_DQ + cc * 32, ra[cc]);
                tmem_ld_wait_tie(ra[0]);
#pragma unroll
                for (int cc = 1; cc < D / 32; ++cc) reg_tie(ra[cc]);
                tc_fence_before();
                mbar_arrive(dq_empty);
                mbar_arrive(dq_empty_hi);
                if (valid) {
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc)
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            red_add_f32x4_hint(acc + static_cast<size_t>(cc * 8 + e) * p.Tq,
                                               make_float4(__uint_as_float(ra[cc][4 * e]), __uint_as_float(ra[cc][4 * e + 1]),
                                                           __uint_as_float(ra[cc][4 * e + 2]),
                                                           __uint_as_float(ra[cc][4 * e + 3])),
                                               acc_pol);
                }
            }
        }
        }
    } else {
        // ------------------------------------------------------------ compute warpgroups (thread = key row)
        const int gq = warp >> 2;                  // query columns [64 gq, 64 gq + 64)
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lb = tmem_lane_base(warp & 3);
        const float c2 = p.scale_log2;
        uint32_t unit_it = 0, q_it = 0, g_it = 0;
        bool ok = true;
        for (uint32_t fi = 0; ok; ++fi) {
            int u;
            if (!feed_get(feed, fi, u, w, true)) { ok = false; break; }
            if (u < 0) break;
            const BUnit t = decode_bunit(p, u);
            if (t.skip) continue;
            const int kj = t.n0 + r;                 // key index inside the sequence
            const bool kvalid = kj < t.Lk;
            // this warpgroup's output row (dV for warpgroup 0, dK for 1)
            auto out_row = [&](const BUnit& tt) {
                const size_t krow = (static_cast<size_t>(tt.k_start) + tt.n0 + r) * p.Hkv + tt.hk;
                return (gq == 0 ? p.dv : p.dk) + krow * D;
            };
            if (t.n_it == 0) {
                if (kvalid) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    __nv_bfloat16* gdst = out_row(t);
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(gdst)[c] = z;
                }
                continue;
            }
            // this key row is seen by query rows q_lo .. q_hi of the sequence
            // (a key row past the sequence is seen by none: an empty range)
            int q_lo = -0x40000000, q_hi = 0x40000000;
            if (p.wr >= 0) q_lo = kj - (t.Lk - t.Lq) - p.wr;
            if (p.wl >= 0) q_hi = kj - (t.Lk - t.Lq) + p.wl;
            if (!kvalid) q_lo = 0x40000000;
            for (int it = 0; it < t.n_it; ++it, ++q_it, ++g_it) {
                const int m0 = (t.m_start + it % t.n_m) * 128;
                const int st = q_it % ST;
                // the statistics arrive with the Q / dO tile
                bool got = mbar_wait(s_full, g_it & 1, w);
                got = got && mbar_wait(q_full(st), (q_it / ST) & 1, w);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                // allowed local query columns of this tile: qmin .. qmax
                const int qmin = q_lo - m0, qmax = q_hi - m0;
                const bool full_row = qmin <= 64 * gq && qmax >= 64 * gq + 63;
                const bool any_mask = __any_sync(0xffffffffu, !full_row);
                const float* lse_t = sLSE + st * 128 + 64 * gq;
                const float* del_t = sDel + st * 128 + 64 * gq;
                const float2 c2v = make_float2(c2, c2);
                uint8_t* ds_row = smem + C::OFF_DS + gq * 128 * 128 + r * 128;
                // the two 32-column halves one after the other, so only one half's values are live;
                // on tiles without masking or rows past the sequence one pair in kBwdFmaExpEvery takes
                // its exponentials from the FMA pipe (both warpgroups run this step at the same time, so
                // they share the exp2 unit; one pair in 6 measured best: +3 % dense, +6 % long-context
                // GQA, +7 % varlen D = 64 over none, ahead of one in 3 or 4)
                auto grad = [&](auto poly) {
                constexpr int kEvery = decltype(poly)::value ? kBwdFmaExpEvery : 0;
                constexpr int kMod = kEvery > 0 ? kEvery : 1;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t sh[32], dh[32];
                    tmem_ld32(tmem + lb + C::COL_S + 64 * gq + 32 * half, sh);
                    tmem_ld32(tmem + lb + C::COL_DP + 64 * gq + 32 * half, dh);
                    tmem_ld_wait_tie(sh);
                    reg_tie(dh);
                    uint32_t pp[16], dd[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float4 l4 = *reinterpret_cast<const float4*>(lse_t + half * 32 + e);
                        const float4 d4 = *reinterpret_cast<const float4*>(del_t + half * 32 + e);
#pragma unroll
                        for (int x = 0; x < 4; x += 2) {
                            const float la = x == 0 ? l4.x : l4.z, lbv = x == 0 ? l4.y : l4.w;
                            const float dla = x == 0 ? d4.x : d4.z, dlb = x == 0 ? d4.y : d4.w;
                            const float2 sv = make_float2(__uint_as_float(sh[e + x]), __uint_as_float(sh[e + x + 1]));
                            const float2 dv = make_float2(__uint_as_float(dh[e + x]), __uint_as_float(dh[e + x + 1]));
                            const float2 a = ffma2(sv, c2v, make_float2(la, lbv));
                            float2 pr = (kEvery > 0 && ((e + x) / 2) % kMod == kMod - 1)
                                            ? exp2_fma2(a) : make_float2(ex2_approx(a.x), ex2_approx(a.y));
                            if (any_mask) {
                                const int qc = 64 * gq + half * 32 + e + x;
                                pr.x = (qc >= qmin && qc <= qmax) ? pr.x : 0.f;
                                pr.y = (qc + 1 >= qmin && qc + 1 <= qmax) ? pr.y : 0.f;
                            }
                            const float2 ds = fmul2(pr, fadd2(dv, make_float2(dla, dlb)));
                            pp[(e + x) / 2] = pack_bf16x2(pr.x, pr.y);
                            dd[(e + x) / 2] = pack_bf16x2(ds.x, ds.y);
                        }
                    }
                    // P^T, dS^T of query columns [64 gq + 32 half, +32) -> packed S^T columns
                    // [64 gq + 32 half, +16) and [64 gq + 32 half + 16, +16): the columns just read
                    tmem_st16(tmem + lb + C::COL_S + 64 * gq + 32 * half, pp);
                    tmem_st16(tmem + lb + C::COL_S + 64 * gq + 32 * half + 16, dd);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int cin = half * 4 + q4;            // 16-byte chunk of the 64-query box row
                        *reinterpret_cast<uint4*>(ds_row + ((cin ^ (r & 7)) << 4)) =
                            make_uint4(dd[4 * q4], dd[4 * q4 + 1], dd[4 * q4 + 2], dd[4 * q4 + 3]);
                    }
                }
                };
                if (kBwdFmaExpEvery > 0 && !any_mask && m0 + 128 <= t.Lq) grad(std::true_type{});
                else grad(std::false_type{});
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(gq == 0 ? p_full : p_full_hi);
            }
            if (!ok) break;
            // -------------------------------------------------- epilogue: warpgroup 0 writes dV, 1 writes dK
            if (!mbar_wait(dkv_full, unit_it & 1, w)) { ok = false; break; }
            ++unit_it;
            tc_fence_after();
            const uint32_t col = gq == 0 ? C::COL_DV : C::COL_DK;
            const float mul = gq == 0 ? 1.f : p.scale;
            const float2 mul2 = make_float2(mul, mul);
            // this warpgroup's half of the dS buffer (16 KB) is free: the last dQ product that read it is
            // complete (dkv_full), and this warpgroup is its next writer
            uint8_t* half_buf = smem + C::OFF_DS + gq * (C::DS_BYTES / 2);
            const BUnit te = decode_bunit(p, u);     // decoded again: nothing of it stays live over the tiles
            if (te.n0 + 128 <= te.Lk) {
                // a whole key tile: each 64-column box goes to shared memory in the tensor map's 128-byte
                // swizzle (thread = row) and leaves with one TMA store; the box is refilled only after
                // the previous store has read it
                const bool issuer = (warp & 3) == 0 && lane == 0;
                const CUtensorMap* map = gq == 0 ? &tmDV : &tmDK;
#pragma unroll 1
                for (int bx = 0; bx < D / 64; ++bx) {
                    if (bx > 0) {
                        if (issuer) bulk_wait_read_all();
                        named_bar_sync(1 + gq, 128);
                    }
#pragma unroll 1
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t ra[32];
                        tmem_ld32(tmem + lb + col + bx * 64 + cc * 32, ra);
                        tmem_ld_wait_tie(ra);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 v = fmul2(make_float2(__uint_as_float(ra[8 * q + 2 * e]),
                                                                   __uint_as_float(ra[8 * q + 2 * e + 1])), mul2);
                                pk[e] = pack_bf16x2(v.x, v.y);
                            }
                            const int ch = cc * 4 + q;   // 16-byte chunk of the 128-byte box row
                            *reinterpret_cast<uint4*>(half_buf + r * 128 + ((ch ^ (r & 7)) << 4)) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                    fence_proxy_async_smem();
                    named_bar_sync(1 + gq, 128);
                    if (issuer) {
                        tma_store_3d(map, smem_u32(half_buf), bx * 64, te.hk, te.k_start + te.n0);
                        bulk_commit();
                    }
                }
                // the next tile's dS^T rows go into this buffer: wait until the last store has read it
                if (issuer) bulk_wait_read_all();
                named_bar_sync(1 + gq, 128);
            } else {
                // the sequence's last, partial key tile: rows leave through 2 KB per warp of the same
                // buffer, 8 rows x 64 bytes per store, and only the rows inside the sequence are written
                uint8_t* stg = half_buf + (warp & 3) * 2048;
                __nv_bfloat16* gdst = out_row(te);
                const int nvalid = min(max(te.Lk - te.n0 - (warp & 3) * 32, 0), 32);
                const long long rstride = static_cast<long long>(p.Hkv) * D * 2;
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t ra[32];
                    tmem_ld32(tmem + lb + col + cc * 32, ra);
                    tmem_ld_wait_tie(ra);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 v = fmul2(make_float2(__uint_as_float(ra[8 * q + 2 * e]),
                                                               __uint_as_float(ra[8 * q + 2 * e + 1])), mul2);
                            pk[e] = pack_bf16x2(v.x, v.y);
                        }
                        stg_put(stg, q, pk[0], pk[1], pk[2], pk[3]);
                    }
                    stg_flush(stg, reinterpret_cast<uint8_t*>(gdst + cc * 32), rstride, nvalid);
                }
            }
            tc_fence_before();
        }
        if ((warp & 3) == 0 && lane == 0) bulk_wait_all();   // this thread's dK / dV stores are complete
    }

    __syncthreads();
    if (threadIdx.x == 0) grid_dep_launch();   // this CTA is done: the dQ convert may be scheduled
    if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) {
        }
    }
    if (warp == MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------- two items in flight (D = 128, no dQ)
// The main kernel of the deterministic backward at head dim 128 (dQ comes from the query-tile-stationary
// pass of bwd_dq.cu), with query items of 64 rows and two tensor-memory buffers, so that the gradient step
// of one item overlaps the tensor-core work of the next:
//   tensor memory: dV [0,128) | dK [128,256) | buffer 0 [256,384) | buffer 1 [384,512),
//   buffer b = S^T (64 columns) | dP^T (64 columns); item i uses buffer i % 2.
// Items alternate between the two compute warpgroups (warpgroup b takes the items of buffer b, the low /
// high 64 query rows of every 128-row query tile).  Per item the MMA warp issues S^T, dP^T of item i,
// then dV += P^T dO, dK += dS^T Q of item i - 1, so the tensor core works on one item while a warpgroup
// works on the other.  A warpgroup packs P^T and dS^T (bf16 pairs) into the 32-column halves of S^T it
// has just read.  Measured on B200 this beats the one-item-at-a-time kernel only without the dQ product:
// with it, the 64-query products read K, V and K^T from shared memory twice per 128-row tile and the
// tensor pipe, not the gradient step, sets the pace.
struct PPCfg {
    static constexpr int D = 128;
    static constexpr int ST = 3;                                 // Q / dO item stages
    static constexpr uint32_t KV_BYTES = 128 * D * 2;            // K or V tile: two [128 x 64] boxes
    static constexpr uint32_t IT_BYTES = 64 * D * 2;             // Q or dO item: two [64 x 64] boxes
    static constexpr uint32_t OFF_K = 0, OFF_V = KV_BYTES, OFF_Q = 2 * KV_BYTES, OFF_DO = OFF_Q + ST * IT_BYTES,
                              OFF_STAT = OFF_DO + ST * IT_BYTES, OFF_STG = OFF_STAT + 2 * ST * 64 * 4,
                              OFF_BAR = OFF_STG + 8 * 2048;   // 2 KB per compute warp for the output rows
    // kv_full, kv_empty, q_full[ST], q_empty[ST], s_full[2], p_full[2], dkv_full, dkv_empty
    static constexpr int NUM_BARS = 2 + 2 * ST + 4 + 2;
    static constexpr size_t SMEM = OFF_BAR + NUM_BARS * 8 + 16;
    static constexpr uint32_t COL_DV = 0, COL_DK = 128;
    static constexpr uint32_t COL_S(int b) { return 256 + 128 * b; }
    static constexpr uint32_t COL_DP(int b) { return 256 + 128 * b + 64; }
    // packed P^T / dS^T of item queries [16 kk, 16 kk + 16): in the 32-column half (kk >> 1) of S^T
    static constexpr uint32_t COL_P(int b, int kk) { return COL_S(b) + (kk >> 1) * 32 + (kk & 1) * 8; }
    static constexpr uint32_t COL_DSP(int b, int kk) { return COL_P(b, kk) + 16; }
    // 12 warps: 0-3 / 4-7 compute warpgroups 0 / 1, 8 producer, 9 MMA, 10-11 idle
    static constexpr int THREADS = 384, LAUNCH_REGS = 168, COMPUTE_REGS = 200, OTHER_REGS = 96;
    static_assert(2 * 128 * COMPUTE_REGS + 128 * OTHER_REGS <= THREADS * LAUNCH_REGS, "register split");
    static_assert(SMEM <= 232448, "shared memory budget");
};

__global__ void __launch_bounds__(384, 1)
    bwd_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ BwdParams p) {
    using C = PPCfg;
    constexpr int D = C::D;
    constexpr int ST = C::ST;
    extern __shared__ __align__(1024) uint8_t smem[];
    float* sLSE = reinterpret_cast<float*>(smem + C::OFF_STAT);          // [ST][64], -LSE2
    float* sDel = sLSE + ST * 64;                                        // [ST][64], -Delta
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t kv_full = b0, kv_empty = b0 + 8;
    auto q_full = [&](int s) { return b0 + 8u * (2 + s); };
    auto q_empty = [&](int s) { return b0 + 8u * (2 + ST + s); };
    const uint32_t bb = b0 + 8u * (2 + 2 * ST);
    auto s_full = [&](int b) { return bb + 8u * b; };
    auto p_full = [&](int b) { return bb + 16 + 8u * b; };
    const uint32_t dkv_full = bb + 32, dkv_empty = bb + 40;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int PRODUCER = 8, MMA = 9;

    if ((smem_u32(smem) & 1023u) != 0) {   // the swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicCAS(p.status, 0, 2);
        return;
    }
    if (threadIdx.x == 0) {
        mbar_init(bars + 0, 1);
        mbar_init(bars + 1, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(bars + 2 + s, 33);        // 32 producer lanes (statistics) + the TMA expect-tx arrival
            mbar_init(bars + 2 + ST + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars + 2 + 2 * ST + b, 1);        // s_full[b]
            mbar_init(bars + 2 + 2 * ST + 2 + b, 128);  // p_full[b]: compute warpgroup b
        }
        mbar_init(bars + 2 + 2 * ST + 4, 1);            // dkv_full
        mbar_init(bars + 2 + 2 * ST + 5, 256);          // dkv_empty: both epilogues read dV / dK
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == PRODUCER && lane == 0) {
        tma_prefetch_map(&tmQ);
        tma_prefetch_map(&tmK);
        tma_prefetch_map(&tmV);
        tma_prefetch_map(&tmDO);
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
    const int G = p.group;

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::OTHER_REGS));
        if (warp == PRODUCER) {
            // -------------------------------------------------------- producer (whole warp)
            uint32_t unit_it = 0, q_it = 0;
            bool ok = true;
            for (int k = 0, u = snake_unit(0, p.num_units); u >= 0 && ok; u = snake_unit(++k, p.num_units)) {
                if (u >= p.num_units) continue;
                const BUnit t = decode_bunit(p, u);
                if (t.skip || t.n_it == 0) continue;
                if (unit_it > 0 && !mbar_wait(kv_empty, (unit_it - 1) & 1, w)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(kv_full, 2 * C::KV_BYTES);
#pragma unroll
                    for (int c = 0; c < D / 64; ++c) {
                        tma_load_3d(smem_u32(smem + C::OFF_K + c * 128 * 128), &tmK, kv_full, c * 64, t.hk,
                                    t.k_start + t.n0);
                        tma_load_3d(smem_u32(smem + C::OFF_V + c * 128 * 128), &tmV, kv_full, c * 64, t.hk,
                                    t.k_start + t.n0);
                    }
                }
                ++unit_it;
                for (int it = 0; it < t.n_it && ok; ++it) {
                    const int h = t.hk * G + it / t.n_m;
                    for (int qh = 0; qh < 2; ++qh, ++q_it) {
                        const int row0 = (t.m_start + it % t.n_m) * 128 + 64 * qh;
                        const int st = q_it % ST;
                        if (q_it >= ST && !mbar_wait(q_empty(st), ((q_it / ST) - 1) & 1, w)) { ok = false; break; }
                        // item statistics; rows past the sequence get LSE2 = +inf (P = 0) and Delta = 0
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int qi = lane * 2 + e;
                            const int row = row0 + qi;
                            const bool in = row < t.Lq;
                            const size_t idx = static_cast<size_t>(h) * p.Tq + t.q_start + row;
                            // stored negated, so the gradient step adds them (no negation per element)
                            sLSE[st * 64 + qi] = in ? -__ldg(p.lse2 + idx) : -INFINITY;
                            sDel[st * 64 + qi] = in ? -__ldg(p.delta + idx) : 0.f;
                        }
                        if (lane == 0) {
                            mbar_arrive_expect_tx(q_full(st), 2 * C::IT_BYTES);
#pragma unroll
                            for (int c = 0; c < D / 64; ++c) {
                                tma_load_3d(smem_u32(smem + C::OFF_Q + st * C::IT_BYTES + c * 64 * 128), &tmQ,
                                            q_full(st), c * 64, h, t.q_start + row0);
                                tma_load_3d(smem_u32(smem + C::OFF_DO + st * C::IT_BYTES + c * 64 * 128), &tmDO,
                                            q_full(st), c * 64, h, t.q_start + row0);
                            }
                        }
                        mbar_arrive(q_full(st));
                    }
                }
            }
            __syncwarp();
        } else if (warp == MMA) {
            // -------------------------------------------------------- MMA issuer
            if (lane == 0) {
                constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);    // S^T, dP^T of an item
                constexpr uint32_t id_t = idesc_bf16_f32(128, D, false, true);      // dV, dK (A in tensor memory)
                // descriptor low words advanced by constant offsets >> 4 (one add per operand per MMA)
                constexpr uint32_t IT16 = C::IT_BYTES >> 4, ROWS16 = (16 * 128) >> 4;
                const uint32_t dK0 = sdesc_lo(smem_u32(smem + C::OFF_K), 16), dV0 = sdesc_lo(smem_u32(smem + C::OFF_V), 16);
                const uint32_t dQ0 = sdesc_lo(smem_u32(smem + C::OFF_Q), 16), dO0 = sdesc_lo(smem_u32(smem + C::OFF_DO), 16);
                const uint32_t dQ0n = sdesc_lo(smem_u32(smem + C::OFF_Q), 64 * 128);
                const uint32_t dO0n = sdesc_lo(smem_u32(smem + C::OFF_DO), 64 * 128);
                auto achunk = [](int kk) { return static_cast<uint32_t>(((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4); };
                auto bchunk = [](int kk) { return static_cast<uint32_t>(((kk >> 2) * 64 * 128 + (kk & 3) * 32) >> 4); };
                uint32_t unit_it = 0, q_it = 0, gi = 0;
                bool ok = true;
                // dV, dK of item g (buffer g % 2, stage st); `first`: the unit's first item overwrites dV, dK
                auto post = [&](uint32_t g, int st, bool first) -> bool {
                    const int b = g & 1;
                    if (!mbar_wait(p_full(b), (g >> 1) & 1, w)) return false;
                    // the previous unit's epilogues must have read dV and dK before they are overwritten
                    if (first && unit_it > 0 && !mbar_wait(dkv_empty, (unit_it - 1) & 1, w)) return false;
                    tc_fence_after();
                    const uint32_t qn = dQ0n + st * IT16, on = dO0n + st * IT16;
                    const uint32_t acc0 = first ? 0u : 1u;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {     // K-dim = 64 item queries
                        umma_ts_lo(tmem + C::COL_DV, tmem + C::COL_P(b, kk), on + kk * ROWS16, id_t, kk > 0 ? 1u : acc0);
                        umma_ts_lo(tmem + C::COL_DK, tmem + C::COL_DSP(b, kk), qn + kk * ROWS16, id_t, kk > 0 ? 1u : acc0);
                    }
                    umma_commit(q_empty(st));
                    return true;
                };
                for (int k = 0, u = snake_unit(0, p.num_units); u >= 0 && ok; u = snake_unit(++k, p.num_units)) {
                    if (u >= p.num_units) continue;
                    const BUnit t = decode_bunit(p, u);
                    if (t.skip || t.n_it == 0) continue;
                    if (!mbar_wait(kv_full, unit_it & 1, w)) { ok = false; break; }
                    const int items = 2 * t.n_it;
                    uint32_t prev_g = 0;
                    int prev_st = 0;
                    for (int i = 0; i < items; ++i, ++q_it, ++gi) {
                        const int st = q_it % ST;
                        const int b = gi & 1;
                        if (!mbar_wait(q_full(st), (q_it / ST) & 1, w)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t qd = dQ0 + st * IT16, od = dO0 + st * IT16;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_ss_lo(tmem + C::COL_S(b), dK0 + achunk(kk), qd + bchunk(kk), id_s, kk > 0);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            umma_ss_lo(tmem + C::COL_DP(b), dV0 + achunk(kk), od + bchunk(kk), id_s, kk > 0);
                        umma_commit(s_full(b));
                        // the previous item's products, while warpgroup b works on this one
                        if (i > 0 && !post(prev_g, prev_st, i == 1)) { ok = false; break; }
                        prev_g = gi;
                        prev_st = st;
                    }
                    if (!ok) break;
                    if (!post(prev_g, prev_st, items == 1)) break;
                    umma_commit(dkv_full);
                    umma_commit(kv_empty);
                    ++unit_it;
                }
            }
            __syncwarp();
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::COMPUTE_REGS));
        // ------------------------------------------------------------ compute warpgroups (thread = key row)
        const int gb = warp >> 2;                  // buffer / item parity of this warpgroup
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lb = tmem_lane_base(warp & 3);
        const float c2 = p.scale_log2;
        const float2 c2v = make_float2(c2, c2);
        uint32_t unit_it = 0, q_it = 0, gi = 0;
        bool ok = true;
        for (int k = 0, u = snake_unit(0, p.num_units); u >= 0 && ok; u = snake_unit(++k, p.num_units)) {
            if (u >= p.num_units) continue;
            const BUnit t = decode_bunit(p, u);
            if (t.skip) continue;
            const int kj = t.n0 + r;                 // key index inside the sequence
            const bool kvalid = kj < t.Lk;
            const size_t krow = (static_cast<size_t>(t.k_start) + kj) * p.Hkv + t.hk;
            __nv_bfloat16* gdst = (gb == 0 ? p.dv : p.dk) + krow * D;
            if (t.n_it == 0) {
                if (kvalid) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(gdst)[c] = z;
                }
                continue;
            }
            // this key row is seen by query rows q_lo .. q_hi of the sequence (none if past the sequence)
            int q_lo = -0x40000000, q_hi = 0x40000000;
            if (p.wr >= 0) q_lo = kj - (t.Lk - t.Lq) - p.wr;
            if (p.wl >= 0) q_hi = kj - (t.Lk - t.Lq) + p.wl;
            if (!kvalid) q_lo = 0x40000000;
            for (int it = 0; it < t.n_it && ok; ++it) {
                for (int qh = 0; qh < 2; ++qh, ++q_it, ++gi) {
                    if ((gi & 1) != static_cast<uint32_t>(gb)) continue;
                    const int row0 = (t.m_start + it % t.n_m) * 128 + 64 * qh;
                    const int st = q_it % ST;
                    bool got = mbar_wait(s_full(gb), (gi >> 1) & 1, w);
                    got = got && mbar_wait(q_full(st), (q_it / ST) & 1, w);
                    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                    tc_fence_after();
                    // allowed item query columns: qmin .. qmax
                    const int qmin = q_lo - row0, qmax = q_hi - row0;
                    const bool any_mask = __any_sync(0xffffffffu, !(qmin <= 0 && qmax >= 63));
                    const float* lse_t = sLSE + st * 64;
                    const float* del_t = sDel + st * 64;
                    // the same FMA-pipe share of the exponentials as bwd_kernel, on the same elements and under
                    // the same condition (no masked column in the warp's 64, the whole 128-row query tile inside
                    // the sequence), so both backward modes compute identical P^T and dS^T
                    auto grad = [&](auto poly) {
                    constexpr int kEvery = decltype(poly)::value ? kBwdFmaExpEvery : 0;
                    constexpr int kMod = kEvery > 0 ? kEvery : 1;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t sh[32], dh[32];
                        tmem_ld32(tmem + lb + C::COL_S(gb) + 32 * half, sh);
                        tmem_ld32(tmem + lb + C::COL_DP(gb) + 32 * half, dh);
                        tmem_ld_wait_tie(sh);
                        reg_tie(dh);
                        uint32_t pp[16], dd[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 l4 = *reinterpret_cast<const float4*>(lse_t + half * 32 + e);
                            const float4 d4 = *reinterpret_cast<const float4*>(del_t + half * 32 + e);
#pragma unroll
                            for (int x = 0; x < 4; x += 2) {
                                const float la = x == 0 ? l4.x : l4.z, lbv = x == 0 ? l4.y : l4.w;
                                const float dla = x == 0 ? d4.x : d4.z, dlb = x == 0 ? d4.y : d4.w;
                                const float2 sv = make_float2(__uint_as_float(sh[e + x]), __uint_as_float(sh[e + x + 1]));
                                const float2 dv = make_float2(__uint_as_float(dh[e + x]), __uint_as_float(dh[e + x + 1]));
                                const float2 a = ffma2(sv, c2v, make_float2(la, lbv));
                                float2 pr = (kEvery > 0 && ((e + x) / 2) % kMod == kMod - 1)
                                                ? exp2_fma2(a) : make_float2(ex2_approx(a.x), ex2_approx(a.y));
                                if (any_mask) {
                                    const int qc = half * 32 + e + x;
                                    pr.x = (qc >= qmin && qc <= qmax) ? pr.x : 0.f;
                                    pr.y = (qc + 1 >= qmin && qc + 1 <= qmax) ? pr.y : 0.f;
                                }
                                const float2 ds = fmul2(pr, fadd2(dv, make_float2(dla, dlb)));
                                pp[(e + x) / 2] = pack_bf16x2(pr.x, pr.y);
                                dd[(e + x) / 2] = pack_bf16x2(ds.x, ds.y);
                            }
                        }
                        // packed P^T, dS^T of item queries [32 half, +32) -> the 32 S^T columns just read
                        tmem_st16(tmem + lb + C::COL_S(gb) + 32 * half, pp);
                        tmem_st16(tmem + lb + C::COL_S(gb) + 32 * half + 16, dd);
                    }
                    };
                    if (kBwdFmaExpEvery > 0 && !any_mask && row0 - 64 * qh + 128 <= t.Lq) grad(std::true_type{});
                    else grad(std::false_type{});
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(p_full(gb));
                }
            }
            if (!ok) break;
            // -------------------------------------------------- epilogue: warpgroup 0 writes dV, 1 writes dK
            if (!mbar_wait(dkv_full, unit_it & 1, w)) { ok = false; break; }
            ++unit_it;
            tc_fence_after();
            const uint32_t col = gb == 0 ? C::COL_DV : C::COL_DK;
            const float mul = gb == 0 ? 1.f : p.scale;
            const float2 mul2 = make_float2(mul, mul);
            uint8_t* stg = smem + C::OFF_STG + warp * 2048;
            const int nvalid = min(max(t.Lk - t.n0 - (warp & 3) * 32, 0), 32);
            const long long rstride = static_cast<long long>(p.Hkv) * D * 2;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t ra[32];
                tmem_ld32(tmem + lb + col + cc * 32, ra);
                tmem_ld_wait_tie(ra);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 v = fmul2(make_float2(__uint_as_float(ra[8 * q + 2 * e]), __uint_as_float(ra[8 * q + 2 * e + 1])), mul2);
                        pk[e] = pack_bf16x2(v.x, v.y);
                    }
                    stg_put(stg, q, pk[0], pk[1], pk[2], pk[3]);
                }
                stg_flush(stg, reinterpret_cast<uint8_t*>(gdst + cc * 32), rstride, nvalid);
            }
            tc_fence_before();
            mbar_arrive(dkv_empty);
        }
    }

    __syncthreads();
    if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) {
        }
    }
    if (warp == MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------- preprocess
// One warp per (query token, head): Delta = sum_d dO * O (fp32), LSE2 = LSE * log2(e)
// (+inf where LSE = -inf).  Also zeroes the dQ accumulator (grid-stride) unless dq_acc is NULL, and
// the main kernel's unit counter unless counter is NULL.  With l2_keep the zeroed accumulator is
// written with the L2 evict_last policy and O, dO are read with evict_first, so that the accumulator
// stays in L2 for the main kernel's reduce-adds and the convert.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* out, const __nv_bfloat16* dout,
                                                      const float* lse, float* lse2, float* delta, float* dq_acc,
                                                      int* counter, int Tq, int Hq, int Sq, long long lse_sB,
                                                      long long lse_sH, int lse_sT, int l2_keep) {
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    // the main kernel may start its prologue now; it waits for this grid before reading anything written here
    if (threadIdx.x == 0) grid_dep_launch();
    if (counter != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *counter = 0;
    const long long rows = static_cast<long long>(Tq) * Hq;
    const uint64_t pol_in = l2_keep ? l2_policy_first() : l2_policy_normal();
    if (dq_acc != nullptr) {
        const uint64_t pol_z = l2_keep ? l2_policy_last() : l2_policy_normal();
        const long long n4 = rows * D / 4;
        float4* z = reinterpret_cast<float4*>(dq_acc);
        for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
             i += static_cast<long long>(gridDim.x) * blockDim.x)
            st_f32x4_hint(z + i, make_float4(0.f, 0.f, 0.f, 0.f), pol_z);
    }
    // D/8 lanes per row, 16 bytes of O and of dO per lane; 32/(D/8) rows per warp per pass.  A row's LSE is
    // loaded together with its O and dO, so that a pass waits for one round trip to memory rather than two,
    // and each iteration takes kPrePasses passes, whose loads are all in flight at once.
    constexpr int LPR = D / 8, RPW = 32 / LPR, NP = kPrePasses;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int sub = lane / LPR, sl = lane % LPR;
    const long long stride = nwarps * RPW;
    for (long long row0 = gw * RPW; row0 < rows; row0 += NP * stride) {
        uint4 a[NP], b[NP];
        float l[NP];
        size_t wi[NP];
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const long long row = row0 + k * stride + sub;
            a[k] = make_uint4(0, 0, 0, 0);
            b[k] = a[k];
            l[k] = 0.f;
            wi[k] = 0;
            if (row < rows) {
                a[k] = ld_u32x4_hint(out + row * D + sl * 8, pol_in);
                b[k] = ld_u32x4_hint(dout + row * D + sl * 8, pol_in);
                const int tok = static_cast<int>(row / Hq), h = static_cast<int>(row % Hq);
                if (sl == 0) {
                    long long li;
                    if (lse_sT) {
                        li = h * lse_sH + tok;
                    } else {
                        const int bb = tok / Sq, i = tok - bb * Sq;
                        li = bb * lse_sB + h * lse_sH + i;
                    }
                    l[k] = lse[li];
                }
                wi[k] = static_cast<size_t>(h) * Tq + tok;
            }
        }
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const uint32_t av[4] = {a[k].x, a[k].y, a[k].z, a[k].w}, bv[4] = {b[k].x, b[k].y, b[k].z, b[k].w};
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
                const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
                s = fmaf(fa.x, fb.x, s);
                s = fmaf(fa.y, fb.y, s);
            }
#pragma unroll
            for (int x = LPR / 2; x > 0; x >>= 1) s += __shfl_xor_sync(0xffffffffu, s, x);
            if (sl == 0 && row0 + k * stride + sub < rows) {
                lse2[wi[k]] = (l[k] == -INFINITY) ? INFINITY : l[k] * 1.4426950408889634f;
                delta[wi[k]] = s;
            }
        }
    }
}

// ---------------------------------------------------------------------------- convert
// dQ[tok][h][:] = bf16(scale * dQacc[h][:/4][tok][:%4]) for 32 tokens of one head per block: float4 columns
// of 32 consecutive tokens are read (512 bytes per warp), staged in shared memory with one float4 of padding
// per token row (each group of 8 lanes then writes 8 different bank groups), and leave as whole D-value rows
// (D / 8 lanes x 16 bytes per token).  Launched after the main kernel with programmatic serialization: the
// wait below covers the main kernel's last reduce-adds.  The accumulator is dead once read: the 128-byte
// L2 lines that lie wholly inside this block's token range are dropped without being written back (a line
// shared with a neighbouring block is left alone), which saves its write-back to HBM.
template <int D>
__global__ void __launch_bounds__(256) bwd_convert_kernel(const float* dq_acc, __nv_bfloat16* dq, int Tq, int Hq,
                                                          float scale) {
    constexpr int W4 = D / 4 + 1;                  // float4 per staged token row, with padding
    __shared__ float4 tile[32 * W4];
    grid_dep_wait();
    const int h = blockIdx.y;
    const int t0 = blockIdx.x * 32;
    const float4* src = reinterpret_cast<const float4*>(dq_acc) + static_cast<size_t>(h) * (D / 4) * Tq + t0;
    for (int i = threadIdx.x; i < 32 * (D / 4); i += blockDim.x) {
        const int d4 = i / 32, tt = i % 32;
        if (t0 + tt < Tq) tile[tt * W4 + d4] = __ldcs(src + static_cast<size_t>(d4) * Tq + tt);
    }
    __syncthreads();
    if (threadIdx.x < (D / 4) * 4) {
        // row d4 of this head: bytes [16 (rowbase + t0), 16 (rowbase + t1)) of the accumulator, whose base
        // is 256-byte aligned; line k of the whole lines inside that range
        const int d4 = threadIdx.x >> 2, k = threadIdx.x & 3;
        const long long rowbase = (static_cast<long long>(h) * (D / 4) + d4) * Tq;
        const long long b0 = (rowbase + t0) * 16, b1 = (rowbase + min(t0 + 32, Tq)) * 16;
        const long long line = ((b0 + 127) & ~127LL) + 128LL * k;
        if (line + 128 <= b1) l2_discard_line(reinterpret_cast<const char*>(dq_acc) + line);
    }
    constexpr int LPR = D / 8;                     // lanes per token row, 8 values (16 bytes) each
    for (int i = threadIdx.x; i < 32 * LPR; i += blockDim.x) {
        const int tt = i / LPR, c8 = i % LPR;
        if (t0 + tt >= Tq) continue;
        const float4 a = tile[tt * W4 + 2 * c8], b = tile[tt * W4 + 2 * c8 + 1];
        const uint4 o = make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                                   pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
        reinterpret_cast<uint4*>(dq + (static_cast<size_t>(t0 + tt) * Hq + h) * D)[c8] = o;
    }
}

// fp32 dQ accumulator | LSE2 | Delta | 256 bytes for the main kernel's unit counter
size_t bwd_workspace_bytes(long long Tq, int Hq, int D) {
    const size_t acc = static_cast<size_t>(Tq) * Hq * D * 4;
    const size_t stat = static_cast<size_t>(Tq) * Hq * 4;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    return up(acc) + 2 * up(stat) + 256;
}

int* bwd_unit_counter(void* workspace, long long Tq, int Hq, int D) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t acc = static_cast<size_t>(Tq) * Hq * D * 4;
    const size_t stat = static_cast<size_t>(Tq) * Hq * 4;
    return reinterpret_cast<int*>(static_cast<char*>(workspace) + up(acc) + 2 * up(stat));
}

// Key-tile units are dealt in chunks of `chunk` (sequence, KV head) groups, heaviest key tile first
// inside a chunk, so that the CTAs working at one time share the Q, dO and dQ accumulator of a few
// heads in L2.  A chunk holds enough units for every CTA (twice over) and, beyond that, as many groups
// as fit about 96 MB of Q, dO and fp32 dQ.
int bwd_chunk_groups(int num_groups, int units_per_group, int group_q_heads, int max_len, int D, int num_sms) {
    const double per_group = static_cast<double>(group_q_heads) * max_len * D * 8.0;
    long long by_l2 = static_cast<long long>(96.0 * (1 << 20) / (per_group > 1.0 ? per_group : 1.0));
    const long long by_balance = (2LL * num_sms + units_per_group - 1) / (units_per_group > 0 ? units_per_group : 1);
    long long c = by_l2 > by_balance ? by_l2 : by_balance;
    if (c < 1) c = 1;
    if (c > num_groups) c = num_groups;
    // chunks of equal size, so the schedule does not end on a lone small chunk
    const long long n_chunks = (num_groups + c - 1) / c;
    return static_cast<int>((num_groups + n_chunks - 1) / n_chunks);
}

template <int D, bool DQ>
static int run_bwd(const Problem& pr, const void* out, const void* dout, const float* lse, void* dq, void* dk, void* dv,
                   void* workspace, const Device& dev, cudaStream_t stream) {
    using C = BwdCfg<D>;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    float* dq_acc = static_cast<float*>(workspace);
    float* lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + up(static_cast<size_t>(pr.Tq) * pr.Hq * D * 4));
    float* delta = reinterpret_cast<float*>(reinterpret_cast<char*>(lse2) + up(static_cast<size_t>(pr.Tq) * pr.Hq * 4));
    const size_t acc_bytes = static_cast<size_t>(pr.Tq) * pr.Hq * D * 4;
    const int l2_keep = (DQ && acc_bytes <= kBwdL2KeepBytes) ? 1 : 0;

    {
        const long long rows = static_cast<long long>(pr.Tq) * pr.Hq;
        long long blocks = (rows + 7) / 8;
        const long long cap = static_cast<long long>(dev.num_sms) * 16;
        if (blocks > cap) blocks = cap;
        bwd_pre_kernel<D><<<static_cast<int>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse, lse2, delta,
            DQ ? dq_acc : nullptr, bwd_unit_counter(workspace, pr.Tq, pr.Hq, D), pr.Tq, pr.Hq, pr.Sq, pr.lse_sB,
            pr.lse_sH, pr.lse_sT, l2_keep);
        if (cudaPeekAtLastError() != cudaSuccess) return 5;
    }

    alignas(64) CUtensorMap mq, mk, mv, mdo;
    const uint64_t rq = static_cast<uint64_t>(pr.Hq) * D * 2, rk = static_cast<uint64_t>(pr.Hkv) * D * 2;
    if (!make_map_3d_bf16(&mq, pr.q, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, 128)) return 5;
    if (!make_map_3d_bf16(&mdo, dout, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, 128)) return 5;
    if (!make_map_3d_bf16(&mk, pr.k, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, 128)) return 5;
    if (!make_map_3d_bf16(&mv, pr.v, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, 128)) return 5;
    alignas(64) CUtensorMap mdk, mdv;   // dK / dV stores of whole key tiles
    if (!make_map_3d_bf16(&mdk, dk, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, 128)) return 5;
    if (!make_map_3d_bf16(&mdv, dv, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, 128)) return 5;

    BwdParams p;
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
    p.n_blocks = (pr.Sk + 127) / 128;
    const long long units = static_cast<long long>(p.n_blocks) * pr.num_seqs * pr.Hkv;
    if (units > 0x7fffffffLL) return 2;
    p.num_units = static_cast<int>(units);
    p.scale = pr.scale;
    p.scale_log2 = pr.scale * 1.4426950408889634f;
    p.wl = pr.wl;
    p.wr = pr.wr;
    p.chunk = bwd_chunk_groups(pr.num_seqs * pr.Hkv, p.n_blocks, p.group, pr.Sq, D, dev.num_sms);
    p.l2_keep = l2_keep;
    p.counter = bwd_unit_counter(workspace, pr.Tq, pr.Hq, D);
    p.timeout_ns = dev.timeout_ns;
    p.status = dev.status;

    auto kern = bwd_kernel<D, DQ>;
    static bool set[64] = {};
    if (!set[dev.id & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM)) !=
            cudaSuccess)
            return 5;
        // the setmaxnreg split assumes exactly LAUNCH_REGS per thread at launch
        cudaFuncAttributes fa_attr;
        if (cudaFuncGetAttributes(&fa_attr, kern) != cudaSuccess || fa_attr.numRegs != C::LAUNCH_REGS) return 2;
        set[dev.id & 63] = true;
    }
    const int grid = p.num_units < dev.num_sms ? p.num_units : dev.num_sms;
    if (grid > 0) {
        prof_before(1, stream);
        if (launch_dependent(kern, dim3(grid), dim3(C::THREADS), C::SMEM, stream, mq, mk, mv, mdo, mdk, mdv, p) !=
            cudaSuccess)
            return 5;
        prof_after(1, stream);
    }
    if (!DQ) return launch_bwd_dq(pr, dout, lse2, delta, dq, dev, stream);
    const dim3 cg((pr.Tq + 31) / 32, pr.Hq);
    if (launch_dependent(bwd_convert_kernel<D>, cg, dim3(256), 0, stream, static_cast<const float*>(dq_acc),
                         static_cast<__nv_bfloat16*>(dq), pr.Tq, pr.Hq, pr.scale) != cudaSuccess)
        return 5;
    return 0;
}

// Head dim 128, deterministic: the two-items-in-flight main kernel, then the dQ pass.
static int run_bwd_pp(const Problem& pr, const void* out, const void* dout, const float* lse, void* dq, void* dk,
                      void* dv, void* workspace, const Device& dev, cudaStream_t stream) {
    using C = PPCfg;
    constexpr int D = C::D;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    float* dq_acc = static_cast<float*>(workspace);
    float* lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + up(static_cast<size_t>(pr.Tq) * pr.Hq * D * 4));
    float* delta = reinterpret_cast<float*>(reinterpret_cast<char*>(lse2) + up(static_cast<size_t>(pr.Tq) * pr.Hq * 4));
    {
        const long long rows = static_cast<long long>(pr.Tq) * pr.Hq;
        long long blocks = (rows + 7) / 8;
        const long long cap = static_cast<long long>(dev.num_sms) * 16;
        if (blocks > cap) blocks = cap;
        bwd_pre_kernel<D><<<static_cast<int>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse, lse2, delta,
            nullptr, nullptr, pr.Tq, pr.Hq, pr.Sq, pr.lse_sB, pr.lse_sH, pr.lse_sT, 0);
        if (cudaPeekAtLastError() != cudaSuccess) return 5;
    }
    alignas(64) CUtensorMap mq, mk, mv, mdo;
    const uint64_t rq = static_cast<uint64_t>(pr.Hq) * D * 2, rk = static_cast<uint64_t>(pr.Hkv) * D * 2;
    if (!make_map_3d_bf16(&mq, pr.q, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, 64)) return 5;
    if (!make_map_3d_bf16(&mdo, dout, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, 64)) return 5;
    if (!make_map_3d_bf16(&mk, pr.k, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, 128)) return 5;
    if (!make_map_3d_bf16(&mv, pr.v, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, 128)) return 5;

    BwdParams p;
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
    p.n_blocks = (pr.Sk + 127) / 128;
    const long long units = static_cast<long long>(p.n_blocks) * pr.num_seqs * pr.Hkv;
    if (units > 0x7fffffffLL) return 2;
    p.num_units = static_cast<int>(units);
    p.scale = pr.scale;
    p.scale_log2 = pr.scale * 1.4426950408889634f;
    p.wl = pr.wl;
    p.wr = pr.wr;
    p.chunk = pr.num_seqs * pr.Hkv;   // the static heaviest-first order over all groups
    p.l2_keep = 0;
    p.counter = nullptr;
    p.timeout_ns = dev.timeout_ns;
    p.status = dev.status;

    auto kern = bwd_pp_kernel;
    static bool set[64] = {};
    if (!set[dev.id & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM)) !=
            cudaSuccess)
            return 5;
        // the setmaxnreg split assumes exactly LAUNCH_REGS per thread at launch
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
    return launch_bwd_dq(pr, dout, lse2, delta, dq, dev, stream);
}

// Head dim 256: same preprocess, then the half-head-dim kernel of bwd256.cu (which also converts dQ).
static int run_bwd256(const Problem& pr, const void* out, const void* dout, const float* lse, void* dq, void* dk,
                      void* dv, void* workspace, bool det, const Device& dev, cudaStream_t stream) {
    constexpr int D = 256;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    float* dq_acc = static_cast<float*>(workspace);
    float* lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + up(static_cast<size_t>(pr.Tq) * pr.Hq * D * 4));
    float* delta = reinterpret_cast<float*>(reinterpret_cast<char*>(lse2) + up(static_cast<size_t>(pr.Tq) * pr.Hq * 4));
    const long long rows = static_cast<long long>(pr.Tq) * pr.Hq;
    long long blocks = (rows + 7) / 8;
    const long long cap = static_cast<long long>(dev.num_sms) * 16;
    if (blocks > cap) blocks = cap;
    bwd_pre_kernel<D><<<static_cast<int>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse, lse2, delta,
        det ? nullptr : dq_acc, bwd_unit_counter(workspace, pr.Tq, pr.Hq, D), pr.Tq, pr.Hq, pr.Sq, pr.lse_sB,
        pr.lse_sH, pr.lse_sT, 0);
    if (cudaPeekAtLastError() != cudaSuccess) return 5;
    const int st = launch_bwd256_main(pr, dout, lse2, delta, dq_acc, dq, dk, dv, !det, dev, stream);
    if (st != 0 || !det) return st;
    return launch_bwd_dq(pr, dout, lse2, delta, dq, dev, stream);
}

int launch_bwd(const Problem& pr, const void* out, const void* dout, const float* lse, void* dq, void* dk, void* dv,
               void* workspace, bool deterministic, const Device& dev, cudaStream_t stream) {
    switch (pr.D) {
        case 64:
            return deterministic ? run_bwd<64, false>(pr, out, dout, lse, dq, dk, dv, workspace, dev, stream)
                                 : run_bwd<64, true>(pr, out, dout, lse, dq, dk, dv, workspace, dev, stream);
        case 128:
            return deterministic ? run_bwd_pp(pr, out, dout, lse, dq, dk, dv, workspace, dev, stream)
                                 : run_bwd<128, true>(pr, out, dout, lse, dq, dk, dv, workspace, dev, stream);
        case 256: return run_bwd256(pr, out, dout, lse, dq, dk, dv, workspace, deterministic, dev, stream);
        default: return 2;
    }
}

}  // namespace fa

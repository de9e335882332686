// fwd.cu -- forward of exact tiled softmax attention on sm_100a.
//
// What it computes (flash-attention README, "How to use FlashAttention"):
//   O = softmax(scale * Q K^T + mask) V,   LSE_i = ln sum_j exp(scale q_i.k_j)
// tile by tile with an online softmax (FlashAttention fork v1.4 notes,
// section 4, softmax_rescale_o / scale_apply_exp2: running row max and row sum,
// exponentials taken as exp2 of one FMA with log2(e) folded into the scale, a
// -inf row max replaced by 0), so the score matrix never leaves the SM.
//
// Design (one persistent CTA per SM):
//   * warps 0..4*NQ-1: NQ softmax warpgroups; warpgroup i owns query tile i
//     (128 rows) of the CTA's work unit, thread t owns row t: it reads its row
//     of S from tensor memory, keeps the row max m and row sum l in registers,
//     writes P (bf16) back into tensor memory, rescales its row of O when its
//     reference max moves, and finally normalises and stores O and the LSE.
//   * warp 4*NQ: TMA producer (Q tiles once per unit, K/V tiles through a
//     KST-stage shared-memory ring, 128-byte swizzle).
//   * warp 4*NQ+1: allocates tensor memory and issues every tcgen05 MMA:
//     S_i = Q_i K^T (both operands K-major in shared memory) and
//     O_i += P_i V (P from tensor memory, V N-major in shared memory).
//   Order per KV tile j: PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so the tensor
//   core computes one tile's scores while the other tile's softmax runs.
//   * work units (sequence, head, block of NQ*128 query rows) are listed
//     heaviest first (query blocks with most KV tiles first for causal masks),
//     in chunks of heads whose K and V fit L2 together; with a workspace the
//     CTAs take them from a counter as they finish (dynamic), without one they
//     are dealt in boustrophedon order (snake_unit); the producer publishes each
//     unit to the other roles through a small shared-memory ring;
//     each query tile only visits the KV tiles its mask can reach: causal
//     blocks stop at the last KV tile they can see, and a sliding window
//     (README, flash_attn_func docstring: query i keeps the keys in
//     [i + Sk - Sq - left, i + Sk - Sq + right]) also starts late.
//
// Exactness of the deferred rescale: P, l and O are all taken against the same
// reference value m_ref of the row, which is only raised when a tile's max
// exceeds it by more than kDeferLog2 (in log2 units).  softmax(x) is independent
// of the reference subtracted, so the result is exact attention; the only effect
// is that P may reach 2^kDeferLog2 before the final division (well inside
// bf16/fp32 range).  With kDeferLog2 = 0 the reference follows every increase
// of the running max.
#include "internal.h"
#include "sm100.cuh"

#include <math.h>

#include <type_traits>

namespace fa {

struct FwdParams {
    __nv_bfloat16* o;
    float* lse;
    const int32_t* cu_q;
    const int32_t* cu_k;
    int num_seqs, Sq, Sk, Tq, Tk, Hq, Hkv, group;
    int m_blocks, num_units;
    float scale_log2;
    int wl, wr;   // window sides, -1 = unbounded; a causal mask is wr = 0
    long long lse_sB, lse_sH;
    int lse_sT;
    int chunk;      // (sequence, query head) groups per chunk of the unit list
    int* counter;   // unit counter of the dynamic schedule (zeroed before the launch), or NULL: static
    unsigned long long timeout_ns;
    int* status;
};

struct Unit {
    int b, h, q_start, k_start, Lq, Lk, q0;
    int kv0, n_kv;   // the unit loads KV tiles kv0 .. kv0 + n_kv - 1
    // query tile i uses the unit's KV tiles lo[i] .. hi[i] - 1 (relative to kv0); lo = hi: none
    // (no row inside the sequence, or no row with a key in reach)
    int lo[2], hi[2];
    bool skip;
};

// LOCAL: the window has a bounded left side, so query tiles may start past KV tile 0.
// Without it kv0 and lo[] are 0 and the accessors below fold them away.
// Unit u: the list is cut into chunks of p.chunk (sequence, query head) groups; inside a chunk the units
// run query block by query block, the blocks that see the most keys first, over the chunk's groups (so
// the CTAs of one moment share a few heads' K and V in L2).  p.chunk = all groups: heaviest first.
template <int ROWS, int BK, bool LOCAL>
__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
    Unit t;
    const int groups = p.num_seqs * p.Hq;
    const int per_chunk = p.chunk * p.m_blocks;
    const int c = u / per_chunk;
    const int g0 = c * p.chunk;
    const int cs = min(p.chunk, groups - g0);
    const int idx = u - c * per_chunk;
    const int m = p.m_blocks - 1 - idx / cs;
    const int r = g0 + idx % cs;
    t.b = r / p.Hq;
    t.h = r % p.Hq;
    if (p.cu_q != nullptr) {
        t.q_start = __ldg(p.cu_q + t.b);
        t.Lq = __ldg(p.cu_q + t.b + 1) - t.q_start;
        t.k_start = __ldg(p.cu_k + t.b);
        t.Lk = __ldg(p.cu_k + t.b + 1) - t.k_start;
        // malformed offsets can only shrink the work: rows are clipped to the tensors
        t.q_start = max(t.q_start, 0);
        t.k_start = max(t.k_start, 0);
        // (and to 2^30 tokens, the longest sequence the window arithmetic below is exact for)
        t.Lq = max(min(min(t.Lq, p.Tq - t.q_start), 1 << 30), 0);
        t.Lk = max(min(min(t.Lk, p.Tk - t.k_start), 1 << 30), 0);
    } else {
        t.q_start = t.b * p.Sq;
        t.Lq = p.Sq;
        t.k_start = t.b * p.Sk;
        t.Lk = p.Sk;
    }
    t.q0 = m * ROWS;
    t.skip = t.q0 >= t.Lq;
    t.kv0 = 0;
    t.lo[0] = t.lo[1] = 0;
    if constexpr (!LOCAL) {
        // every query tile starts at KV tile 0 and stops after the last tile its rows can see
        t.n_kv = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int row_begin = t.q0 + 128 * i;              // query tiles are 128 rows
            const int row_end = min(row_begin + 128, t.Lq);   // exclusive
            int kend = row_end > row_begin ? t.Lk : 0;
            if (p.wr >= 0 && row_end > row_begin) kend = min(kend, row_end + (t.Lk - t.Lq) + p.wr);
            t.hi[i] = kend > 0 ? (kend + BK - 1) / BK : 0;
            if (i * 128 < ROWS) t.n_kv = max(t.n_kv, t.hi[i]);
            else t.hi[i] = 0;
        }
        return t;
    }
    int f[2], e[2], kmin = 0x7fffffff, kmax = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int row_begin = t.q0 + 128 * i;
        const int row_end = min(row_begin + 128, t.Lq);
        f[i] = e[i] = 0;
        if (i * 128 < ROWS && row_end > row_begin) {
            // keys reachable from rows row_begin .. row_end-1 (lengths <= 2^30 and window sides < 2^30
            // keep every term inside int32)
            const int off = t.Lk - t.Lq;
            const int lo = max(0, row_begin + off - p.wl);
            int hi = t.Lk - 1;
            if (p.wr >= 0) hi = min(hi, row_end - 1 + off + p.wr);
            if (hi >= lo) {
                f[i] = lo / BK;
                e[i] = hi / BK + 1;
                kmin = min(kmin, f[i]);
                kmax = max(kmax, e[i]);
            }
        }
    }
    t.kv0 = kmax > 0 ? kmin : 0;
    t.n_kv = kmax > 0 ? kmax - kmin : 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        t.lo[i] = e[i] > 0 ? f[i] - t.kv0 : 0;
        t.hi[i] = e[i] > 0 ? e[i] - t.kv0 : 0;
    }
    return t;
}

template <bool LOCAL>
__device__ __forceinline__ int unit_lo(const Unit& t, int i) {
    if constexpr (LOCAL) return i == 0 ? t.lo[0] : t.lo[1];
    else return 0;
}
__device__ __forceinline__ int unit_hi(const Unit& t, int i) { return i == 0 ? t.hi[0] : t.hi[1]; }
template <bool LOCAL>
__device__ __forceinline__ int unit_kv0(const Unit& t) {
    if constexpr (LOCAL) return t.kv0;
    else return 0;
}

template <int D, int NQ, int BK, int KST>
struct FwdCfg {
    static constexpr int BM = 128;
    static constexpr int NCHUNK = D / 64;
    static constexpr uint32_t Q_BYTES = BM * D * 2;
    static constexpr uint32_t KV_BYTES = BK * D * 2;
    static constexpr int NUM_BARS = 5 * NQ + 4 * KST + 2 * kFeedSlots;
    static constexpr size_t SMEM = 1024 + NQ * Q_BYTES + 2 * KST * KV_BYTES + NUM_BARS * 8 + 16 + 4 * kFeedSlots;
    // NQ softmax warpgroups + one warpgroup holding the producer warp, the MMA warp and two idle warps
    static constexpr int THREADS = (4 * NQ + 4) * 32;
    // register split with setmaxnreg (NQ = 2): launch at 168 per thread (384 x 168 = 64512),
    // the producer/MMA warpgroup drops to 96 and the two softmax warpgroups rise to 200:
    // 2 x 128 x 200 + 128 x 96 = 63488 <= 64512.  The host checks the launch count before the first launch.
    static constexpr int LAUNCH_REGS = 168, SOFTMAX_REGS = 200, OTHER_REGS = 96;
    static_assert(NQ != 2 || 2 * 128 * SOFTMAX_REGS + 128 * OTHER_REGS <= THREADS * LAUNCH_REGS, "register split");
    static constexpr uint32_t S_COL(int i) { return i * BK; }
    static constexpr uint32_t O_COL(int i) { return NQ * BK + i * D; }
    static_assert(NQ * BK + NQ * D <= 512, "tensor memory budget");
    static_assert(D % 64 == 0 && BK % 64 == 0, "tile shape");
};

constexpr float kDeferLog2 = 8.0f;
// Share of the softmax exponentials computed on the FMA pipe (exp2_fma2) instead of the
// multi-function unit: one pair in fma_exp_every(D) of each row's pairs (tiles with masked
// scores use the multi-function unit only), 0 = none.  Measured on B200 at D = 64 and 128 with
// one pair in 2, 3, 4 and 6: every share made the forward slower (-22 % to -5 % on the dense
// and long-context workloads), so it is off: a softmax warp's exponentials are bound by its own
// instruction stream and latency, and the polynomial lengthens both.
#ifndef FA_FMA_EXP_EVERY_64
#define FA_FMA_EXP_EVERY_64 0
#endif
#ifndef FA_FMA_EXP_EVERY_128
#define FA_FMA_EXP_EVERY_128 0
#endif
#ifndef FA_FMA_EXP_EVERY_256
#define FA_FMA_EXP_EVERY_256 0
#endif
__host__ __device__ constexpr int fma_exp_every(int D) {
    return D == 64 ? FA_FMA_EXP_EVERY_64 : D == 128 ? FA_FMA_EXP_EVERY_128 : FA_FMA_EXP_EVERY_256;
}
constexpr float kLn2 = 0.69314718055994530942f;

// DYN: units come from p.counter through the shared-memory feed (varlen batches, head chunks sized for
// L2); otherwise each role walks the static boustrophedon deal itself (dense problems whose K and V fit
// L2: the static deal is balanced there, and the feed's per-unit hand-off measured 2-3 % slower).
template <int D, int NQ, int BK, int KST, bool LOCAL, bool DYN>
__global__ void __launch_bounds__(FwdCfg<D, NQ, BK, KST>::THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
    using C = FwdCfg<D, NQ, BK, KST>;
    constexpr int BM = C::BM;
    constexpr int ROWS = BM * NQ;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + NQ * C::Q_BYTES;
    uint8_t* sV = sK + KST * C::KV_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sV + KST * C::KV_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* feed_slot = reinterpret_cast<int*>(tmem_slot + 4);

    const uint32_t bar0 = smem_u32(bars);
    const UnitFeed feed{feed_slot, bar0 + 8u * (5 * NQ + 4 * KST), bar0 + 8u * (5 * NQ + 4 * KST + kFeedSlots)};
    auto q_full = [&](int i) { return bar0 + 8u * (0 * NQ + i); };
    auto q_empty = [&](int i) { return bar0 + 8u * (1 * NQ + i); };
    auto s_full = [&](int i) { return bar0 + 8u * (2 * NQ + i); };
    auto p_full = [&](int i) { return bar0 + 8u * (3 * NQ + i); };
    auto o_full = [&](int i) { return bar0 + 8u * (4 * NQ + i); };
    auto k_full = [&](int s) { return bar0 + 8u * (5 * NQ + s); };
    auto k_empty = [&](int s) { return bar0 + 8u * (5 * NQ + KST + s); };
    auto v_full = [&](int s) { return bar0 + 8u * (5 * NQ + 2 * KST + s); };
    auto v_empty = [&](int s) { return bar0 + 8u * (5 * NQ + 3 * KST + s); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr int PRODUCER = 4 * NQ;
    constexpr int MMA = 4 * NQ + 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NQ; ++i) {
            mbar_init(bars + 0 * NQ + i, 1);
            mbar_init(bars + 1 * NQ + i, 1);
            mbar_init(bars + 2 * NQ + i, 1);
            mbar_init(bars + 3 * NQ + i, 128);
            mbar_init(bars + 4 * NQ + i, 1);
        }
        for (int s = 0; s < 4 * KST; ++s) mbar_init(bars + 5 * NQ + s, 1);
        for (int s = 0; s < kFeedSlots; ++s) {
            mbar_init(bars + 5 * NQ + 4 * KST + s, 1);                       // unit published
            mbar_init(bars + 5 * NQ + 4 * KST + kFeedSlots + s, 1 + 4 * NQ); // read by the MMA and softmax warps
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == PRODUCER && lane == 0) {
        tma_prefetch_map(&tmQ);
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
    // The last warpgroup (producer, MMA issuer, two idle warps) gives registers to the softmax warpgroups;
    // each setmaxnreg is executed by all four warps of its warpgroup at the same instruction.
    if (warp >= 4 * NQ) {
    if constexpr (NQ == 2) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::OTHER_REGS));
    if (warp == PRODUCER) {
        if (lane == 0) {
            uint32_t kv_it = 0, q_it = 0;
            // DYN: units come from the counter; the next one is taken and published one ahead of the one
            // being loaded, so the counter's latency is hidden.  Static: the boustrophedon deal.
            int k_static = 0;
            auto take = [&]() -> int {
                if constexpr (DYN) {
                    const int v = atomicAdd(p.counter, 1);
                    return v < p.num_units ? v : -1;
                } else {
                    return snake_unit(k_static++, p.num_units);   // -1 at the end, num_units = an empty slot
                }
            };
            auto publish = [&](uint32_t it, int v) -> bool {
                if constexpr (!DYN) return true;
                const uint32_t s = it % kFeedSlots;
                if (it >= kFeedSlots && !mbar_wait(feed.empty0 + 8 * s, ((it / kFeedSlots) - 1) & 1, w)) return false;
                feed.slot[s] = v;
                mbar_arrive(feed.full0 + 8 * s);
                return true;
            };
            int u_next = take();
            bool ok = publish(0, u_next);
            for (uint32_t fi = 0; ok && u_next >= 0; ++fi) {
                const int u = u_next;
                u_next = take();
                if (!publish(fi + 1, u_next)) break;
                if (u >= p.num_units) continue;
                const Unit t = decode_unit<ROWS, BK, LOCAL>(p, u);
                if (t.skip || t.n_kv == 0) continue;
                const int hk = t.h / p.group;
                for (int i = 0; i < NQ && ok; ++i) {
                    if (q_it > 0 && !mbar_wait(q_empty(i), (q_it - 1) & 1, w)) ok = false;
                    if (!ok) break;
                    mbar_arrive_expect_tx(q_full(i), C::Q_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c)
                        tma_load_3d(smem_u32(sQ + i * C::Q_BYTES + c * BM * 128), &tmQ, q_full(i), c * 64, t.h,
                                    t.q_start + t.q0 + i * BM);
                }
                if (!ok) break;
                ++q_it;
                for (int j = 0; j < t.n_kv && ok; ++j, ++kv_it) {
                    const int st = kv_it % KST;
                    const uint32_t n = kv_it / KST;
                    if (n > 0 && !mbar_wait(k_empty(st), (n - 1) & 1, w)) { ok = false; break; }
                    mbar_arrive_expect_tx(k_full(st), C::KV_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c)
                        tma_load_3d(smem_u32(sK + st * C::KV_BYTES + c * BK * 128), &tmK, k_full(st), c * 64, hk,
                                    t.k_start + (unit_kv0<LOCAL>(t) + j) * BK);
                    if (n > 0 && !mbar_wait(v_empty(st), (n - 1) & 1, w)) { ok = false; break; }
                    mbar_arrive_expect_tx(v_full(st), C::KV_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c)
                        tma_load_3d(smem_u32(sV + st * C::KV_BYTES + c * BK * 128), &tmV, v_full(st), c * 64, hk,
                                    t.k_start + (unit_kv0<LOCAL>(t) + j) * BK);
                }
                if (!ok) break;
            }
        }
        __syncwarp();
    } else if (warp == MMA) {
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BK, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, true);
            // each product's descriptors are formed once and advanced by constant byte offsets >> 4 in the
            // start-address field (shared-memory addresses stay below 2^18, so the 14-bit field never
            // carries): two adds per MMA, so the issuer keeps up with the tensor pipe
            auto issue_qk = [&](int i, int st) {
                const uint32_t qd = sdesc_lo(smem_u32(sQ + i * C::Q_BYTES), 16);
                const uint32_t kd = sdesc_lo(smem_u32(sK + st * C::KV_BYTES), 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss_lo(tmem + C::S_COL(i), qd + (((kk >> 2) * BM * 128 + (kk & 3) * 32) >> 4),
                               kd + (((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4), idesc_qk, kk > 0 ? 1u : 0u);
            };
            auto issue_pv = [&](int i, int st, bool acc) {
                const uint32_t vd = sdesc_lo(smem_u32(sV + st * C::KV_BYTES), BK * 128);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    umma_ts_lo(tmem + C::O_COL(i), tmem + C::S_COL(i) + kk * 8, vd + ((kk * 16 * 128) >> 4), idesc_pv,
                               (acc || kk > 0) ? 1u : 0u);
            };
            uint32_t kv_it = 0, q_it = 0, p_it[NQ] = {};
            bool ok = true;
            for (uint32_t fi = 0; ok; ++fi) {
                int u;
                if constexpr (DYN) {
                    if (!feed_get(feed, fi, u, w, false)) break;
                } else {
                    u = snake_unit(static_cast<int>(fi), p.num_units);
                }
                if (u < 0) break;
                if (u >= p.num_units) continue;
                const Unit t = decode_unit<ROWS, BK, LOCAL>(p, u);
                if (t.skip || t.n_kv == 0) continue;
                for (int i = 0; i < NQ && ok; ++i)
                    if (!mbar_wait(q_full(i), q_it & 1, w)) ok = false;
                if (!ok) break;
                ++q_it;
                {
                    const int st = kv_it % KST;
                    if (!mbar_wait(k_full(st), (kv_it / KST) & 1, w)) break;
                    tc_fence_after();
                    for (int i = 0; i < NQ; ++i) {
                        if (unit_lo<LOCAL>(t, i) != 0 || unit_hi(t, i) == 0) continue;   // tile i starts later (or never)
                        issue_qk(i, st);
                        umma_commit(s_full(i));
                    }
                    umma_commit(k_empty(st));
                    if (t.n_kv == 1)
                        for (int i = 0; i < NQ; ++i) umma_commit(q_empty(i));
                }
                // query tile i works on the unit's KV tiles lo[i] .. hi[i]-1
                for (int j = 0; j < t.n_kv && ok; ++j) {
                    const uint32_t cur = kv_it + j;
                    const int st = cur % KST;
                    const uint32_t nxt = cur + 1;
                    const int stn = nxt % KST;
                    if (!mbar_wait(v_full(st), (cur / KST) & 1, w)) { ok = false; break; }
                    tc_fence_after();
                    bool k_ready = false;
                    for (int i = 0; i < NQ; ++i) {
                        if (j >= unit_lo<LOCAL>(t, i) && j < unit_hi(t, i)) {
                            if (!mbar_wait(p_full(i), p_it[i] & 1, w)) { ok = false; break; }
                            ++p_it[i];
                            tc_fence_after();
                            issue_pv(i, st, j > unit_lo<LOCAL>(t, i));
                            umma_commit(o_full(i));
                        }
                        if (j + 1 >= unit_lo<LOCAL>(t, i) && j + 1 < unit_hi(t, i)) {
                            if (!k_ready) {
                                if (!mbar_wait(k_full(stn), (nxt / KST) & 1, w)) { ok = false; break; }
                                tc_fence_after();
                                k_ready = true;
                            }
                            issue_qk(i, stn);
                            umma_commit(s_full(i));
                        }
                    }
                    if (!ok) break;
                    // K(j+1) was waited for above whenever j+1 < n_kv: the two query tiles' ranges
                    // overlap or touch (the first key row of tile 1 is at most one past the last key
                    // row of tile 0, since the window sides are >= 0), so their union has no gap
                    // and some tile issues QK(j+1)
                    umma_commit(v_empty(st));
                    if (j + 1 < t.n_kv) {
                        umma_commit(k_empty(stn));
                        if (j + 2 == t.n_kv)
                            for (int i = 0; i < NQ; ++i) umma_commit(q_empty(i));
                    }
                }
                kv_it += t.n_kv;
            }
        }
        __syncwarp();
    }
    } else {
        if constexpr (NQ == 2) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::SOFTMAX_REGS));
        // ------------------------------------------------------------- softmax warpgroups
        const int i = warp >> 2;
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_base = tmem_lane_base(wq);
        const uint32_t tS = tmem + lane_base + C::S_COL(i);
        const uint32_t tO = tmem + lane_base + C::O_COL(i);
        const float c2 = p.scale_log2;
        uint32_t s_it = 0, pv_total = 0;
        bool ok = true;
        for (uint32_t fi = 0; ok; ++fi) {
            int u;
            if constexpr (DYN) {
                if (!feed_get(feed, fi, u, w, true)) break;
            } else {
                u = snake_unit(static_cast<int>(fi), p.num_units);
            }
            if (u < 0) break;
            if (u >= p.num_units) continue;
            const Unit t = decode_unit<ROWS, BK, LOCAL>(p, u);
            if (t.skip) continue;
            const int row = t.q0 + i * BM + r;
            const bool valid = row < t.Lq;
            __nv_bfloat16* orow = p.o + (static_cast<size_t>(t.q_start + row) * p.Hq + t.h) * D;
            float* lse_ptr = p.lse + t.b * p.lse_sB + t.h * p.lse_sH + static_cast<long long>(t.q_start) * p.lse_sT + row;
            const int lo_i = unit_lo<LOCAL>(t, i);
            const int n_mine = unit_hi(t, i) - lo_i;       // KV tiles this query tile sees
            if (n_mine == 0) {
                if (valid) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
                    *lse_ptr = -INFINITY;
                }
                continue;
            }
            // keys key_lo .. key_hi of the sequence are allowed for this row
            int key_lo = 0, key_hi = t.Lk - 1;
            if (LOCAL) key_lo = max(0, row + (t.Lk - t.Lq) - p.wl);
            if (p.wr >= 0) key_hi = min(key_hi, row + (t.Lk - t.Lq) + p.wr);
            float m_ref = -INFINITY;
            float l = 0.f;
            for (int j = 0; j < n_mine; ++j) {
                if (!mbar_wait(s_full(i), s_it & 1, w)) { ok = false; break; }
                ++s_it;
                tc_fence_after();
                float s[BK];
                {
                    // the whole row in one round trip: BK/32 loads, one wait
                    uint32_t* sr = reinterpret_cast<uint32_t*>(s);
#pragma unroll
                    for (int cc = 0; cc < BK / 32; ++cc)
                        tmem_ld32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + cc * 32));
                    tmem_ld_wait_tie(*reinterpret_cast<uint32_t(*)[32]>(sr));
#pragma unroll
                    for (int cc = 1; cc < BK / 32; ++cc) reg_tie(*reinterpret_cast<uint32_t(*)[32]>(sr + cc * 32));
                }
                const int kbase = (unit_kv0<LOCAL>(t) + lo_i + j) * BK;
                const bool masked = __any_sync(0xffffffffu, kbase + BK - 1 > key_hi || (LOCAL && kbase < key_lo));
                if (masked) {
#pragma unroll
                    for (int c = 0; c < BK; ++c)
                        s[c] = (kbase + c <= key_hi && (!LOCAL || kbase + c >= key_lo)) ? s[c] : -INFINITY;
                }
                float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
                for (int c = 4; c < BK; c += 2) mx[(c >> 1) & 3] = max3f(mx[(c >> 1) & 3], s[c], s[c + 1]);
                const float mt = max3f(mx[0], mx[1], fmaxf(mx[2], mx[3]));
                const bool need = (mt - m_ref) * c2 > kDeferLog2;   // NaN (both -inf) -> false
                if (__any_sync(0xffffffffu, need)) {
                    const float m_new = fmaxf(m_ref, mt);
                    const float alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx((m_ref - m_new) * c2);
                    const bool rescale = (j > 0) && __any_sync(0xffffffffu, m_ref != -INFINITY && alpha < 1.f);
                    if (rescale) {
                        if (!mbar_wait(o_full(i), (pv_total + j - 1) & 1, w)) { ok = false; }
                        // all lanes reach here together; the abort case skips the work
                        if (__all_sync(0xffffffffu, ok)) {
                            tc_fence_after();
                            uint32_t ro[32];
                            const float2 a2 = make_float2(alpha, alpha);
#pragma unroll 1
                            for (int cc = 0; cc < D / 32; ++cc) {
                                tmem_ld32(tO + cc * 32, ro);
                                tmem_ld_wait_tie(ro);
#pragma unroll
                                for (int e = 0; e < 32; e += 2) {
                                    const float2 v = fmul2(make_float2(__uint_as_float(ro[e]), __uint_as_float(ro[e + 1])), a2);
                                    ro[e] = __float_as_uint(v.x);
                                    ro[e + 1] = __float_as_uint(v.y);
                                }
                                tmem_st32(tO + cc * 32, ro);
                            }
                            tmem_st_wait();
                        } else {
                            ok = false;
                            break;
                        }
                    }
                    l *= alpha;
                    m_ref = m_new;
                }
                const float ms = (m_ref == -INFINITY) ? 0.f : m_ref * c2;
                const float2 c2v = make_float2(c2, c2), nms = make_float2(-ms, -ms);
                float2 sum0 = make_float2(0.f, 0.f), sum1 = make_float2(0.f, 0.f);
                // exp(scale * s - scale * m) as exp2 of one fused multiply-add per pair; on tiles
                // without masked scores one pair in fma_exp_every(D) may go to the FMA pipe
                auto exp_row = [&](auto poly) {
                    constexpr int kEvery = decltype(poly)::value ? fma_exp_every(D) : 0;
                    constexpr int kMod = kEvery > 0 ? kEvery : 1;
#pragma unroll
                    for (int half = 0; half < BK / 64; ++half) {
                        uint32_t pk[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const float2 x = ffma2(make_float2(s[half * 64 + 2 * e], s[half * 64 + 2 * e + 1]), c2v, nms);
                            const float2 p2 = (kEvery > 0 && e % kMod == kMod - 1)
                                                  ? exp2_fma2(x)
                                                  : make_float2(ex2_approx(x.x), ex2_approx(x.y));
                            if (e & 1) sum1 = fadd2(sum1, p2); else sum0 = fadd2(sum0, p2);
                            pk[e] = pack_bf16x2(p2.x, p2.y);
                        }
                        tmem_st32(tS + half * 32, pk);
                    }
                };
                if (fma_exp_every(D) > 0 && !masked) exp_row(std::true_type{});
                else exp_row(std::false_type{});
                {
                    const float2 sm = fadd2(sum0, sum1);
                    l += sm.x + sm.y;
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(p_full(i));
            }
            if (!ok) break;
            pv_total += n_mine;
            // ------------------------------------------------ epilogue: O / l, LSE
            if (!mbar_wait(o_full(i), (pv_total - 1) & 1, w)) { ok = false; break; }
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            uint32_t ro[32];
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                tmem_ld32(tO + cc * 32, ro);
                tmem_ld_wait_tie(ro);
                uint32_t pk[16];
                const float2 il = make_float2(inv_l, inv_l);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 v = fmul2(make_float2(__uint_as_float(ro[2 * e]), __uint_as_float(ro[2 * e + 1])), il);
                    pk[e] = pack_bf16x2(v.x, v.y);
                }
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
            if (valid) *lse_ptr = l > 0.f ? (m_ref * c2 + log2f(l)) * kLn2 : -INFINITY;
            tc_fence_before();
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

// Groups (sequence, query head) per chunk of the unit list: every group of a chunk keeps its K and V
// (shared by the group of query heads reading one KV head) in L2 while the chunk's query blocks run;
// chunks of about 96 MB of K and V, and at least twice as many units as CTAs.
static int fwd_chunk_groups(const Problem& pr, int D, int m_blocks, int num_sms) {
    const int groups = pr.num_seqs * pr.Hq;
    const double kv_per_group = 4.0 * pr.Sk * D / (pr.Hq / pr.Hkv);
    long long c = static_cast<long long>(96.0 * (1 << 20) / (kv_per_group > 1.0 ? kv_per_group : 1.0));
    const long long by_balance = (2LL * num_sms + m_blocks - 1) / m_blocks;
    if (c < by_balance) c = by_balance;
    if (c < 1) c = 1;
    if (c > groups) c = groups;
    const long long n_chunks = (groups + c - 1) / c;
    return static_cast<int>((groups + n_chunks - 1) / n_chunks);
}

template <int D, int NQ, int BK, int KST, bool LOCAL, bool DYN>
static int run_fwd(const Problem& pr, void* out, float* lse, int* counter, const Device& dev, cudaStream_t stream) {
    using C = FwdCfg<D, NQ, BK, KST>;
    alignas(64) CUtensorMap mq, mk, mv;
    const uint64_t rq = static_cast<uint64_t>(pr.Hq) * D * 2, rk = static_cast<uint64_t>(pr.Hkv) * D * 2;
    if (!make_map_3d_bf16(&mq, pr.q, D, pr.Hq, pr.Tq, D * 2, rq, 64, 1, C::BM)) return 5;
    if (!make_map_3d_bf16(&mk, pr.k, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, BK)) return 5;
    if (!make_map_3d_bf16(&mv, pr.v, D, pr.Hkv, pr.Tk, D * 2, rk, 64, 1, BK)) return 5;

    FwdParams p;
    p.o = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
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
    p.m_blocks = (pr.Sq + C::BM * NQ - 1) / (C::BM * NQ);
    const long long units = static_cast<long long>(p.m_blocks) * pr.num_seqs * pr.Hq;
    if (units > 0x7fffffffLL) return 2;
    p.num_units = static_cast<int>(units);
    p.scale_log2 = pr.scale * 1.4426950408889634f;
    p.wl = pr.wl;
    p.wr = pr.wr;
    p.lse_sB = pr.lse_sB;
    p.lse_sH = pr.lse_sH;
    p.lse_sT = pr.lse_sT;
    // DYN (a counter from the caller's workspace): head-chunked order taken dynamically; otherwise the
    // static heaviest-first deal over all groups
    p.counter = DYN ? counter : nullptr;
    p.chunk = DYN ? fwd_chunk_groups(pr, D, p.m_blocks, dev.num_sms) : pr.num_seqs * pr.Hq;
    p.timeout_ns = dev.timeout_ns;
    p.status = dev.status;
    if (p.num_units == 0) return 0;
    if (DYN && cudaMemsetAsync(counter, 0, sizeof(int), stream) != cudaSuccess) return 5;

    auto kern = fwd_kernel<D, NQ, BK, KST, LOCAL, DYN>;
    static bool attr_set[64] = {};
    if (!attr_set[dev.id & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM)) !=
            cudaSuccess)
            return 5;
        if (NQ == 2) {
            // the setmaxnreg split assumes exactly LAUNCH_REGS per thread at launch; with fewer the
            // increase could never be granted, so refuse to launch instead
            cudaFuncAttributes fa_attr;
            if (cudaFuncGetAttributes(&fa_attr, kern) != cudaSuccess || fa_attr.numRegs != C::LAUNCH_REGS) return 2;
        }
        attr_set[dev.id & 63] = true;
    }
    const int grid = p.num_units < dev.num_sms ? p.num_units : dev.num_sms;
    prof_before(0, stream);
    kern<<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, p);
    prof_after(0, stream);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 5;
}

template <int D, int NQ, int BK, int KST>
static int run_fwd_d(const Problem& pr, void* out, float* lse, int* counter, const Device& dev,
                     cudaStream_t stream) {
    // the dynamic schedule where it pays: varlen batches (unequal lengths unbalance the static deal) and
    // problems whose K and V do not fit L2 together (head chunks); it needs the caller's workspace
    const int m_blocks = (pr.Sq + 128 * NQ - 1) / (128 * NQ);
    const bool dyn = counter != nullptr &&
                     (pr.cu_q != nullptr || fwd_chunk_groups(pr, D, m_blocks, dev.num_sms) < pr.num_seqs * pr.Hq);
    const bool local = pr.wl >= 0;
    if (dyn) return local ? run_fwd<D, NQ, BK, KST, true, true>(pr, out, lse, counter, dev, stream)
                          : run_fwd<D, NQ, BK, KST, false, true>(pr, out, lse, counter, dev, stream);
    return local ? run_fwd<D, NQ, BK, KST, true, false>(pr, out, lse, nullptr, dev, stream)
                 : run_fwd<D, NQ, BK, KST, false, false>(pr, out, lse, nullptr, dev, stream);
}

int launch_fwd(const Problem& pr, void* out, float* lse, int* counter, const Device& dev, cudaStream_t stream) {
    switch (pr.D) {
        case 64: return run_fwd_d<64, 2, 128, 4>(pr, out, lse, counter, dev, stream);
        case 128: return run_fwd_d<128, 2, 128, 2>(pr, out, lse, counter, dev, stream);
        case 256: return run_fwd_d<256, 1, 128, 1>(pr, out, lse, counter, dev, stream);
        default: return 2;
    }
}

}  // namespace fa

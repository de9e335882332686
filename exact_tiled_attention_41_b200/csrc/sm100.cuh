// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// attention kernels use: mbarriers with bounded waits, TMA tile loads, tensor
// memory (TMEM) allocation / load / store, and tcgen05 MMAs with shared-memory
// matrix descriptors.  Written from the PTX ISA; nothing here is attention math.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Status codes mirrored from include/fa.h (device side cannot include it twice harmlessly).
constexpr int kStatusTimeout = 6;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ bounded waits
// Every wait in the kernels polls with a time limit.  When it runs out the
// thread records the timeout in the device status word, raises the CTA-wide
// abort flag in shared memory, and returns false; every other wait of the CTA
// then returns false too, so all roles leave their loops and the CTA exits
// cleanly (tensor memory is still freed).
struct Watch {
    volatile int* abort_flag;   // shared memory
    int* status;                // global status word
    unsigned long long limit_ns;

    __device__ __forceinline__ void fail() const {
        atomicCAS(status, 0, kStatusTimeout);
        *abort_flag = 1;
    }
    __device__ __forceinline__ bool aborted() const { return *abort_flag != 0; }
};

__device__ __forceinline__ void mbar_init(void* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the completion of the phase with the given parity.  false = gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Watch& w) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (w.aborted()) return false;
            if (global_timer_ns() - t0 > w.limit_ns) {
                w.fail();
                return false;
            }
        }
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load into shared memory; completion is signalled as tx bytes on `bar`.
// The innermost coordinate c0 must be a multiple of 8 elements (16 bytes of bf16).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// 3-D tiled store of a shared-memory box into global memory, in the issuing thread's bulk async-group;
// parts of the box outside the tensor are not written.  c0 must be a multiple of 8 bf16 elements and
// no coordinate may be negative.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the issuing thread's bulk stores have finished reading shared memory / have completed
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Make generic-proxy writes to shared memory visible to the async proxy (tensor cores, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tensor memory
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Lane field of a tensor-memory address: bits [31:16]; column: bits [15:0].
__device__ __forceinline__ uint32_t tmem_lane_base(int warp_in_group) {
    return static_cast<uint32_t>(warp_in_group * 32) << 16;
}

#define FA_R4(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3])
#define FA_R16(i) FA_R4(i), FA_R4(i + 4), FA_R4(i + 8), FA_R4(i + 12)

// 32 lanes x 32 columns of 32-bit words: thread t of the warp receives lane
// (base lane + t), columns c .. c+31 in r[0..31].
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : FA_R16(0), FA_R16(16)
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : FA_R16(0)
        : "r"(taddr));
}
#undef FA_R16
#undef FA_R4

// Wait for outstanding tcgen05.ld and tie the destination registers to the wait,
// so the compiler cannot move a use of them above it.
#define FA_T4(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3])
#define FA_T16(i) FA_T4(i), FA_T4(i + 4), FA_T4(i + 8), FA_T4(i + 12)
__device__ __forceinline__ void tmem_ld_wait_tie(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : FA_T16(0), FA_T16(16)::"memory");
}
__device__ __forceinline__ void tmem_ld_wait_tie16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : FA_T16(0)::"memory");
}
// Tie further registers loaded before an earlier wait (no instruction emitted).
__device__ __forceinline__ void reg_tie(uint32_t (&r)[32]) { asm volatile("" : FA_T16(0), FA_T16(16)); }
#undef FA_T16
#undef FA_T4

#define FA_S4(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3])
#define FA_S16(i) FA_S4(i), FA_S4(i + 4), FA_S4(i + 8), FA_S4(i + 12)
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        FA_S16(0), FA_S16(16)
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        FA_S16(0)
        : "memory");
}
#undef FA_S16
#undef FA_S4

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ tcgen05 MMA
// Instruction descriptor for kind::f16 with bf16 inputs and an f32 accumulator
// (field positions per the PTX ISA instruction-descriptor table):
//   [4,6) D format (1 = f32)  [7,10) A format (1 = bf16)  [10,13) B format (1 = bf16)
//   [15] A major (0 = K, 1 = MN)  [16] B major  [17,23) N >> 3  [24,29) M >> 4
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100 version 1.
//   start address >> 4 in [0,14); leading byte offset >> 4 in [16,30);
//   stride byte offset >> 4 in [32,46); version 1 at bit 46; layout type at [61,64).
// K-major operands: SBO = byte distance between groups of 8 rows (1024 for a
//   dense 128-byte-row tile); LBO unused (set to 16).
// MN-major operands: LBO = byte distance between 64-element column blocks,
//   SBO = byte distance between groups of 8 rows along K (1024).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same descriptors split into two 32-bit words, for issue loops that advance a descriptor by a
// constant byte offset with one 32-bit add: every descriptor here shares the high word (SBO 1024,
// version 1, 128-byte swizzle); the low word holds start address >> 4 and LBO >> 4.  Shared-memory
// addresses stay below 2^18, so adding offset >> 4 never carries out of the 14-bit address field.
constexpr uint32_t kSDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo) {
    return ((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}

// D[tmem] (+)= A[smem] * B[smem], descriptors given by their low words
__device__ __forceinline__ void umma_ss_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "mov.b64 da, {%1, %5};\n\tmov.b64 db, {%2, %5};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(kSDescHi)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], B's descriptor given by its low word
__device__ __forceinline__ void umma_ts_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "mov.b64 db, {%2, %5};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(kSDescHi)
        : "memory");
}

// Programmatic dependent launch: a kernel launched with the programmatic-serialization attribute may start
// before the previous kernel on its stream has finished; grid_dep_wait() blocks until that kernel has
// completed and its memory writes are visible (it returns at once for an ordinary launch), and
// grid_dep_launch() lets the next such kernel start once every CTA of this grid has called it or exited.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// ------------------------------------------------------------------ math helpers
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Three-input max (PTX max.f32 with three sources, sm_100+).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Packed two-lane fp32 arithmetic (PTX fma/add/mul .f32x2, round to nearest even).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    uint64_t d, x, y, z;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(z) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(x), "l"(y), "l"(z));
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
    return r;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    uint64_t d, x, y;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x), "l"(y));
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
    return r;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    uint64_t d, x, y;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x), "l"(y));
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
    return r;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
    uint64_t d, x, y;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x), "l"(y));
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
    return r;
}

// Two exp2 on the FMA pipe, for the share of the softmax exponentials taken off the
// multi-function unit.  x is clamped to >= -126, then split as x = j + f with j = rint(x)
// (adding 1.5 * 2^23 leaves rint(x) in the low mantissa bits of t) and f in [-1/2, 1/2];
// 2^f is the degree-5 polynomial whose coefficients minimise the maximum relative error on
// [-1/2, 1/2] (Remez exchange; exact_tiled_attention_41_b200/fit_exp2_poly.py prints them), and
// 2^j is applied by adding j to the exponent field (t << 23 keeps only j's bits there).  Worst
// relative error 2.3e-7 over [-125, 8] (about 2 ulp, the class of the hardware ex2.approx).
// Below -125 the result is a non-negative value under 2^-125 rather than exactly 0, so the
// softmax calls this only on tiles without masked (-inf) scores; x <= 127.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
    const float2 xc = make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f));
    const float2 t = fadd2(xc, make_float2(kRound, kRound));
    const float2 f = fsub2(xc, fsub2(t, make_float2(kRound, kRound)));   // x - rint(x)
    float2 p = ffma2(make_float2(1.3276472e-3f, 1.3276472e-3f), f, make_float2(9.675541e-3f, 9.675541e-3f));
    p = ffma2(p, f, make_float2(5.550713e-2f, 5.550713e-2f));
    p = ffma2(p, f, make_float2(2.402212e-1f, 2.402212e-1f));
    p = ffma2(p, f, make_float2(6.9314694e-1f, 6.9314694e-1f));
    p = ffma2(p, f, make_float2(1.0000001f, 1.0000001f));
    const uint32_t bx = __float_as_uint(p.x) + (__float_as_uint(t.x) << 23);
    const uint32_t by = __float_as_uint(p.y) + (__float_as_uint(t.y) << 23);
    return make_float2(__uint_as_float(bx), __uint_as_float(by));
}

// ------------------------------------------------------------------ L2 eviction priority
// Cache policies for the .L2::cache_hint forms of loads, stores and reductions: lines brought in or
// written with evict_last are replaced after the others, evict_first before them, evict_normal as
// without a hint.  The hint changes no value, only which lines L2 keeps.
__device__ __forceinline__ uint64_t l2_policy_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_normal() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void red_add_f32x4_hint(float4* addr, float4 v, uint64_t pol) {
    asm volatile("red.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(addr), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_f32x4_hint(float4* addr, float4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(addr), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ uint4 ld_u32x4_hint(const void* addr, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(addr), "l"(pol));
    return v;
}
// Drop one 128-byte L2 line without writing it back: its contents become undefined.  addr must be
// 128-byte aligned, and no other thread may still read the line.
__device__ __forceinline__ void l2_discard_line(const void* addr) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(addr) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Row stores through shared memory: each lane puts the four 16-byte pieces of 64 bytes of its own row
// into 2 KB of shared memory (stg, this warp's alone, 16-byte aligned; stg_put), then stg_flush writes
// them so that each store instruction covers 8 rows x 64 contiguous bytes rather than 32 rows x 16
// bytes: four times fewer cache lines per instruction.  Piece q of row r sits at 16-byte slot
// 32 q + (r ^ q), so the row-wise writes and the piece-wise reads of every 8 lanes touch 8 different banks.
__device__ __forceinline__ void stg_put(uint8_t* stg, int q, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
    const int lane = threadIdx.x & 31;
    *reinterpret_cast<uint4*>(stg + ((q * 32 + (lane ^ q)) << 4)) = make_uint4(w0, w1, w2, w3);
}

// dst: this lane's destination of the 64 bytes (16-byte aligned); rows are row_stride bytes apart;
// only the rows of lanes 0 .. nvalid-1 are written.  The warp may refill stg after this returns.
__device__ __forceinline__ void stg_flush(const uint8_t* stg, uint8_t* dst, long long row_stride, int nvalid) {
    const int lane = threadIdx.x & 31;
    __syncwarp();
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int rr = 4 * g + j;   // lanes 4g .. 4g+3 write row rr, 16 bytes each
        const uint4 v = *reinterpret_cast<const uint4*>(stg + ((c * 32 + (rr ^ c)) << 4));
        if (rr < nvalid) *reinterpret_cast<uint4*>(dst + (rr - lane) * row_stride + c * 16) = v;
    }
    __syncwarp();
}

__device__ __forceinline__ int elect_lane0() { return (threadIdx.x & 31) == 0; }

// Dynamic persistent schedule: one thread of the producer warp takes unit indices from a global
// counter (zeroed before the launch, on the same stream) and hands them to the CTA's other roles
// through kFeedSlots shared-memory slots.  Slot s has a full barrier (one arrival: the producer,
// whose arrive releases the slot write) and an empty barrier (one arrival per consuming warp).
// When the list is exhausted the producer publishes -1, and every role stops there.
constexpr int kFeedSlots = 4;

struct UnitFeed {
    int* slot;         // [kFeedSlots] in shared memory
    uint32_t full0;    // full barrier of slot s: full0 + 8 s
    uint32_t empty0;   // empty barrier of slot s: empty0 + 8 s
};

// Producer thread: publish this CTA's it-th unit (or -1); false = gave up waiting for the slot.
__device__ __forceinline__ bool feed_put(const UnitFeed& f, uint32_t it, int* counter, int num_units, int& u,
                                         const Watch& w) {
    const uint32_t s = it % kFeedSlots;
    if (it >= kFeedSlots && !mbar_wait(f.empty0 + 8 * s, ((it / kFeedSlots) - 1) & 1, w)) return false;
    const int v = atomicAdd(counter, 1);
    u = v < num_units ? v : -1;
    f.slot[s] = u;
    mbar_arrive(f.full0 + 8 * s);
    return true;
}

// Consumer: the it-th unit (every calling thread waits; lane 0 of each warp releases the slot, so the
// whole warp must call it together, or only lane 0 when the warp's other lanes never consume).
__device__ __forceinline__ bool feed_get(const UnitFeed& f, uint32_t it, int& u, const Watch& w, bool whole_warp) {
    const uint32_t s = it % kFeedSlots;
    if (!mbar_wait(f.full0 + 8 * s, (it / kFeedSlots) & 1, w)) return false;
    u = f.slot[s];
    if (whole_warp) __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(f.empty0 + 8 * s);
    return true;
}

// Persistent schedule over work units sorted heaviest first: round k of CTA c takes unit
// k*G + c on even rounds and k*G + (G-1-c) on odd rounds (a boustrophedon), so the CTA that
// got the heaviest unit of one round gets the lightest of the next.  Returns -1 past the end
// of the list (stop) and num_units (skip) when this round's slot is empty.
__device__ __forceinline__ int snake_unit(int k, int num_units) {
    const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    const long long base = static_cast<long long>(k) * G;
    if (base >= num_units) return -1;
    const long long u = base + ((k & 1) ? (G - 1 - c) : c);
    return u < num_units ? static_cast<int>(u) : num_units;
}

}  // namespace fa

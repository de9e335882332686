// selftest.cu -- two diagnostic kernels exported through the C ABI:
//   * a wait that nobody ever completes, to show that every bounded wait ends
//     with FA_ERR_TIMEOUT in the status word instead of hanging the GPU;
//   * one 128x128x128 tcgen05 product in the three operand arrangements the
//     attention kernels use (K-major x K-major, K-major x N-major, tensor-memory
//     A x N-major), to check descriptor and tensor-memory conventions on their own.
#include "internal.h"
#include "sm100.cuh"

namespace fa {

__global__ void wait_selftest_kernel(unsigned long long limit_ns, int* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const Watch w{&abort_flag, status, limit_ns};
    // nobody arrives: this wait must run out and record the timeout
    (void)mbar_wait(smem_u32(&bar), 0, w);
}

// y = 2^x through the FMA-pipe exponential used by the softmax kernels (pairs of elements).
__global__ void exp2_selftest_kernel(const float* x, float* y, int n2) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += gridDim.x * blockDim.x) {
        const float2 r = exp2_fma2(make_float2(x[2 * i], x[2 * i + 1]));
        y[2 * i] = r.x;
        y[2 * i + 1] = r.y;
    }
}

int launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t stream) {
    if (n <= 0 || (n & 1)) return 1;
    const int n2 = n / 2;
    exp2_selftest_kernel<<<(n2 + 255) / 256 < 1024 ? (n2 + 255) / 256 : 1024, 256, 0, stream>>>(x, y, n2);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 5;
}

int launch_wait_selftest(unsigned long long timeout_ns, const Device& dev, cudaStream_t stream) {
    if (timeout_ns == 0 || timeout_ns > 10000000000ull) return 1;
    wait_selftest_kernel<<<1, 32, 0, stream>>>(timeout_ns, dev.status);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 5;
}

// One CTA, 128 threads.  a, b: bf16 [128][128] row-major (16 KB boxes of 64 columns).
__global__ void __launch_bounds__(128, 1) umma_selftest_kernel(const __grid_constant__ CUtensorMap ma,
                                                               const __grid_constant__ CUtensorMap mb,
                                                               const __nv_bfloat16* a, float* c, int mode,
                                                               int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;             // 2 boxes x 16 KB
    uint8_t* sB = smem + 32768;     // 2 boxes x 16 KB
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 65536);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bars + 0, 1);
        mbar_init(bars + 1, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Watch wl{&abort_flag, status, 1000000000ull};

    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(smem_u32(bars), 65536);
        for (int cc = 0; cc < 2; ++cc) {
            tma_load_2d(smem_u32(sA + cc * 16384), &ma, smem_u32(bars), cc * 64, 0);
            tma_load_2d(smem_u32(sB + cc * 16384), &mb, smem_u32(bars), cc * 64, 0);
        }
    }
    const bool ok = mbar_wait(smem_u32(bars), 0, wl);
    const uint32_t lane_base = tmem_lane_base(warp);
    if (mode == 2) {
        // thread = row of A; pack bf16 pairs (element 2c in the low half) into 64 columns
        const __nv_bfloat16* arow = a + threadIdx.x * 128;
        uint32_t pk[32];
        for (int half = 0; half < 2; ++half) {
            for (int e = 0; e < 32; ++e) {
                __nv_bfloat162 v;
                v.x = arow[half * 64 + 2 * e];
                v.y = arow[half * 64 + 2 * e + 1];
                pk[e] = *reinterpret_cast<uint32_t*>(&v);
            }
            tmem_st32(tmem + lane_base + 256 + half * 32, pk);
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0 && ok) {
        const uint32_t idesc = idesc_bf16_f32(128, 128, false, mode != 0);
        for (int kk = 0; kk < 8; ++kk) {
            if (mode == 0) {
                const uint32_t aa = smem_u32(sA + (kk >> 2) * 16384 + (kk & 3) * 32);
                const uint32_t bb = smem_u32(sB + (kk >> 2) * 16384 + (kk & 3) * 32);
                umma_ss(tmem, sdesc_sw128(aa, 16, 1024), sdesc_sw128(bb, 16, 1024), idesc, kk > 0);
            } else if (mode == 1) {
                const uint32_t aa = smem_u32(sA + (kk >> 2) * 16384 + (kk & 3) * 32);
                const uint32_t bb = smem_u32(sB + kk * 16 * 128);
                umma_ss(tmem, sdesc_sw128(aa, 16, 1024), sdesc_sw128(bb, 16384, 1024), idesc, kk > 0);
            } else {
                const uint32_t bb = smem_u32(sB + kk * 16 * 128);
                umma_ts(tmem, tmem + 256 + kk * 8, sdesc_sw128(bb, 16384, 1024), idesc, kk > 0);
            }
        }
        umma_commit(smem_u32(bars + 1));
    }
    __syncwarp();
    const bool done = ok && mbar_wait(smem_u32(bars + 1), 0, wl);
    tc_fence_after();
    if (__all_sync(0xffffffffu, done)) {
        uint32_t r[32];
        for (int cc = 0; cc < 4; ++cc) {
            tmem_ld32(tmem + lane_base + cc * 32, r);
            tmem_ld_wait_tie(r);
            for (int e = 0; e < 32; ++e) c[threadIdx.x * 128 + cc * 32 + e] = __uint_as_float(r[e]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    (void)lane;
}

int launch_umma_selftest(const void* a, const void* b, float* c, int mode, const Device& dev, cudaStream_t stream) {
    alignas(64) CUtensorMap ma, mb;
    if (!make_map_2d_bf16(&ma, a, 128, 128, 256, 64, 128)) return 5;
    if (!make_map_2d_bf16(&mb, b, 128, 128, 256, 64, 128)) return 5;
    const int smem = 1024 + 65536 + 64;
    static bool set = false;
    if (!set) {
        if (cudaFuncSetAttribute(umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return 5;
        set = true;
    }
    umma_selftest_kernel<<<1, 128, smem, stream>>>(ma, mb, static_cast<const __nv_bfloat16*>(a), c, mode, dev.status);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : 5;
}

}  // namespace fa

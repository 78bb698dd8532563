// Measurement utilities of the benchmark (not part of the library's ABI).
//
// dsa_probe_l2_read: the read bandwidth of L2 for a buffer that stays
// resident in it, the bound of kernels whose gathered rows hit L2 (the sparse
// attention).  Every thread streams 16-byte loads that bypass L1
// (ld.global.cg) over the buffer, `passes` times, and folds them into one
// word so that no load is dead.
//
// dsa_probe_fp8_mma: the rate of the 5th-generation tensor cores on the
// indexer's own product shape (tcgen05.mma kind::f8f6f4, e4m3 x e4m3 -> f32,
// M = 128, N = 256, K = 32 per instruction; A and B K-major with the 128-byte
// swizzle), with operands resident in shared memory and nothing else to do:
// one CTA per SM, one thread issuing `iters` x 4 instructions (K = 128) into
// two TMEM accumulators.  FLOP = 2 * 128 * 256 * 128 * iters per CTA.
//
// dsa_probe_wait_timeout: a test hook for the bounded waits every kernel
// uses (ptx.cuh): one thread waits on an mbarrier that nothing arrives at;
// after the limit (2 s) the wait gives up, records DSA_DEVERR_TIMEOUT in the
// given error word and the kernel returns, leaving the context usable.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace {

__global__ void __launch_bounds__(512) l2_read_kernel(const uint4* buf, size_t n16, int passes,
                                                      uint32_t* sink) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    uint32_t acc = 0;
    for (int p = 0; p < passes; ++p) {
        // each pass starts at a rotated offset so that no CTA keeps one slice
        const size_t rot = ((size_t)p * 7919u * blockDim.x) % n16;
        for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) {
            size_t j = i + rot;
            if (j >= n16) j -= n16;
            uint4 v;
            asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "l"(buf + j));
            acc ^= v.x ^ v.y ^ v.z ^ v.w;
        }
    }
    if (acc == 0x9e3779b9u) sink[0] = acc;  // practically never: keeps the loads live
}

constexpr int kProbeM = 128, kProbeN = 256, kProbeK = 128;  // bytes per row = K (e4m3)
constexpr int kProbeA = 0;                                   // A: 128 rows x 128 B
constexpr int kProbeB = kProbeM * kProbeK;                   // B: 256 rows x 128 B
constexpr int kProbeBar = kProbeB + kProbeN * kProbeK;
// more than half of an SM's shared memory, so that one CTA (which takes all
// of TMEM) runs per SM
constexpr int kProbeSmem = 120 * 1024;

__global__ void __launch_bounds__(128, 1) fp8_mma_kernel(int iters, uint32_t* sink, int* err) {
    extern __shared__ __align__(1024) uint8_t probe_smem[];
    const uint32_t sb = dsa::smem_u32(probe_smem);
    uint64_t* bar = reinterpret_cast<uint64_t*>(probe_smem + kProbeBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(probe_smem + kProbeBar + 8);
    const int warp = threadIdx.x >> 5;
    if ((sb & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
        if (threadIdx.x == 0) dsa::record_error_to(err, 1);
        return;
    }
    // operands: e4m3 values +-1, +-2 (bytes 0x38, 0xB8, 0x40, 0xC0) in a
    // position-dependent pattern
    for (int i = threadIdx.x; i < kProbeBar / 4; i += blockDim.x) {
        const uint32_t h = (uint32_t)i * 2654435761u;
        const uint32_t b0 = (h >> 7) & 1u ? 0xB8u : 0x38u, b1 = (h >> 11) & 1u ? 0xC0u : 0x40u;
        reinterpret_cast<uint32_t*>(probe_smem)[i] = b0 | (b1 << 8) | (b1 << 16) | (b0 << 24);
    }
    if (threadIdx.x == 0) {
        dsa::mbar_init(dsa::smem_u32(bar), 1);
        dsa::fence_mbar_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 0) {
        dsa::tmem_alloc(dsa::smem_u32(tmem_slot), 512);
        dsa::tmem_relinquish();
    }
    dsa::tc_fence_before();
    __syncthreads();
    dsa::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) {
        constexpr uint32_t idesc = dsa::idesc_e4m3_f32(kProbeN);
        const uint64_t adesc = dsa::smem_desc_kmajor(sb + kProbeA, kProbeK);
        const uint64_t bdesc = dsa::smem_desc_kmajor(sb + kProbeB, kProbeK);
        for (int i = 0; i < iters; ++i) {
            const uint32_t d = tmem + (uint32_t)((i & 1) * kProbeN);
#pragma unroll
            for (int kk = 0; kk < kProbeK / 32; ++kk)
                dsa::umma_f8f6f4(d, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk), idesc,
                                 (i >= 2 || kk > 0) ? 1u : 0u);
        }
        dsa::umma_commit(dsa::smem_u32(bar));
        dsa::mbar_wait_to(err, dsa::smem_u32(bar), 0);
    }
    dsa::tc_fence_before();
    __syncthreads();
    dsa::tc_fence_after();
    if (warp == 0) {
        float v[4];
        dsa::tmem_ld_32x32b_x4(tmem, v);  // one accumulator value per lane: the products are live
        if (v[0] == 1.2345678e30f) sink[0] = 1u;
        dsa::tmem_dealloc(tmem, 512);
    }
}

__global__ void wait_timeout_kernel(int* err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        dsa::mbar_init(dsa::smem_u32(&bar), 1);
        dsa::fence_mbar_init();
        dsa::mbar_wait_to(err, dsa::smem_u32(&bar), 0);  // no arrival ever comes
    }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int dsa_probe_wait_timeout(void* err,
                                                                             void* stream) {
    if (err == nullptr || (reinterpret_cast<uintptr_t>(err) & 3u) != 0) return 1;
    wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int*>(err));
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" __attribute__((visibility("default"))) int dsa_probe_l2_read(const void* buf,
                                                                        size_t bytes, int passes,
                                                                        int ctas, void* sink,
                                                                        void* stream) {
    if (buf == nullptr || sink == nullptr || bytes < 16 || passes < 1 || ctas < 1) return 1;
    if ((reinterpret_cast<uintptr_t>(buf) & 15u) != 0) return 1;
    l2_read_kernel<<<ctas, 512, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(buf), bytes / 16, passes, static_cast<uint32_t*>(sink));
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

// One CTA per SM, `iters` groups of four MMAs each; err: a device int for
// the bounded wait (DSA_DEVERR_TIMEOUT = 1).  Returns 0, 1 (bad argument) or
// 2 (launch error).
extern "C" __attribute__((visibility("default"))) int dsa_probe_fp8_mma(int iters, void* sink,
                                                                        void* err, void* stream) {
    if (iters < 1 || sink == nullptr || err == nullptr) return 1;
    if ((reinterpret_cast<uintptr_t>(err) & 3u) != 0) return 1;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 2;
    if (cudaFuncSetAttribute(fp8_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kProbeSmem) != cudaSuccess)
        return 2;
    fp8_mma_kernel<<<sms, 128, kProbeSmem, static_cast<cudaStream_t>(stream)>>>(
        iters, static_cast<uint32_t*>(sink), static_cast<int*>(err));
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

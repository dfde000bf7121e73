// peak.cu -- libcsa2_peak.so: the tensor-core rate of this library's own
// instruction forms, for the roofline denominators of the measurement
// (not part of the decode path). One CTA per SM issues a chain of
// tcgen05.mma instructions of one shape (operands in shared memory,
// accumulators in TMEM, four accumulators used in turn) and the host times
// the whole grid with CUDA events.
//   peak_tcgen05(kind, n, iters, stream): kind 0 = kind::f16 (f16 x f16 ->
//   f32, K = 16 per instruction), kind 1 = kind::f8f6f4 (E4M3 x E4M3 -> f32,
//   K = 32); M = 128; n in {64, 128, 256}. Returns the device time in
//   milliseconds (negative on error); FLOPs = 2 * 128 * n * K * iters * SMs.
#include "common.cuh"

using namespace csa2;

namespace {

template <int KIND, int N>
__global__ void __launch_bounds__(128, 1) k_peak(int iters) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *a = base;          // 128 rows x 128 B
    uint8_t *b = base + 16384;  // N rows x 128 B
    __shared__ uint64_t bar;
    __shared__ uint32_t slot;
    for (int i = threadIdx.x; i < (128 + N) * 8; i += blockDim.x)
        reinterpret_cast<uint4 *>(base)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (threadIdx.x < 32) {
        tmem_alloc(&slot, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = slot;
    if (threadIdx.x == 0) {
        const uint64_t ad = make_sdesc(smem_u32(a), 16, 1024, kSw128);
        const uint64_t bd = make_sdesc(smem_u32(b), 16, 1024, kSw128);
        const uint32_t id = KIND == 0 ? idesc_f16_f32(128, N, 0, 0) : idesc_e4m3_f32(128, N);
        constexpr int kAcc = 512 / N < 4 ? 512 / N : 4;
        for (int i = 0; i < iters; ++i) {
            const uint32_t d = tmem + (uint32_t)((i % kAcc) * N);
            const uint64_t off = (uint64_t)((i & 3) * 2);
            if (KIND == 0)
                mma_f16(d, ad + off, bd + off, id, 1u);
            else
                mma_e4m3(d, ad + off, bd + off, id, 1u);
        }
        tc_commit(&bar);
        mbar_wait(&bar, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int KIND, int N>
float run(int iters, cudaStream_t stream) {
    auto k = k_peak<KIND, N>;
    const int smem = 1024 + (128 + N) * 128 + 100 * 1024;  // one CTA per SM
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -1.0f;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1.0f;
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return -1.0f;
    k<<<sms, 128, smem, stream>>>(iters / 4);  // warm-up
    cudaEventRecord(e0, stream);
    k<<<sms, 128, smem, stream>>>(iters);
    cudaEventRecord(e1, stream);
    float ms = -1.0f;
    if (cudaEventSynchronize(e1) != cudaSuccess || cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess) ms = -1.0f;
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (cudaGetLastError() != cudaSuccess) return -1.0f;
    return ms;
}

}  // namespace

extern "C" float peak_tcgen05(int kind, int n, int iters, cudaStream_t stream) {
    if (iters < 4) return -1.0f;
    if (kind == 0) {
        if (n == 64) return run<0, 64>(iters, stream);
        if (n == 128) return run<0, 128>(iters, stream);
        if (n == 256) return run<0, 256>(iters, stream);
    } else if (kind == 1) {
        if (n == 64) return run<1, 64>(iters, stream);
        if (n == 128) return run<1, 128>(iters, stream);
        if (n == 256) return run<1, 256>(iters, stream);
    }
    return -1.0f;
}

extern "C" int peak_device_status(void) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof v) != cudaSuccess) return -1;
    return (int)v;
}

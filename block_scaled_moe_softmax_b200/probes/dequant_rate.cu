// dequant_rate.cu -- how fast the CUDA cores turn MXFP4 into scaled bf16 on this GPU.
//
// The design question it answers: should FC1/FC2 dequantise the E2M1 weight codes to
// bf16 (scaled by their E8M0 block scale) in shared memory for a bf16 MMA, or hand the
// codes and scales to the block-scaled MMA directly?  A dequantising GEMM must turn
// every weight element into bf16 once per tile it loads.  This program measures the
// rate at which one SM can do that: each CTA (one per SM, 1024 threads) repeatedly
// reads packed codes and a scale byte from shared memory, converts them to bf16 and
// writes the bf16 pairs back to shared memory, as a dequantising producer stage would.
// Two conversions are timed: the hardware E2M1 -> f16 conversion followed by the
// scale multiply and a bf16 conversion, and an integer construction of the bf16 bit
// pattern (exponent = scale + code exponent, one mantissa bit).  Reported: elements
// per clock per SM (from clock64 inside the kernel) and per second (CUDA events).
//
// Build and run: python -m block_scaled_moe_softmax_b200.probes.dequant_rate
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>

constexpr int kThreads = 1024;
constexpr int kWords = 2048; // 8 KB of packed codes per CTA (16 K elements); 42 KB of shared memory in all

// 8 packed E2M1 codes (one 32-bit word) times 2^(sb - 127) -> 4 bf16x2 words, hardware path
__device__ __forceinline__ void convert_hw(uint32_t w, float scale, uint32_t (&o)[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint16_t b = (uint16_t)((w >> (8 * i)) & 0xFF);
        uint32_t h2;
        asm("{\n\t.reg .b8 c;\n\tcvt.u8.u16 c, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, c;\n\t}" : "=r"(h2) : "h"(b));
        float lo, hi;
        asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
            : "=f"(lo), "=f"(hi)
            : "r"(h2));
        uint32_t r;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi * scale), "f"(lo * scale));
        o[i] = r;
    }
}

// the same with integer arithmetic on the bit patterns (scale bytes 2..252: normal results)
__device__ __forceinline__ uint32_t e2m1_bf16_bits(uint32_t nib, uint32_t sb)
{
    const uint32_t c = nib & 7;
    const uint32_t expo = sb + (c >> 1) - 1;                // biased bf16 exponent of 2^(sb-127) * value
    const uint32_t mant = (c > 1) ? ((c & 1) << 6) : 0u;   // one mantissa bit (x1.5)
    const uint32_t mag = (c == 0) ? 0u : ((expo << 7) | mant);
    return mag | ((nib & 8) << 12);
}

__device__ __forceinline__ void convert_int(uint32_t w, uint32_t sb, uint32_t (&o)[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = e2m1_bf16_bits(w >> (8 * i), sb) | (e2m1_bf16_bits(w >> (8 * i + 4), sb) << 16);
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    dequant_kernel(const uint32_t *__restrict__ src, int iters, uint32_t *__restrict__ sink,
                   long long *__restrict__ cycles)
{
    __shared__ uint32_t codes[kWords];
    __shared__ uint32_t out[4 * kWords];
    __shared__ uint8_t scales[kWords];
    for (int i = threadIdx.x; i < kWords; i += kThreads) {
        codes[i] = src[(blockIdx.x * kWords + i) % (1 << 20)];
        scales[i] = (uint8_t)(120 + (i & 7));
    }
    __syncthreads();
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
        for (int i = threadIdx.x; i < kWords; i += kThreads) {
            const uint32_t w = codes[(i + it) & (kWords - 1)];
            const uint32_t sb = scales[i];
            uint32_t o[4];
            if (kMode == 0)
                convert_hw(w, __uint_as_float(sb << 23), o);
            else
                convert_int(w, sb, o);
            *reinterpret_cast<uint4 *>(&out[4 * i]) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncthreads();
    }
    const long long t1 = clock64();
    if (threadIdx.x == 0)
        cycles[blockIdx.x] = t1 - t0;
    uint32_t acc = 0;
    for (int i = threadIdx.x; i < 4 * kWords; i += kThreads)
        acc ^= out[i];
    sink[blockIdx.x * kThreads + threadIdx.x] = acc;
}

int main()
{
    int dev = 0, nsm = 0, clk_khz = 0;
    cudaSetDevice(dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&clk_khz, cudaDevAttrClockRate, dev);
    uint32_t *src, *sink;
    long long *cyc;
    cudaMalloc(&src, sizeof(uint32_t) << 20);
    cudaMalloc(&sink, sizeof(uint32_t) * nsm * kThreads);
    cudaMalloc(&cyc, sizeof(long long) * nsm);
    cudaMemset(src, 0x5B, sizeof(uint32_t) << 20);
    const int iters = 2000;
    const char *names[2] = {"hardware cvt e2m1x2->f16x2, scale, cvt bf16x2", "integer bf16 bit construction"};
    for (int mode = 0; mode < 2; ++mode) {
        cudaEvent_t a, b;
        cudaEventCreate(&a);
        cudaEventCreate(&b);
        for (int rep = 0; rep < 2; ++rep) { // first run warms up
            cudaEventRecord(a);
            if (mode == 0)
                dequant_kernel<0><<<nsm, kThreads>>>(src, iters, sink, cyc);
            else
                dequant_kernel<1><<<nsm, kThreads>>>(src, iters, sink, cyc);
            cudaEventRecord(b);
            cudaEventSynchronize(b);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) {
            printf("error: %s\n", cudaGetErrorString(e));
            return 1;
        }
        float ms = 0.f;
        cudaEventElapsedTime(&ms, a, b);
        long long hc[1024];
        cudaMemcpy(hc, cyc, sizeof(long long) * nsm, cudaMemcpyDeviceToHost);
        double mean = 0;
        for (int i = 0; i < nsm; ++i)
            mean += (double)hc[i] / nsm;
        const double elems_per_sm = (double)iters * kWords * 8;
        printf("%s: %.1f elements/clk/SM (clock64), %.2f T elements/s over %d SMs (events, %.3f ms)\n", names[mode],
               elems_per_sm / mean, elems_per_sm * nsm / (ms * 1e-3) / 1e12, nsm, ms);
    }
    printf("device clock attribute: %d MHz\n", clk_khz / 1000);
    return 0;
}

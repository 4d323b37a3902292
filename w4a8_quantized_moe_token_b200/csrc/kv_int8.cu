// INT8 KV cache with static per-head scales, sm_100a.
//
// Method: the Kimi 2.7T MoE W4A8 article (hotelren.com 5173946), section 5 -- the
// attention KV cache is quantised to INT8 statically, with one scale per head fixed
// from a little calibration data; the scale is the symmetric form of the LLM
// quantisation primer (hotelren.com 5982361), section 2.1: max|x| / 127.
//
// Layout: x [T][H][D] bf16 row-major (token, head, channel), q [T][H][D] int8,
// scale [H] fp32.  D is a multiple of 16, so every 16-value chunk lies inside one
// (token, head) row: a thread moves one chunk (32 bytes of bf16, 16 bytes of int8)
// per iteration with 16-byte loads and stores.  The three kernels are HBM-bound
// streams; grids are a whole number of waves of 148 SMs and stride over the chunks.
#include "w4a8_common.cuh"
#include "w4a8_internal.h"

namespace w4a8 {

namespace {

constexpr int kKvThreads = 256;
constexpr int kKvMaxHeads = 1024;

inline int kv_grid(size_t chunks, int sm_count) {
    const size_t want = (chunks + kKvThreads - 1) / kKvThreads;
    const size_t cap = (size_t)sm_count * 8;  // 8 CTAs of 256 threads per SM
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

__device__ __forceinline__ float kv_bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ void load_bf16x16(const uint16_t* p, float (&f)[16]) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint4 b = *reinterpret_cast<const uint4*>(p + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        f[2 * i] = kv_bf16_to_f32((uint16_t)(w[i] & 0xFFFFu));
        f[2 * i + 1] = kv_bf16_to_f32((uint16_t)(w[i] >> 16));
    }
}

// per-head max|x| (as the bits of a non-negative float, which order like the floats)
__global__ void __launch_bounds__(kKvThreads) kv_amax_kernel(const uint16_t* __restrict__ x, size_t chunks, int H,
                                                            int cpr, uint32_t* __restrict__ amax_bits) {
    __shared__ uint32_t s_max[kKvMaxHeads];
    for (int h = threadIdx.x; h < H; h += blockDim.x) s_max[h] = 0u;
    __syncthreads();
    for (size_t c = (size_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks; c += (size_t)gridDim.x * blockDim.x) {
        float f[16];
        load_bf16x16(x + c * 16, f);
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(f[i]));
        const int h = (int)((c / (size_t)cpr) % (size_t)H);
        atomicMax(&s_max[h], __float_as_uint(m));
    }
    __syncthreads();
    for (int h = threadIdx.x; h < H; h += blockDim.x)
        if (s_max[h] != 0u) atomicMax(&amax_bits[h], s_max[h]);
}

// scale[h] = max|x| / 127 (correctly rounded), in place over the max bits
__global__ void kv_scale_kernel(uint32_t* __restrict__ amax_bits, int H) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h < H) {
        const float s = __fdiv_rn(__uint_as_float(amax_bits[h]), 127.0f);
        reinterpret_cast<float*>(amax_bits)[h] = s;
    }
}

__global__ void __launch_bounds__(kKvThreads) kv_quant_kernel(const uint16_t* __restrict__ x, size_t chunks, int H,
                                                             int cpr, const float* __restrict__ scale,
                                                             int8_t* __restrict__ q) {
    for (size_t c = (size_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks; c += (size_t)gridDim.x * blockDim.x) {
        const int h = (int)((c / (size_t)cpr) % (size_t)H);
        const float s = __ldg(scale + h);
        float f[16];
        load_bf16x16(x + c * 16, f);
        uint32_t out[4] = {0u, 0u, 0u, 0u};
        if (s > 0.f) {
            const float inv = __fdiv_rn(1.0f, s);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                out[i >> 2] |= (uint32_t)(quant_i8_fast(f[i], s, inv) & 0xFF) << (8 * (i & 3));
        }
        *reinterpret_cast<uint4*>(q + c * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

__global__ void __launch_bounds__(kKvThreads) kv_dequant_kernel(const int8_t* __restrict__ q, size_t chunks, int H,
                                                               int cpr, const float* __restrict__ scale,
                                                               uint16_t* __restrict__ x) {
    for (size_t c = (size_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks; c += (size_t)gridDim.x * blockDim.x) {
        const int h = (int)((c / (size_t)cpr) % (size_t)H);
        const float s = __ldg(scale + h);
        const uint4 p = *reinterpret_cast<const uint4*>(q + c * 16);
        const uint32_t w[4] = {p.x, p.y, p.z, p.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int v0 = (int)(int8_t)((w[i >> 1] >> (16 * (i & 1))) & 0xFF);
            const int v1 = (int)(int8_t)((w[i >> 1] >> (16 * (i & 1) + 8)) & 0xFF);
            const uint32_t b0 = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)v0, s)));
            const uint32_t b1 = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)v1, s)));
            o[i] = b0 | (b1 << 16);
        }
        *reinterpret_cast<uint4*>(x + c * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(x + c * 16 + 8) = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

}  // namespace

int kv_max_heads() { return kKvMaxHeads; }

cudaError_t launch_kv_calibrate(const uint16_t* x, int T, int H, int D, float* scale, int sm_count,
                                cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(scale, 0, sizeof(float) * (size_t)H, stream);
    if (e != cudaSuccess) return e;
    const size_t chunks = (size_t)T * H * (D / 16);
    if (chunks > 0) {
        kv_amax_kernel<<<kv_grid(chunks, sm_count), kKvThreads, 0, stream>>>(x, chunks, H, D / 16,
                                                                             reinterpret_cast<uint32_t*>(scale));
    }
    kv_scale_kernel<<<(H + 127) / 128, 128, 0, stream>>>(reinterpret_cast<uint32_t*>(scale), H);
    return cudaGetLastError();
}

cudaError_t launch_kv_quant(const uint16_t* x, int T, int H, int D, const float* scale, int8_t* q, int sm_count,
                            cudaStream_t stream) {
    const size_t chunks = (size_t)T * H * (D / 16);
    if (chunks == 0) return cudaSuccess;
    kv_quant_kernel<<<kv_grid(chunks, sm_count), kKvThreads, 0, stream>>>(x, chunks, H, D / 16, scale, q);
    return cudaGetLastError();
}

cudaError_t launch_kv_dequant(const int8_t* q, int T, int H, int D, const float* scale, uint16_t* x, int sm_count,
                              cudaStream_t stream) {
    const size_t chunks = (size_t)T * H * (D / 16);
    if (chunks == 0) return cudaSuccess;
    kv_dequant_kernel<<<kv_grid(chunks, sm_count), kKvThreads, 0, stream>>>(q, chunks, H, D / 16, scale, x);
    return cudaGetLastError();
}

}  // namespace w4a8

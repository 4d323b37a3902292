// Grouped W4A8 GEMM for sm_100a: INT4 weights (group 128, asymmetric) x INT8
// tokens on the 5th-generation tensor cores, one INT32 partial per K group.
//
// Method (W4A8 linear): «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» (pptc.cn) section 3.2
// -- the INT4 weights are expanded to INT8, multiplied with INT8 activations,
// accumulated in INT32, then scaled back to floating point; section 2.1 -- one scale
// and zero point per 128 weights; the Kimi 2.7T MoE W4A8 article (hotelren.com
// 5173946) section 4.3 -- the 4-bit -> INT8 expansion and the requantisation are
// fused into the kernel instead of going through memory.
//
// Design (one persistent CTA per SM, warp-specialised, 320 threads):
//   warp 8   producer : 1-D bulk copies of one packed weight block (8192 B of
//                       nibbles + fp16 scales + fp16 zero points for 128 output
//                       channels x 128 K) and of the matching rows of the tiled INT8
//                       token planes into an 8-stage shared-memory ring;
//   warps 0-3 converter: each thread owns one weight row, expands its 128 nibbles to
//                       signed INT8 (code - zp) in registers and writes them to a
//                       tensor-memory A slot with tcgen05.st (the expanded weights never
//                       touch shared memory);
//   warp 9   MMA       : 4 x tcgen05.mma.kind::i8 (M=128 channels, N=tokens, K=32)
//                       per group into a fresh INT32 accumulator (double-buffered);
//   warps 4-7 epilogue : tcgen05.ld of the group's INT32 partials, acc += scale[n,g] *
//                       partial in fp32 registers; after the last group the token
//                       scale is applied and the tile is written (plain, or with
//                       SwiGLU + per-row amax for the requantisation that follows).
// Weights take the MMA's M slot ("swap AB"): tokens per expert are few in decode,
// output channels are many, so M=128 is always full and N = tokens rounded to 16.
#include "w4a8_common.cuh"
#include "w4a8_internal.h"

namespace w4a8 {

namespace {

constexpr int kStages = 8;
constexpr int kBStageBytes = kBN * 128;  // 16 KB of token rows per stage
constexpr int kThreads = 320;
constexpr int kEpiWarp0 = 4, kProdWarp = 8, kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDCol0 = 0;          // two INT32 accumulators of kBN columns
constexpr uint32_t kACol0 = 2 * kBN;    // kStages A slots of 32 columns (128 x 128 int8)
static_assert(kACol0 + kStages * 32 <= kTmemCols, "tensor memory over-subscribed");

constexpr int kOffB = 0;
constexpr int kOffA = kOffB + kStages * kBStageBytes;
constexpr int kOffRed = kOffA + kStages * kBlockBytes;
constexpr int kOffBar = kOffRed + 4 * kBN * 4;
constexpr int kNumBars = 3 * kStages + 2 * 2 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack

constexpr long long kWaitLimitCycles = 4000000000ll;  // ~2 s: a bounded wait

struct Item {
    int e, nt, row0, nrows;
};

__device__ __forceinline__ Item decode_item(int u, const GemmArgs& a) {
    int lo = 0, hi = a.E;  // largest e in [0, E) with NT * mtstart[e] <= u
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (a.NT * __ldg(a.mtstart + mid) <= u) lo = mid; else hi = mid;
    }
    Item it;
    it.e = lo;
    const int m0 = __ldg(a.mtstart + lo);
    const int nmt = __ldg(a.mtstart + lo + 1) - m0;
    const int local = u - a.NT * m0;
    it.nt = local / nmt;
    const int j = local - it.nt * nmt;
    it.row0 = __ldg(a.poffs + lo) + j * kBN;
    it.nrows = min(kBN, __ldg(a.counts + lo) - j * kBN);
    return it;
}

// Bounded wait on an mbarrier phase.  Returns false (and flags the CTA and the
// device error word) when the wait runs out or another role already gave up.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitLimitCycles) {
            *abort_flag = 1;
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1) gemm_w4a8_kernel(const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base_addr - raw_addr);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    uint8_t* smA = smem + kOffA;
    float* red = reinterpret_cast<float*>(smem + kOffRed);
    const uint32_t sA = base_addr + kOffA;
    const uint32_t sB = base_addr + kOffB;
    const uint32_t bar0 = base_addr + kOffBar;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto conv_bar = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
    auto dfull_bar = [&](int b) { return bar0 + 8u * (3 * kStages + b); };
    auto dempty_bar = [&](int b) { return bar0 + 8u * (3 * kStages + 2 + b); };
    const uint32_t final_bar = bar0 + 8u * (3 * kStages + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1 + 4);  // MMA commit + 4 epilogue warps (scale read)
            mbar_init(conv_bar(s), 4);       // 4 converter warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(dfull_bar(b), 1);
            mbar_init(dempty_bar(b), 4);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = a.NT * __ldg(a.mtstart + a.E);
    const int G = a.G;

    if (warp == kProdWarp) {
        if (lane == 0) {
            uint32_t j = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                const Item it = decode_item(u, a);
                const uint32_t bbytes = (uint32_t)round_up(it.nrows, 16) * 128u;
                const uint8_t* wsrc = a.wblocks + (size_t)(it.e * a.NT + it.nt) * G * kBlockBytes;
                const int8_t* asrc = a.act + (size_t)it.row0 * 128;
                for (int g = 0; g < G; ++g, ++j) {
                    const int s = j % kStages;
                    const uint32_t ph = (j / kStages) & 1u;
                    if (!wait_bar(empty_bar(s), ph ^ 1u, abort_flag, a.err)) { ok = false; break; }
                    mbar_arrive_expect_tx(full_bar(s), kBlockBytes + bbytes);
                    bulk_g2s(sA + s * kBlockBytes, wsrc + (size_t)g * kBlockBytes, kBlockBytes, full_bar(s));
                    bulk_g2s(sB + s * kBStageBytes, asrc + (size_t)g * a.act_plane, bbytes, full_bar(s));
                }
            }
            // never leave the CTA with copies still landing in its shared memory
            const uint32_t first = j > (uint32_t)kStages ? j - kStages : 0u;
            for (uint32_t q = first; q < j; ++q) {
                const long long t0 = clock64();
                while (!mbar_try_wait(full_bar(q % kStages), (q / kStages) & 1u)) {
                    if (clock64() - t0 > kWaitLimitCycles) { atomicOr(a.err, kErrTimeout); break; }
                }
            }
        }
        __syncwarp();
    } else if (warp < 4) {
        // ---------------- converter: nibbles -> signed INT8 (code - zp) in TMEM ----------------
        const int r = threadIdx.x;  // tile row = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        uint32_t j = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            for (int g = 0; g < G; ++g, ++j) {
                const int s = j % kStages;
                const uint32_t ph = (j / kStages) & 1u;
                if (!wait_bar(full_bar(s), ph, abort_flag, a.err)) { ok = false; break; }
                const uint8_t* blk = smA + s * kBlockBytes;
                uint4 w[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) w[c] = *reinterpret_cast<const uint4*>(blk + code_chunk_offset(r, c));
                const int zp = (int)__half2float(reinterpret_cast<const __half*>(blk + kZpOff)[r]);
                const uint32_t nz = (uint32_t)(0x80 - zp) * 0x01010101u;
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t x[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int i = 4 * c + q;  // word i holds K = 8i .. 8i+7 of the group
                        v[2 * i] = ((x[q] & 0x0F0F0F0Fu) + nz) ^ 0x80808080u;
                        v[2 * i + 1] = (((x[q] >> 4) & 0x0F0F0F0Fu) + nz) ^ 0x80808080u;
                    }
                }
                tmem_st32(tmem_base + lane_base + kACol0 + (uint32_t)s * 32u, v);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(conv_bar(s));
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issue (one thread) ----------------
        if (lane == 0) {
            uint32_t j = 0, d = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                const Item it = decode_item(u, a);
                const uint32_t idesc = idesc_i8(128, round_up(it.nrows, 16));
                for (int g = 0; g < G; ++g, ++j, ++d) {
                    const int s = j % kStages;
                    const uint32_t ph = (j / kStages) & 1u;
                    const int b = d & 1;
                    const uint32_t dph = (d >> 1) & 1u;
                    if (!wait_bar(conv_bar(s), ph, abort_flag, a.err)) { ok = false; break; }
                    if (!wait_bar(dempty_bar(b), dph ^ 1u, abort_flag, a.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t dt = tmem_base + kDCol0 + (uint32_t)b * kBN;
                    const uint32_t at = tmem_base + kACol0 + (uint32_t)s * 32u;
                    const uint32_t sb = sB + s * kBStageBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_i8_ts(dt, at + kk * 8, smem_desc_sw128(sb + kk * 32), idesc, kk > 0 ? 1u : 0u);
                    tc_commit(empty_bar(s));
                    tc_commit(dfull_bar(b));
                }
            }
            // every MMA issued above must be complete before tensor memory is freed
            tc_commit(final_bar);
            const long long t0 = clock64();
            while (!mbar_try_wait(final_bar, 0)) {
                if (clock64() - t0 > kWaitLimitCycles) { atomicOr(a.err, kErrTimeout); break; }
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: fold partials, apply scales, write ----------------
        const int q = warp - kEpiWarp0;  // TMEM lane quarter
        const int r = q * 32 + lane;     // tile row
        const int et = threadIdx.x - kEpiWarp0 * 32;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        uint32_t j = 0, d = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const Item it = decode_item(u, a);
            const int nch = round_up(it.nrows, 16) >> 4;
            float acc[kBN];
#pragma unroll
            for (int i = 0; i < kBN; ++i) acc[i] = 0.f;
            const int n_out = (a.mode == 1) ? -1 : it.nt * kTileRows + r;
            for (int g = 0; g < G; ++g, ++j, ++d) {
                const int s = j % kStages;
                const int b = d & 1;
                const uint32_t dph = (d >> 1) & 1u;
                if (!wait_bar(dfull_bar(b), dph, abort_flag, a.err)) { ok = false; break; }
                tc_fence_after();
                const float sc = __half2float(reinterpret_cast<const __half*>(smA + s * kBlockBytes + kScaleOff)[r]);
                const uint32_t taddr = tmem_base + lane_base + kDCol0 + (uint32_t)b * kBN;
#pragma unroll
                for (int c = 0; c < kBN / 16; ++c) {
                    if (c < nch) {
                        uint32_t v[16];
                        tmem_ld16(taddr + c * 16, v);
                        tmem_ld_wait();
                        if (a.partials != nullptr && n_out < a.nvalid) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int m = c * 16 + i;
                                if (m < it.nrows)
                                    a.partials[((size_t)(it.row0 + m) * a.nvalid + n_out) * G + g] = (int32_t)v[i];
                            }
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc[c * 16 + i] = fmaf(sc, (float)(int32_t)v[i], acc[c * 16 + i]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(dempty_bar(b));
                    mbar_arrive(empty_bar(s));
                }
            }
            if (!ok) break;
            if (a.mode != 1) {
                if (n_out < a.nvalid) {
#pragma unroll
                    for (int m = 0; m < kBN; ++m) {
                        if (m < it.nrows) {
                            const float sa = __ldg(a.act_scale + it.row0 + m);
                            a.out[(size_t)(it.row0 + m) * a.ldo + n_out] = acc[m] * sa;
                        }
                    }
                }
            } else {
                // SwiGLU: even tile rows hold gate channel f, odd rows the matching up channel
                const int f = it.nt * (kTileRows / 2) + (r >> 1);
                const bool is_gate = (r & 1) == 0;
                const bool valid = is_gate && f < a.nvalid;
#pragma unroll
                for (int m = 0; m < kBN; ++m) {
                    if (m < it.nrows) {
                        const float sa = __ldg(a.act_scale + it.row0 + m);
                        const float y = acc[m] * sa;
                        const float yo = __shfl_xor_sync(0xffffffffu, y, 1);
                        float hv = 0.f;
                        if (valid) {
                            hv = (y / (1.0f + expf(-y))) * yo;
                            a.out[(size_t)(it.row0 + m) * a.ldo + f] = hv;
                        }
                        const uint32_t am = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(hv)));
                        if (lane == 0) red[q * kBN + m] = __uint_as_float(am);
                    }
                }
                named_bar_sync(1, 128);
                for (int m = et; m < it.nrows; m += 128) {
                    const float mx = fmaxf(fmaxf(red[m], red[kBN + m]), fmaxf(red[2 * kBN + m], red[3 * kBN + m]));
                    atomicMax(a.amax + it.row0 + m, __float_as_uint(mx));
                }
                named_bar_sync(1, 128);
            }
        }
    }

    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace

size_t gemm_smem_bytes() { return (size_t)kSmemBytes; }

cudaError_t launch_gemm(const GemmArgs& a, int num_ctas, cudaStream_t stream) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemm_w4a8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    gemm_w4a8_kernel<<<num_ctas, kThreads, kSmemBytes, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace w4a8

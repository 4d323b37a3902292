// Grouped W4A8 GEMM for sm_100a: INT4 weights (group 128, asymmetric) x INT8
// tokens on the 5th-generation tensor cores, one INT32 partial per K group.
//
// Method (W4A8 linear): «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» (pptc.cn) section 3.2
// -- the INT4 weights are expanded to INT8, multiplied with INT8 activations,
// accumulated in INT32, then scaled back to floating point; section 2.1 -- one scale
// and zero point per 128 weights; the Kimi 2.7T MoE W4A8 article (hotelren.com
// 5173946) section 4.3 -- the 4-bit -> INT8 expansion is fused into the kernel
// instead of going through memory.
//
// One persistent CTA per SM, warp-specialised.  A "step" is one 128-wide K group of
// one tile (128 output channels x up to BN tokens); steps are numbered j = 0, 1, ...
// over all the tiles a CTA processes, and every role walks the same sequence.
//   2 producer warps    : (alternate steps) 1-D bulk copies of the step's packed weight block (8192 B
//                         of nibbles + fp16 scales + fp16 zero points) and of its run
//                         of tiled INT8 token rows into an NS-stage shared-memory ring;
//   converter groups    : (4 warps each, alternate steps) each thread owns one weight
//                         row, expands its 128 nibbles to signed INT8 (code - zp) in
//                         registers and stores them to one of NA tensor-memory A slots
//                         with tcgen05.st; it also publishes the row's fp32 scale in a
//                         ring for the epilogue;
//   2 MMA warps         : (alternate steps; the issue rate of tcgen05.mma is a
//                         per-thread limit, two issuers double it) 4 x
//                         tcgen05.mma.kind::i8 per step (M=128 channels, N=tokens,
//                         K=32, A in tensor memory, B in shared memory) into one of ND
//                         INT32 accumulators;
//   epilogue warpgroups : tcgen05.ld of a step's partials and acc += scale[n,g] *
//                         partial in fp32 registers; after the tile's last step the
//                         token scale is applied and the tile stored (plain, or
//                         SwiGLU on gate/up lane pairs).
// Weights take the MMA's M slot ("swap AB"): decode has few tokens per expert and
// many channels, so M=128 is always full and N shrinks to the tokens.
//
// This kernel serves layers with many tokens per expert (tiles of up to 128 tokens);
// decode-shaped layers use gemm_decode.cu.  Every step starts with a bf16 MMA that
// resets its accumulator to 0x4B400000 (the fp32 bit pattern of 1.5 * 2^23, see
// mma_reset_acc); the step's INT8 MMAs add the INT32 partial P (|P| < 2^22) on top, so
// the result read as fp32 is exactly 1.5 * 2^23 + P and the epilogue recovers P with
// one packed fp32 subtraction instead of an int -> float conversion.  The epilogue
// only reads the accumulator and releases it: no tensor-memory writes on the CUDA cores.
#include "w4a8_common.cuh"
#include "w4a8_internal.h"

namespace w4a8 {

namespace {

constexpr uint32_t kMagicBits = 0x4B400000u;  // 1.5 * 2^23 (what the reset MMA writes)
constexpr float kMagicF = 12582912.0f;

#ifndef W4A8_BACKOFF
#define W4A8_BACKOFF() ((void)0)
#endif

// Compile-time shape of one kernel instance.
//   BN    : tokens per tile at most (MMA N <= BN)
//   NS    : shared-memory stages        NA : tensor-memory A slots
//   ND    : INT32 accumulators          NEPI: epilogue warpgroups (split the columns)
//   NCG   : converter warpgroups (they take alternate steps)
//   GRP   : weights per scale along K (64, 128 or 256; a step is always one 128-wide plane)
template <int BN_, int NS_, int NA_, int ND_, int NEPI_, int NCG_, int GRP_ = 128>
struct Cfg {
    static constexpr int BN = BN_, NS = NS_, NA = NA_, ND = ND_, NEPI = NEPI_, NCG = NCG_, GRP = GRP_;
    static constexpr int kBlk = block_bytes_for(GRP);  // packed weight block of one plane
    static constexpr int kNSC = 16;       // scale ring slots (>= NA + ND + 4)
    static constexpr int kCW = BN / NEPI;  // accumulator columns per epilogue thread
    // warpgroups: NCG converter groups, NEPI epilogue groups, 1 control group
    // (producer warp, two MMA warps, second producer warp)
    static constexpr int kConvWarps = 4 * NCG;
    static constexpr int kEpiWarp0 = kConvWarps;
    static constexpr int kProdWarp = kEpiWarp0 + 4 * NEPI;
    static constexpr int kMmaWarp0 = kProdWarp + 1;
    static constexpr int kThreads = 32 * (kProdWarp + 4);
    // register split (setmaxnreg): the launch gives every thread kRegLaunch; the
    // converter and control groups shrink, the epilogue groups grow
    static constexpr int kRegLaunch = (65536 / kThreads) / 8 * 8;
    static constexpr int kRegConv = 80;
    static constexpr int kRegCtrl = 48;
    static constexpr int kRegEpiFit = ((kRegLaunch * kThreads / 128 - NCG * kRegConv - kRegCtrl) / NEPI) / 8 * 8;
    static constexpr int kRegEpi = kRegEpiFit > 232 ? 232 : kRegEpiFit;
    static_assert(128 * (NCG * kRegConv + kRegCtrl + NEPI * kRegEpi) <= kRegLaunch * kThreads, "register split");
    static constexpr int kBStageBytes = BN * 128;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kACol0 = 0;
    static constexpr uint32_t kDCol0 = NA * 32;
    static_assert(kDCol0 + ND * BN <= kTmemCols, "tensor memory over-subscribed");
    static_assert(kNSC >= NA + ND + 4, "scale ring too small");
    static_assert(NS % 2 == 0, "the two producers own the stages of one parity each");
    static_assert(kCW % 16 == 0 && (kCW <= 64 || kCW % 64 == 0), "epilogue column split");
    // shared memory carve-up
    static constexpr int kOffB = 0;  // 1024-aligned (128-byte swizzle atoms)
    static constexpr int kOffA = kOffB + NS * kBStageBytes;
    static constexpr int kOffSc = kOffA + NS * kBlk;  // ring: fp32 scale per row and group
    static constexpr int kOffReset = kOffSc + kNSC * kTileRows * 4;  // the accumulator-reset operands
    // output staging tile: fp32 [BN tokens][128 channels] (plain output) or
    // [BN tokens][kStageH] (SwiGLU output, 64 channels + padding against bank conflicts)
    static constexpr int kStageH = 80;
    // bf16 outputs (SwiGLU h): rows of kStageH16 bf16 values (64 channels + 16 against
    // bank conflicts, a 16-byte multiple)
    static constexpr int kStageH16 = 80;
    static constexpr int kOffStage = kOffReset + 2 * kResetTileBytes;
    static constexpr int kOffSa = kOffStage + BN * kTileRows * 4;  // the tile's token scales
    static constexpr int kOffBar = kOffSa + BN * 4;
    // full[NS] empty[NS] conv[NA] aempty[NA] dfull[ND] dempty[ND] scfull[NSC] final[2] stage[2]
    static constexpr int kNumBars = 2 * NS + 2 * NA + 2 * ND + kNSC + 2 + 2;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
    static_assert(kSmemBytes <= 227 * 1024, "shared memory over-subscribed");
};

struct Item {
    int e, nt, row0, nrows;
};

// Tiles are ordered row-tile-major, weight tile fastest: the CTAs working at the
// same time share the row tile's tokens (and, for experts with several row tiles,
// the weights of nearby tiles) in L2.
template <int BN>
__device__ __forceinline__ Item decode_item(int u, const GemmArgs& a) {
    const int mt = u / a.NT;
    const int4 t = __ldg(a.mt_tab + mt);
    Item it;
    it.e = t.x;
    it.nt = u - mt * a.NT;
    it.row0 = t.y;
    it.nrows = t.z;
    return it;
}

// Bounded wait on an mbarrier phase.  Returns false (and flags the CTA and the
// device error word) when the wait runs out or another role already gave up.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint32_t* err,
                                         long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t n = 1;; ++n) {
        W4A8_BACKOFF();
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 15u) == 0) {
            if (*abort_flag) return false;
            if (clock64() - t0 > limit) {
                *abort_flag = 1;
                atomicOr(err, kErrTimeout);
                return false;
            }
        }
    }
}

// wait without the abort bookkeeping, for draining at exit
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint32_t* err, long long limit) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) {
            atomicOr(err, kErrTimeout);
            return;
        }
    }
}

// a packed pair of accumulators (low word: even column) += sc * (x - 1.5*2^23) with
// fp32x2 arithmetic: acc2 += sc2 * (x - m2), sc2 and m2 holding the value twice; x holds
// the INT32 partial P as the fp32 value 1.5 * 2^23 + P, so the subtraction is exact
__device__ __forceinline__ void fold2_packed(uint64_t& acc2, uint64_t sc2, uint64_t m2, uint32_t x0, uint32_t x1) {
    asm("{\n\t.reg .b64 x;\n\t"
        "mov.b64 x, {%1, %2};\n\t"
        "sub.rn.f32x2 x, x, %3;\n\t"
        "fma.rn.f32x2 %0, %4, x, %0;\n\t}"
        : "+l"(acc2)
        : "r"(x0), "r"(x1), "l"(m2), "l"(sc2));
}

__device__ __forceinline__ uint64_t splat2(float v) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ void unpack2(uint64_t p, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}

__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// mbarrier addresses (used with bar0, NS, NA, ND, kNSC of the kernel's configuration in scope)
#define FULL_BAR(s) (bar0 + 8u * (uint32_t)(s))
#define EMPTY_BAR(s) (bar0 + 8u * (uint32_t)(NS + (s)))
#define CONV_BAR(x) (bar0 + 8u * (uint32_t)(2 * NS + (x)))
#define AEMPTY_BAR(x) (bar0 + 8u * (uint32_t)(2 * NS + NA + (x)))
#define DFULL_BAR(b) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + (b)))
#define DEMPTY_BAR(b) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + ND + (b)))
#define SCFULL_BAR(i) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + 2 * ND + (i)))
#define FINAL_BAR(m) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + 2 * ND + kNSC + (m)))
#define STAGE_BAR(m) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + 2 * ND + kNSC + 2 + (m)))

template <class C, bool kPartials>
__global__ void __launch_bounds__(C::kThreads, 1) gemm_w4a8_kernel(const GemmArgs a) {
    constexpr int BN = C::BN, NS = C::NS, NA = C::NA, ND = C::ND, kNSC = C::kNSC, kCW = C::kCW;
    constexpr int GRP = C::GRP, kBlk = C::kBlk;
    // groups per plane (group 64) and planes per group (group 256)
    constexpr int kGPP = GRP < kGroup ? kGroup / GRP : 1, kPPG = GRP > kGroup ? GRP / kGroup : 1;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base_addr - raw_addr);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    uint8_t* smA = smem + C::kOffA;
    float* sc_ring = reinterpret_cast<float*>(smem + C::kOffSc);
    const uint32_t sA = base_addr + C::kOffA;
    const uint32_t sB = base_addr + C::kOffB;
    const uint32_t bar0 = base_addr + C::kOffBar;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(FULL_BAR(s), 1);
            mbar_init(EMPTY_BAR(s), 1);  // commit of the MMAs that read the stage
        }
        for (int x = 0; x < NA; ++x) {
            mbar_init(CONV_BAR(x), 4);    // the 4 warps of one converter group
            mbar_init(AEMPTY_BAR(x), 1);  // commit of the MMAs that read the A slot
        }
        for (int b = 0; b < ND; ++b) {
            mbar_init(DFULL_BAR(b), 1);
            mbar_init(DEMPTY_BAR(b), 4 * C::NEPI);
        }
        for (int i = 0; i < kNSC; ++i) mbar_init(SCFULL_BAR(i), 4);
        mbar_init(FINAL_BAR(0), 1);
        mbar_init(FINAL_BAR(1), 1);
        mbar_init(STAGE_BAR(0), 4 * C::NEPI);  // staging tile free, token scales written
        mbar_init(STAGE_BAR(1), 4 * C::NEPI);  // staging tile written
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::kMmaWarp0) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    fill_reset_tiles(smem + C::kOffReset);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t sReset = base_addr + C::kOffReset;

    const int q = warp & 3;  // TMEM lane quarter of this warp
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;

    // the set-up above (barriers, tensor memory, reset tiles) overlaps the previous
    // kernel's tail; from here on this kernel reads its results
    grid_dep_wait();
    const int total = a.NT * __ldg(a.n_mtiles);
    const int G = a.G;                // 128-wide K planes (steps) per tile
    const int Gq = G * kGroup / GRP;  // quantisation groups per tile

    // each role first moves its warpgroup's register budget (converter and control
    // groups give registers to the epilogue groups), then runs
    if (warp >= C::kProdWarp) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegCtrl));
    }
    if (warp == C::kProdWarp || warp == C::kProdWarp + 3) {
        // ---------------- producers: warp pi takes the steps with j % 2 == pi ----------------
        // (the time a thread needs per ring step is fixed, whatever the copy size, so two
        // issuing threads are needed to keep HBM busy with 8.7 KB weight blocks)
        const int pi = warp == C::kProdWarp ? 0 : 1;
        if (lane == 0) {
            uint32_t j = 0, last = 0;
            bool ok = true, rdy = false;  // rdy: an early test found this step's stage free
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                const Item it = decode_item<BN>(u, a);
                const uint32_t bbytes = (uint32_t)round_up(it.nrows, 16) * 128u;
                const uint8_t* wsrc = a.wblocks + (size_t)(it.e * a.NT + it.nt) * G * kBlk;
                const int8_t* asrc = a.act + (size_t)it.row0 * 128;
                for (int g = 0; g < G; ++g, ++j) {
                    if ((int)(j & 1u) != pi) continue;
                    last = j + 1;
                    const int s = j % NS;
                    if (!rdy && !wait_bar(EMPTY_BAR(s), ((j / NS) & 1u) ^ 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                    rdy = mbar_test(EMPTY_BAR((j + 2) % NS), (((j + 2) / NS) & 1u) ^ 1u);
                    // test hook: leave the first step's stage empty, so that its consumers time out
                    if (j == 0 && blockIdx.x == 0 && (a.debug & kDebugSkipFirstCopy)) continue;
                    mbar_arrive_expect_tx(FULL_BAR(s), kBlk + bbytes);
                    bulk_g2s(sA + s * kBlk, wsrc + (size_t)g * kBlk, kBlk, FULL_BAR(s));
                    bulk_g2s(sB + s * C::kBStageBytes, asrc + (size_t)g * a.act_plane, bbytes, FULL_BAR(s));
                }
            }
            // never leave the CTA with copies still landing in its shared memory
            for (uint32_t qq = (last > (uint32_t)NS ? last - NS : 0u); qq < last; ++qq)
                if ((int)(qq & 1u) == pi) drain_wait(FULL_BAR(qq % NS), (qq / NS) & 1u, a.err, a.wait_limit);
        }
        __syncwarp();
    } else if (warp < C::kConvWarps) {
        // ---------------- converters: nibbles -> signed INT8 (code - zp) in TMEM ----------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegConv));
        const int cg = warp >> 2;         // converter group: takes the steps with j % NCG == cg
        const int r = threadIdx.x & 127;  // tile row = TMEM lane
        const int nsteps = ((total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * G;
        // The tensor-memory store of step j completes while step j + NCG is fetched and
        // converted; step j is signalled just before step j + NCG's store.
        int prev = -1;  // step stored but not yet signalled
        auto signal = [&](int jp) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(CONV_BAR(jp % NA));
                // the scales of the groups that start in plane jp
                if (kPPG == 1 || jp % kPPG == 0) {
#pragma unroll
                    for (int sub = 0; sub < kGPP; ++sub) mbar_arrive(SCFULL_BAR((jp * kGPP / kPPG + sub) % kNSC));
                }
            }
        };
        bool full_rdy = false, aslot_rdy = false;  // early tests of this step's barriers
        for (int j = cg; j < nsteps; j += C::NCG) {
            const int s = j % NS;
            const int x = j % NA;
            if (!full_rdy && !wait_bar(FULL_BAR(s), (j / NS) & 1u, abort_flag, a.err, a.wait_limit)) break;
            if (!aslot_rdy && !wait_bar(AEMPTY_BAR(x), ((j / NA) & 1u) ^ 1u, abort_flag, a.err, a.wait_limit)) break;
            {
                const int jn = j + C::NCG;
                full_rdy = mbar_test(FULL_BAR(jn % NS), (jn / NS) & 1u);
                aslot_rdy = mbar_test(AEMPTY_BAR(jn % NA), ((jn / NA) & 1u) ^ 1u);
            }
            const uint8_t* blk = smA + s * kBlk;
            uint4 w[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) w[c] = *reinterpret_cast<const uint4*>(blk + code_chunk_offset(r, c));
            // zero point of each half plane (one group 64 per half; else the plane's group)
            int zp[2];
            zp[0] = (int)__half2float(reinterpret_cast<const __half*>(blk + kZpOff)[r]);
            zp[1] = kGPP == 2 ? (int)__half2float(reinterpret_cast<const __half*>(blk + kZpOff + 512)[r]) : zp[0];
            // the scales of the groups that start in this plane
            if (kPPG == 1 || j % kPPG == 0) {
#pragma unroll
                for (int sub = 0; sub < kGPP; ++sub)
                    sc_ring[((j * kGPP / kPPG + sub) % kNSC) * kTileRows + r] =
                        __half2float(reinterpret_cast<const __half*>(blk + kScaleOff + sub * 512)[r]);
            }
            uint32_t v[32];
            {
                // signed INT8 (code - zp): byte-wise (code + 128 - zp) ^ 128, no carries
                const uint32_t nz0 = (uint32_t)(0x80 - zp[0]) * 0x01010101u;
                const uint32_t nz1 = (uint32_t)(0x80 - zp[1]) * 0x01010101u;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t xw[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
                    const uint32_t nz = c < 2 ? nz0 : nz1;  // chunks 0-1: K 0..63, 2-3: K 64..127
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        const int i = 4 * c + qq;  // word i holds K = 8i .. 8i+7 of the plane
                        v[2 * i] = ((xw[qq] & 0x0F0F0F0Fu) + nz) ^ 0x80808080u;
                        v[2 * i + 1] = (((xw[qq] >> 4) & 0x0F0F0F0Fu) + nz) ^ 0x80808080u;
                    }
                }
            }
            if (prev >= 0) signal(prev);
            tmem_st32(tmem_base + lane_base + C::kACol0 + (uint32_t)x * 32u, v);
            prev = j;
        }
        if (prev >= 0) signal(prev);
    } else if (warp >= C::kMmaWarp0) {
        // ---------------- MMA issue: warp mi takes the steps with j % 2 == mi ----------------
        // The whole warp runs the loop (its values stay warp-uniform, so the operands of
        // tcgen05.mma need no per-instruction moves); one elected thread issues.
        const int mi = warp - C::kMmaWarp0;
        {
            uint32_t j = 0;
            bool ok = true, conv_rdy = false, acc_rdy = false;  // early tests of this step's barriers
            for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                const Item it = decode_item<BN>(u, a);
                const int ncols = round_up(it.nrows, 16);
                const uint32_t idesc = idesc_i8(128, ncols);
                for (int g = 0; g < G; ++g, ++j) {
                    if constexpr (GRP != kGroup) {
                        // group 64: two accumulators per plane; group 256: the two planes of a
                        // group go to the same warp and accumulator.  Plain waits.
                        if ((int)((j / kPPG) & 1u) != mi) continue;
                        const int s = j % NS, x = j % NA;
                        const bool starts = kPPG == 1 || j % kPPG == 0;  // a group starts in this plane
                        if (!wait_bar(CONV_BAR(x), (j / NA) & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                        if (starts) {
#pragma unroll
                            for (int sub = 0; sub < kGPP; ++sub) {
                                const uint32_t qg = j * kGPP / kPPG + sub;
                                if (ok && !wait_bar(DEMPTY_BAR(qg % ND), ((qg / ND) & 1u) ^ 1u, abort_flag, a.err, a.wait_limit))
                                    ok = false;
                            }
                            if (!ok) break;
                        }
                        tc_fence_after();
                        const uint32_t at = tmem_base + C::kACol0 + (uint32_t)x * 32u;
                        const uint32_t sb = sB + s * C::kBStageBytes;
                        if (elect_one()) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t kg = j * (uint32_t)kGroup + kk * 32u;  // K position of the MMA
                                const uint32_t qg = kg / GRP;                          // its group
                                const uint32_t dt = tmem_base + C::kDCol0 + (qg % ND) * BN;
                                if (kg % GRP == 0) mma_reset_acc(dt, sReset, ncols);
                                mma_i8_ts(dt, at + kk * 8, smem_desc_sw128(sb + kk * 32), idesc, 1u);
                                if ((kg + 32u) % GRP == 0) tc_commit(DFULL_BAR(qg % ND));
                            }
                            tc_commit(EMPTY_BAR(s));
                            tc_commit(AEMPTY_BAR(x));
                        }
                        __syncwarp();
                        continue;
                    }
                    if ((int)(j & 1u) != mi) continue;
                    const int s = j % NS, x = j % NA, b = j % ND;
                    if (!conv_rdy && !wait_bar(CONV_BAR(x), (j / NA) & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                    if (!acc_rdy && !wait_bar(DEMPTY_BAR(b), ((j / ND) & 1u) ^ 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                    conv_rdy = mbar_test(CONV_BAR((j + 2) % NA), ((j + 2) / NA) & 1u);
                    acc_rdy = mbar_test(DEMPTY_BAR((j + 2) % ND), (((j + 2) / ND) & 1u) ^ 1u);
                    tc_fence_after();
                    const uint32_t dt = tmem_base + C::kDCol0 + (uint32_t)b * BN;
                    const uint32_t at = tmem_base + C::kACol0 + (uint32_t)x * 32u;
                    const uint32_t sb = sB + s * C::kBStageBytes;
                    if (elect_one()) {
                        mma_reset_acc(dt, sReset, ncols);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_i8_ts(dt, at + kk * 8, smem_desc_sw128(sb + kk * 32), idesc, 1u);
                        tc_commit(EMPTY_BAR(s));
                        tc_commit(AEMPTY_BAR(x));
                        tc_commit(DFULL_BAR(b));
                    }
                    __syncwarp();
                }
            }
            // every MMA this warp issued must be complete before tensor memory is freed
            if (elect_one()) tc_commit(FINAL_BAR(mi));
            __syncwarp();
            drain_wait(FINAL_BAR(mi), 0, a.err, a.wait_limit);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue ----------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kRegEpi));
        const int eh = (warp - C::kEpiWarp0) >> 2;  // epilogue warpgroup: columns [eh*kCW, eh*kCW + kCW)
        const int r = q * 32 + lane;                 // tile row = TMEM lane
        const int col0 = eh * kCW;
        const int nsteps = ((total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * G;
        // The tile is written through a shared-memory staging tile and 1-D bulk copies
        // (one output row per issuing thread), so the epilogue goes on with the next
        // tile while the stores drain; this needs every output row to start on a
        // 16-byte boundary.  Otherwise (a dense output with N % 4 != 0) it stores directly.
        // (bf16 outputs, mode 1 with out_bf16: rows must start on 16 bytes too)
        const bool obf = a.out_bf16 != 0 && a.mode == 1;
        const int oal = obf ? 8 : 4;
        const bool staged = !kPartials && (a.ldo % oal == 0) && (a.mode == 1 || a.nvalid % oal == 0);
        float* stage = reinterpret_cast<float*>(smem + C::kOffStage);
        uint16_t* stage16 = reinterpret_cast<uint16_t*>(smem + C::kOffStage);
        uint16_t* out16 = reinterpret_cast<uint16_t*>(a.out);
        float* sa_s = reinterpret_cast<float*>(smem + C::kOffSa);
        const int et = threadIdx.x - 32 * C::kEpiWarp0;  // epilogue thread 0 .. 128 * NEPI - 1
        bool issued = false;                            // a bulk copy of this thread is in flight
        uint32_t ntile = 0;
        float sc4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t j = 0;
        bool ok = true, acc_rdy = false, sc_rdy = false;  // early tests of this step's barriers
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++ntile) {
            const Item it = decode_item<BN>(u, a);
            // the tile's token scales, loaded now and used at its end
            const float my_sa = (staged && eh == 0 && r < it.nrows) ? __ldg(a.act_scale + it.row0 + r) : 0.f;
            uint64_t acc2[kCW / 2];  // column pairs, packed fp32x2
#pragma unroll
            for (int i = 0; i < kCW / 2; ++i) acc2[i] = 0ull;
            const uint64_t m2 = splat2(kMagicF);
            const int n_out = (a.mode == 1) ? -1 : it.nt * kTileRows + r;
            if constexpr (GRP != kGroup) {
                // one pass per quantisation group (j counts groups here); plain waits
                for (int g = 0; g < Gq; ++g, ++j) {
                    const int b = j % ND;
                    if (!wait_bar(SCFULL_BAR(j % kNSC), (j / kNSC) & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                    const uint64_t sc2 = splat2(sc_ring[(j % kNSC) * kTileRows + r]);
                    if (!wait_bar(DFULL_BAR(b), (j / ND) & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t taddr = tmem_base + lane_base + C::kDCol0 + (uint32_t)b * BN + col0;
                    if constexpr (!kPartials) {
                        static_assert(kCW == 64, "64 columns per epilogue thread");
                        uint32_t v[64];
                        tmem_ld32(taddr, v);
                        tmem_ld_wait();
                        tmem_ld32(taddr + 32, v + 32);
#pragma unroll
                        for (int i = 0; i < 32; i += 2) fold2_packed(acc2[i / 2], sc2, m2, v[i], v[i + 1]);
                        tmem_ld_wait();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(DEMPTY_BAR(b));
#pragma unroll
                        for (int i = 32; i < 64; i += 2) fold2_packed(acc2[i / 2], sc2, m2, v[i], v[i + 1]);
                    } else {
#pragma unroll
                        for (int rd = 0; rd < kCW / 16; ++rd) {
                            const int m0 = col0 + rd * 16;
                            uint32_t v[16];
                            tmem_ld16(taddr + rd * 16, v);
                            tmem_ld_wait();
                            if (n_out < a.nvalid) {
                                int32_t* pp = a.partials + ((size_t)(it.row0 + m0) * a.nvalid + n_out) * Gq + g;
                                const size_t pstride = (size_t)a.nvalid * Gq;
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    if (m0 + i < it.nrows) pp[i * pstride] = (int32_t)(v[i] - kMagicBits);
                            }
#pragma unroll
                            for (int i = 0; i < 16; i += 2)
                                fold2_packed(acc2[(rd * 16 + i) / 2], sc2, m2, v[i], v[i + 1]);
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(DEMPTY_BAR(b));
                    }
                }
            }
            for (int g = 0; g < (GRP == kGroup ? G : 0); ++g, ++j) {
                const int b = j % ND;
                // the scales come in blocks of four steps: one wait on the last step of
                // the block (of each converter group, which work in step order) covers all four
                if ((j & 3u) == 0) {
                    const uint32_t jl = min(j + 3u, (uint32_t)nsteps - 1u);
#pragma unroll
                    for (int d = 0; d < C::NCG; ++d) {
                        const uint32_t jj = jl - (uint32_t)d;
                        if (jj >= j && !(sc_rdy && d == 0) &&
                            !wait_bar(SCFULL_BAR(jj % kNSC), (jj / kNSC) & 1u, abort_flag, a.err, a.wait_limit))
                            ok = false;
                    }
                    if (!ok) break;
#pragma unroll
                    for (int d = 0; d < 4; ++d) sc4[d] = sc_ring[((j + d) % kNSC) * kTileRows + r];
                } else {
#pragma unroll
                    for (int d = 0; d < 3; ++d) sc4[d] = sc4[d + 1];
                }
                const uint64_t sc2 = splat2(sc4[0]);
                if (!acc_rdy && !wait_bar(DFULL_BAR(b), (j / ND) & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                // early tests for the next step (the scales of the next block of four when
                // this step ends one)
                acc_rdy = mbar_test(DFULL_BAR((j + 1) % ND), ((j + 1) / ND) & 1u);
                if ((j & 3u) == 3u) {
                    const uint32_t jl = min(j + 4u, (uint32_t)nsteps - 1u);
                    sc_rdy = jl > j && mbar_test(SCFULL_BAR(jl % kNSC), (jl / kNSC) & 1u);
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + lane_base + C::kDCol0 + (uint32_t)b * BN + col0;
                // Columns past the tile's tokens (beyond the MMAs' N) hold stale values:
                // they only reach outputs that are never stored.
                if constexpr (!kPartials) {
                    // the first 32 columns are folded while the second 32 are loaded; the
                    // buffer goes back to the MMA warps once both loads are complete
                    static_assert(kCW == 64, "64 columns per epilogue thread");
                    uint32_t v[64];
                    tmem_ld32(taddr, v);
                    tmem_ld_wait();
                    tmem_ld32(taddr + 32, v + 32);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) fold2_packed(acc2[i / 2], sc2, m2, v[i], v[i + 1]);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(DEMPTY_BAR(b));
#pragma unroll
                    for (int i = 32; i < 64; i += 2) fold2_packed(acc2[i / 2], sc2, m2, v[i], v[i + 1]);
                } else {
                    // the INT32-partials output: batches of 16 columns (no spill)
#pragma unroll
                    for (int rd = 0; rd < kCW / 16; ++rd) {
                        const int m0 = col0 + rd * 16;
                        uint32_t v[16];
                        tmem_ld16(taddr + rd * 16, v);
                        tmem_ld_wait();
                        if (n_out < a.nvalid) {
                            int32_t* pp = a.partials + ((size_t)(it.row0 + m0) * a.nvalid + n_out) * G + g;
                            const size_t pstride = (size_t)a.nvalid * G;
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                if (m0 + i < it.nrows) pp[i * pstride] = (int32_t)(v[i] - kMagicBits);
                        }
#pragma unroll
                        for (int i = 0; i < 16; i += 2) fold2_packed(acc2[(rd * 16 + i) / 2], sc2, m2, v[i], v[i + 1]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(DEMPTY_BAR(b));
                }
            }
            if (!ok) break;
            float acc[kCW];
#pragma unroll
            for (int i = 0; i < kCW; i += 2) unpack2(acc2[i / 2], acc[i], acc[i + 1]);
            const float* sap = a.act_scale + it.row0 + col0;
            const int ncol = it.nrows - col0;
            if (staged) {
                // 1. this thread's previous copy has read the staging tile; publish the token
                //    scales; all epilogue warps agree (bounded waits: an abort ends the loop)
                if (issued) bulk_wait_read_all();
                if (eh == 0) sa_s[r] = my_sa;
                __syncwarp();
                if (lane == 0) mbar_arrive(STAGE_BAR(0));
                if (!wait_bar(STAGE_BAR(0), ntile & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                // 2. scaled (and SwiGLU-combined) results into the staging tile
                if (a.mode != 1) {
#pragma unroll
                    for (int i = 0; i < kCW; i += 4) {
                        const float4 s4 = *reinterpret_cast<const float4*>(sa_s + col0 + i);
                        stage[(col0 + i) * kTileRows + r] = acc[i] * s4.x;
                        stage[(col0 + i + 1) * kTileRows + r] = acc[i + 1] * s4.y;
                        stage[(col0 + i + 2) * kTileRows + r] = acc[i + 2] * s4.z;
                        stage[(col0 + i + 3) * kTileRows + r] = acc[i + 3] * s4.w;
                    }
                } else {
                    // even tile rows hold gate channel f, odd rows the matching up channel;
                    // per token pair (i, i+1) the lanes of a pair swap one value: the even
                    // lane finishes token i, the odd lane token i+1
                    const int odd = r & 1;
                    float* srow = stage + (col0 + odd) * C::kStageH + (r >> 1);
                    uint16_t* srow16 = stage16 + (col0 + odd) * C::kStageH16 + (r >> 1);
#pragma unroll
                    for (int i = 0; i < kCW; i += 2) {
                        const float send = odd ? acc[i] : acc[i + 1];
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                        const float si = sa_s[col0 + i + odd];
                        const float g = (odd ? recv : acc[i]) * si;
                        const float uu = (odd ? acc[i + 1] : recv) * si;
                        if (obf)
                            srow16[i * C::kStageH16] = bf16_bits(silu_mul(g, uu));
                        else
                            srow[i * C::kStageH] = silu_mul(g, uu);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(STAGE_BAR(1));
                if (!wait_bar(STAGE_BAR(1), ntile & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                // 3. one bulk copy per token row of the tile, each by its own thread
                if (et < it.nrows) {
                    if (a.mode != 1) {
                        const int n0 = it.nt * kTileRows;
                        const int w = min(kTileRows, a.nvalid - n0);
                        bulk_s2g(a.out + (size_t)(it.row0 + et) * a.ldo + n0,
                                 smem_u32(stage + et * kTileRows), (uint32_t)w * 4u);
                    } else if (obf) {
                        // all 64 channels: past F they land in the row's padding
                        bulk_s2g(out16 + (size_t)(it.row0 + et) * a.ldo + it.nt * (kTileRows / 2),
                                 smem_u32(stage16 + et * C::kStageH16), (kTileRows / 2) * 2u);
                    } else {
                        bulk_s2g(a.out + (size_t)(it.row0 + et) * a.ldo + it.nt * (kTileRows / 2),
                                 smem_u32(stage + et * C::kStageH), (kTileRows / 2) * 4u);
                    }
                    bulk_commit();
                    issued = true;
                }
            } else if (a.mode != 1) {
                // token scales in halves of 32, all loads of a half before its stores (the
                // compiler may not move a load across a store it cannot prove disjoint)
                const bool valid = n_out < a.nvalid;
                float* op = a.out + (size_t)(it.row0 + col0) * a.ldo + (valid ? n_out : 0);
#pragma unroll
                for (int h0 = 0; h0 < kCW; h0 += 32) {
                    float sa[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) sa[i] = h0 + i < ncol ? __ldg(sap + h0 + i) : 0.f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (valid && h0 + i < ncol) *op = acc[h0 + i] * sa[i];
                        op += a.ldo;
                    }
                }
            } else {
                // SwiGLU: even tile rows hold gate channel f, odd rows the matching up
                // channel.  Per pair of tokens (i, i+1) the lanes of a pair swap one value:
                // the even lane finishes token i, the odd lane token i+1.
                const int f = it.nt * (kTileRows / 2) + (r >> 1);
                const int odd = r & 1;
                const bool valid = f < a.nvalid;
                const size_t o0 = (size_t)(it.row0 + col0 + odd) * a.ldo + f;
                float sa[kCW / 2];
#pragma unroll
                for (int i = 0; i < kCW; i += 2) sa[i / 2] = i + odd < ncol ? __ldg(sap + i + odd) : 0.f;
#pragma unroll
                for (int i = 0; i < kCW; i += 2) {
                    // even lane: own gate_i, needs the partner's up_i; odd lane: own up_{i+1},
                    // needs the partner's gate_{i+1}
                    const float send = odd ? acc[i] : acc[i + 1];
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                    const float g = (odd ? recv : acc[i]) * sa[i / 2];
                    const float u = (odd ? acc[i + 1] : recv) * sa[i / 2];
                    if (valid && i + odd < ncol) {
                        const size_t o = o0 + (size_t)i * a.ldo;
                        if (obf)
                            out16[o] = bf16_bits(silu_mul(g, u));
                        else
                            a.out[o] = silu_mul(g, u);
                    }
                }
            }
        }
        if (issued) bulk_wait_all();  // the output is complete before the CTA exits
    }

    __syncthreads();
    if (warp == C::kMmaWarp0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

#undef FULL_BAR
#undef EMPTY_BAR
#undef CONV_BAR
#undef AEMPTY_BAR
#undef DFULL_BAR
#undef DEMPTY_BAR
#undef SCFULL_BAR
#undef FINAL_BAR
#undef STAGE_BAR

using CfgLarge = Cfg<128, 6, 4, 3, 2, 1>;  // many tokens per expert
// the other group sizes (group 64's larger blocks leave room for 4 stages)
using CfgLarge64 = Cfg<128, 4, 4, 3, 2, 1, 64>;
using CfgLarge256 = Cfg<128, 6, 4, 3, 2, 1, 256>;

template <class C, bool kPartials>
cudaError_t launch_cfg(const GemmArgs& a, int num_ctas, cudaStream_t stream) {
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        // the register split only holds if the kernel really launches with
        // kRegLaunch registers per thread; otherwise setmaxnreg.inc could not be
        // satisfied, so refuse to launch
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, gemm_w4a8_kernel<C, kPartials>);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != C::kRegLaunch) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(gemm_w4a8_kernel<C, kPartials>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = 1;
    }
    return launch_pdl(gemm_w4a8_kernel<C, kPartials>, num_ctas, C::kThreads, C::kSmemBytes, stream, a);
}

}  // namespace

int gemm_tile_tokens(int avg_tokens_per_expert) { return avg_tokens_per_expert <= 16 ? 16 : CfgLarge::BN; }

cudaError_t launch_gemm(const GemmArgs& a, int tile_tokens, int num_ctas, cudaStream_t stream) {
    if (tile_tokens == 16) return launch_gemm_decode(a, num_ctas, stream);
    // the INT32-partials output (a parity check of the dense entry point) has its own instance
    if (a.group == 64)
        return a.partials != nullptr ? launch_cfg<CfgLarge64, true>(a, num_ctas, stream)
                                     : launch_cfg<CfgLarge64, false>(a, num_ctas, stream);
    if (a.group == 256)
        return a.partials != nullptr ? launch_cfg<CfgLarge256, true>(a, num_ctas, stream)
                                     : launch_cfg<CfgLarge256, false>(a, num_ctas, stream);
    if (a.partials != nullptr) return launch_cfg<CfgLarge, true>(a, num_ctas, stream);
    return launch_cfg<CfgLarge, false>(a, num_ctas, stream);
}

}  // namespace w4a8

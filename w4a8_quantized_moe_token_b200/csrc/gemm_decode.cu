// Grouped W4A8 GEMM for decode-shaped layers (at most 16 tokens per tile), sm_100a.
//
// Same method as gemm_w4a8.cu (INT4 group-128 weights x per-token INT8 tokens on
// tcgen05 kind::i8 MMAs, one exact INT32 partial per 128-wide K group, scales folded
// in fp32): «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» (pptc.cn) sections 2.1 and 3.2,
// the Kimi 2.7T MoE W4A8 article (hotelren.com 5173946) section 4.3.
//
// Decode streams every touched expert's weights once for a handful of tokens, so the
// kernel must run at HBM speed.  Every synchronisation between the roles (mbarrier
// wait / arrive, tcgen05 commit, tensor-memory store + wait) costs a few hundred
// cycles, which is as long as one 8.7 KB weight block takes to arrive at full
// bandwidth; so one pipeline step here carries 4 consecutive K groups of a tile
// (35 KB of weights, 16 MMAs), paying the synchronisation once per 4 groups.
//
// Roles (one persistent CTA per SM, 20 warps):
//   2 producer warps   : (alternate steps) one 1-D bulk copy of the step's weight blocks
//                        (contiguous in the packed layout) and one of its token rows
//                        (contiguous in the 16-row-block activation layout);
//   2 converter groups : (alternate steps) each thread expands one weight row's codes
//                        to unsigned INT8 (the raw 4-bit codes: a mask and a
//                        multiply-high per 8 codes), stores them to a tensor-memory A
//                        slot, publishes the row's scale and zero point, and sums each
//                        token's 128 INT8 codes per group (S, with dp4a);
//   2 MMA warps        : (both on every step, two groups each) per group 4 x
//                        tcgen05.mma.kind::i8 u8 x s8,
//                        M=128 weight rows, N=16 tokens, K=32, into the group's own
//                        INT32 accumulator (preloaded with 1.5 * 2^23, see below);
//   2 epilogue groups  : each reads the partials of two of the step's groups, removes
//                        the zero point exactly (P = sum a*c - zp * S) and folds
//                        acc += scale * P in fp32 (packed fp32x2); at the end of a tile
//                        group 1 passes its sums to group 0, which applies the token
//                        scale and stores.
// Each MMA warp first resets its groups' accumulators to the bit pattern 0x4B400000
// (1.5 * 2^23) with one bf16 MMA (mma_reset_acc); the INT8 MMAs add the partial
// (|P| < 2^22), so the bits read back as fp32 are exactly 1.5 * 2^23 + P, and one packed
// fp32 subtraction yields P without an int -> float conversion.  The epilogue only
// reads the accumulators.
//
// Other group sizes (the «Kimi 2.7 Moe» page, section 4.3, tried 64, 128 and 256): the
// pipeline still moves 128-wide K planes, but accumulators, scales, zero points and
// code sums S follow the groups -- two per plane for group 64 (2 MMAs each), one per
// two planes for group 256 (8 MMAs into one accumulator; |P| <= 256 * 128 * 15 stays
// below 2^22).  A second instance serves the W4A16 comparison (see DecCfg).
#include "w4a8_common.cuh"
#include "w4a8_internal.h"

namespace w4a8 {

namespace {

constexpr uint32_t kMagicBits = 0x4B400000u;  // 1.5 * 2^23 (what the reset MMA writes)
constexpr float kMagicF = 12582912.0f;

// Pipeline shape per operand kind and group size.  A step carries PPS 128-wide K
// planes (one packed weight block each) and the GQ quantisation groups they hold.
// W4A8, group 128: INT8 token rows (128 bytes per row and plane), 4 planes per step.
// Group 256: the same, 2 groups per step.  Group 64: 2 planes (4 groups) per step,
// whose accumulators take as many columns as 4 planes of group 128, and 6 stages.
// W4A16 (group 128): bf16 token rows (256 bytes per row and plane); a plane's
// converted weights take 64 tensor-memory columns instead of 32, so a step carries
// 2 planes and the rings are deeper (6 stages) to keep as many weight bytes in flight.
template <bool kBf16, int GRP>
struct DecCfg {
    static_assert(!kBf16 || GRP == 128, "W4A16 uses group 128");
    static constexpr int PPS = (kBf16 || GRP == 64) ? 2 : 4;  // K planes per pipeline step
    static constexpr int GQ = PPS * 128 / GRP;                // quantisation groups per step
    static constexpr int NS = (kBf16 || GRP == 64) ? 6 : 4;   // shared-memory stages
    static constexpr int NA = 2;                              // tensor-memory A slots
    static constexpr int ND = NS;                             // accumulators (GQ x BN columns each)
    // scale ring slots: the converters write step j's slot once the MMAs of step j - NA
    // are done, which only proves that the epilogue has loaded the accumulators of step
    // j - NA - ND -- it may still be reading that step's scales -- so the slot's previous
    // step must be older: NSC >= NA + ND + 1
    static constexpr int NSC = NS + NA + 1;
    static constexpr int kRowBytes = kBf16 ? 256 : 128;       // token row bytes per K plane
    static constexpr int kGCols = kBf16 ? 64 : 32;            // A columns per K plane
    static constexpr int kBlk = block_bytes_for(GRP);         // packed weight block
};

constexpr int BN = 16;    // tokens per tile (one 16-row block)
constexpr uint32_t kTmemCols = 512;

// warps: 0-7 converters (2 groups), 8-15 epilogue (2 groups), 16 producer 0, 17-18 MMA,
// 19 producer 1
constexpr int kThreads = 640;
constexpr int kEpiWarp0 = 8, kCtrlWarp0 = 16;
constexpr int kRegLaunch = 96;  // 65536 / 640, rounded down to the allocation unit
constexpr int kRegConv = 88, kRegCtrl = 48, kRegEpi = 128;
static_assert(128 * (2 * kRegConv + kRegCtrl + 2 * kRegEpi) <= kRegLaunch * kThreads, "register split");

template <bool kBf16, int GRP>
struct DecLayout {
    using C = DecCfg<kBf16, GRP>;
    static constexpr int PPS = C::PPS, GQ = C::GQ, NS = C::NS, NA = C::NA, ND = C::ND, NSC = C::NSC;
    static constexpr int kAStage = PPS * C::kBlk;            // weight blocks of one step
    static constexpr int kBStage = PPS * BN * C::kRowBytes;  // token rows of one step
    static constexpr int kACols = PPS * C::kGCols;
    static constexpr int kDCols = GQ * BN;
    static constexpr uint32_t kACol0 = 0;
    static constexpr uint32_t kDCol0 = NA * kACols;
    static_assert(kDCol0 + ND * kDCols <= kTmemCols, "tensor memory over-subscribed");
    static_assert(NSC >= NA + ND + 1, "scale ring too small");
    static_assert(NS % 2 == 0, "the two producers own the stages of one parity each");
    static_assert(GQ % 2 == 0, "the two MMA warps split the groups of a step");
    // one "MMA of step j done" barrier per j % NS serves the stage ring, the A slots and
    // the accumulators: their rings must step together
    static_assert(ND == NS && NS % NA == 0, "shared completion ring");
    // shared memory carve-up (offsets from a 1024-aligned base)
    static constexpr int kOffB = 0;
    static constexpr int kOffA = kOffB + NS * kBStage;
    static constexpr int kOffSc = kOffA + NS * kAStage;         // ring: fp32 scale       [NSC][GQ][128]
    static constexpr int kOffZp = kOffSc + NSC * GQ * 128 * 4;  // ring: fp32 zero point  [NSC][GQ][128]
    static constexpr int kOffS = kOffZp + NSC * GQ * 128 * 4;   // ring: token group sums [NSC][GQ][BN]
    static constexpr int kOffX = kOffS + NSC * GQ * BN * 4;     // epilogue exchange: [2][128][BN] fp32
    static constexpr int kOffReset = kOffX + 2 * 128 * BN * 4;   // the accumulator-reset operands
    static constexpr int kOffBar = kOffReset + 2 * kResetTileBytes;
    // full[NS] empty[NS] conv[NA] (unused: NA + ND) dempty[ND] side[NSC] final[2]
    // xfull[2] xempty[2]
    static constexpr int kNumBars = 2 * NS + 2 * NA + 2 * ND + NSC + 2 + 4;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory over-subscribed");
};

#define FULL_BAR(s) (bar0 + 8u * (uint32_t)(s))
#define EMPTY_BAR(s) (bar0 + 8u * (uint32_t)(NS + (s)))
#define CONV_BAR(x) (bar0 + 8u * (uint32_t)(2 * NS + (x)))
// (slots 2 NS + NA .. 2 NS + 2 NA + ND - 1 are unused: the MMA completion of a step is
// the EMPTY barrier of its stage)
#define DEMPTY_BAR(b) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + ND + (b)))
#define SIDE_BAR(i) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + 2 * ND + (i)))
#define FINAL_BAR(m) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + 2 * ND + NSC + (m)))
#define XFULL_BAR(p) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + 2 * ND + NSC + 2 + (p)))
#define XEMPTY_BAR(p) (bar0 + 8u * (uint32_t)(2 * NS + 2 * NA + 2 * ND + NSC + 4 + (p)))

struct Item {
    int e, nt, row0, nrows;
};

__device__ __forceinline__ Item decode_item(int u, const GemmArgs& a) {
    const int mt = u / a.NT;
    const int4 t = __ldg(a.mt_tab + mt);
    return Item{t.x, u - mt * a.NT, t.y, t.z};
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint32_t* err,
                                         long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t n = 1;; ++n) {
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

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint32_t* err, long long limit) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) {
            atomicOr(err, kErrTimeout);
            return;
        }
    }
}

// a packed pair of accumulators (low word: even token) += sc * P with the zero point
// removed, in fp32x2 arithmetic: acc2 += sc2 * ((x - m2) + nzp2 * s2), where x holds
// the bits of 1.5*2^23 + sum a*c, m2 = 1.5*2^23 twice, nzp2 = -zp twice and s2 the two
// tokens' code sums S; all values are integers below 2^24, so P = sum a*c - zp*S comes
// out exact
__device__ __forceinline__ void fold2_packed_zp(uint64_t& acc2, uint64_t sc2, uint64_t m2, uint64_t nzp2, uint64_t s2,
                                                uint32_t x0, uint32_t x1) {
    asm("{\n\t.reg .b64 x;\n\t"
        "mov.b64 x, {%1, %2};\n\t"
        "sub.rn.f32x2 x, x, %3;\n\t"
        "fma.rn.f32x2 x, %4, %5, x;\n\t"
        "fma.rn.f32x2 %0, %6, x, %0;\n\t}"
        : "+l"(acc2)
        : "r"(x0), "r"(x1), "l"(m2), "l"(nzp2), "l"(s2), "l"(sc2));
}

// a packed pair of fp32 accumulators += sc * (d0, d1) (the W4A16 fold)
__device__ __forceinline__ void fold2_f32(uint64_t& acc2, uint64_t sc2, uint32_t d0, uint32_t d1) {
    asm("{\n\t.reg .b64 x;\n\t"
        "mov.b64 x, {%1, %2};\n\t"
        "fma.rn.f32x2 %0, %3, x, %0;\n\t}"
        : "+l"(acc2)
        : "r"(d0), "r"(d1), "l"(sc2));
}

// two bf16 values (128 + code) minus the packed offset nz2 = -(128 + zp): exact
__device__ __forceinline__ uint32_t bf16x2_sub_offset(uint32_t v, uint32_t nz2) {
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(v), "r"(0x3F803F80u), "r"(nz2));
    return r;
}

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
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

template <bool kBf16, int GRP>
__global__ void __launch_bounds__(kThreads, 1) gemm_decode_kernel(const GemmArgs a) {
    using L = DecLayout<kBf16, GRP>;
    constexpr int PPS = L::PPS, GQ = L::GQ, NS = L::NS, NA = L::NA, ND = L::ND, NSC = L::NSC;
    constexpr int kAStage = L::kAStage, kBStage = L::kBStage, kACols = L::kACols, kDCols = L::kDCols;
    constexpr uint32_t kACol0 = L::kACol0, kDCol0 = L::kDCol0;
    constexpr int kRowBytes = DecCfg<kBf16, GRP>::kRowBytes, kGCols = DecCfg<kBf16, GRP>::kGCols;
    constexpr int kBlk = DecCfg<kBf16, GRP>::kBlk;
    constexpr int kOffA = L::kOffA, kOffB = L::kOffB, kOffSc = L::kOffSc, kOffZp = L::kOffZp, kOffS = L::kOffS;
    constexpr int kOffX = L::kOffX, kOffReset = L::kOffReset, kOffBar = L::kOffBar, kOffMisc = L::kOffMisc;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base_addr - raw_addr);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint8_t* smA = smem + kOffA;
    float* sc_ring = reinterpret_cast<float*>(smem + kOffSc);
    float* zp_ring = reinterpret_cast<float*>(smem + kOffZp);
    float* s_ring = reinterpret_cast<float*>(smem + kOffS);
    const uint8_t* smB = smem + kOffB;
    const uint32_t sA = base_addr + kOffA, sB = base_addr + kOffB;
    const uint32_t bar0 = base_addr + kOffBar;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(FULL_BAR(s), 1);
            mbar_init(EMPTY_BAR(s), 2);  // MMA of step j (j % NS == s) done: both MMA warps commit
        }
        for (int x = 0; x < NA; ++x) {
            mbar_init(CONV_BAR(x), 4);

        }
        for (int b = 0; b < ND; ++b) {
            mbar_init(DEMPTY_BAR(b), 8);  // the 8 epilogue warps
        }
        for (int i = 0; i < NSC; ++i) mbar_init(SIDE_BAR(i), 4);
        mbar_init(FINAL_BAR(0), 1);
        mbar_init(FINAL_BAR(1), 1);
        for (int p = 0; p < 2; ++p) {
            mbar_init(XFULL_BAR(p), 4);   // epilogue group 1 has written its sums
            mbar_init(XEMPTY_BAR(p), 4);  // epilogue group 0 has read them
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kCtrlWarp0 + 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    fill_reset_tiles(smem + kOffReset);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t sReset = base_addr + kOffReset;
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;

    // the set-up above (barriers, tensor memory, reset tiles) overlaps the previous
    // kernel's tail; from here on this kernel reads its results
    grid_dep_wait();
    const int total = a.NT * __ldg(a.n_mtiles);
    const int G = a.G;                 // 128-wide K planes (packed blocks) per tile
    const int Gq = G * kGroup / GRP;   // quantisation groups per row
    const int steps_per_item = (G + PPS - 1) / PPS;

    if (warp >= kCtrlWarp0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegCtrl));
        const int cw = warp - kCtrlWarp0;  // 0: producer 0, 1-2: MMA, 3: producer 1
        if (cw == 0 || cw == 3) {
            // ---------------- producers ----------------
            const int pi = cw == 0 ? 0 : 1;
            if (lane == 0) {
                uint32_t j = 0, last = 0;
                bool ok = true, rdy = false;  // rdy: an early test found this step's stage free
                for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                    const Item it = decode_item(u, a);
                    const uint8_t* wsrc = a.wblocks + (size_t)(it.e * a.NT + it.nt) * G * kBlk;
                    const int8_t* bsrc = a.act + (size_t)(it.row0 / BN) * a.act_rb_stride;
                    for (int t = 0; t < steps_per_item; ++t, ++j) {
                        if ((int)(j & 1u) != pi) continue;
                        last = j + 1;
                        const int g0 = t * PPS, ng = min(PPS, G - g0);
                        const int s = j % NS;
                        if (!rdy && !wait_bar(EMPTY_BAR(s), ((j / NS) & 1u) ^ 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                        rdy = mbar_test(EMPTY_BAR((j + 2) % NS), (((j + 2) / NS) & 1u) ^ 1u);
                        // test hook: leave the first step's stage empty, so that its consumers time out
                        if (j == 0 && blockIdx.x == 0 && (a.debug & kDebugSkipFirstCopy)) continue;
                        mbar_arrive_expect_tx(FULL_BAR(s), (uint32_t)ng * (kBlk + BN * kRowBytes));
                        bulk_g2s(sA + s * kAStage, wsrc + (size_t)g0 * kBlk, ng * kBlk, FULL_BAR(s));
                        bulk_g2s(sB + s * kBStage, bsrc + (size_t)g0 * BN * kRowBytes, ng * BN * kRowBytes, FULL_BAR(s));
                    }
                }
                for (uint32_t qq = (last > (uint32_t)NS ? last - NS : 0u); qq < last; ++qq)
                    if ((int)(qq & 1u) == pi) drain_wait(FULL_BAR(qq % NS), (qq / NS) & 1u, a.err, a.wait_limit);
            }
            __syncwarp();
        } else {
            // ---------------- MMA issuers ----------------
            // Both warps take every step, warp mi issuing the MMAs of groups 2mi and
            // 2mi+1: the issue rate of tcgen05.mma is a per-thread limit, so splitting a
            // step halves the time its A slot stays busy.  Each warp commits to the
            // step's barriers (two arrivals each), also when it had no group to issue.
            // the whole warp runs the loop (warp-uniform operands for tcgen05.mma); one
            // elected thread issues
            const int mi = cw - 1;
            {
                uint32_t j = 0;
                bool ok = true, conv_rdy = false, acc_rdy = false;  // early tests of this step's barriers
                // u8 codes x s8 tokens, or bf16 (code - zp) x bf16 tokens
                const uint32_t idesc = kBf16 ? idesc_bf16(128, BN) : idesc_i8(128, BN, false);
                for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
                    for (int t = 0; t < steps_per_item; ++t, ++j) {
                        const int nq = min(PPS, G - t * PPS) * kGroup / GRP;  // groups of this step
                        const int s = j % NS, x = j % NA, b = j % ND;
                        if (!conv_rdy && !wait_bar(CONV_BAR(x), (j / NA) & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                        if (!acc_rdy && !wait_bar(DEMPTY_BAR(b), ((j / ND) & 1u) ^ 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                        conv_rdy = mbar_test(CONV_BAR((j + 1) % NA), ((j + 1) / NA) & 1u);
                        acc_rdy = mbar_test(DEMPTY_BAR((j + 1) % ND), (((j + 1) / ND) & 1u) ^ 1u);
                        tc_fence_after();
                        if (elect_one()) {
                        // W4A8: reset this warp's groups' INT32 accumulators to the magic
                        // pattern, then add the partials.  W4A16: the first MMA of a group
                        // overwrites its fp32 accumulator.
                        if (!kBf16 && mi * (GQ / 2) < nq)
                            mma_reset_acc(tmem_base + kDCol0 + (uint32_t)(b * kDCols + mi * (GQ / 2) * BN), sReset,
                                          (GQ / 2) * BN);
#pragma unroll
                        for (int gh = 0; gh < GQ / 2; ++gh) {
                            const int gq = mi * (GQ / 2) + gh;
                            if (gq < nq) {
                                const uint32_t dt = tmem_base + kDCol0 + (uint32_t)(b * kDCols + gq * BN);
                                if constexpr (kBf16) {
                                    const uint32_t at = tmem_base + kACol0 + (uint32_t)(x * kACols + gq * kGCols);
                                    const uint32_t sb = sB + s * kBStage + gq * BN * kRowBytes;
                                    // K = 16 per MMA: steps 0-3 in the group's first 64-column
                                    // plane of token rows, 4-7 in the second
#pragma unroll
                                    for (int kk = 0; kk < 8; ++kk)
                                        mma_bf16_ts(dt, at + kk * 8,
                                                    smem_desc_sw128(sb + (kk >> 2) * BN * 128 + (kk & 3) * 32), idesc,
                                                    kk > 0 ? 1u : 0u);
                                } else {
                                    // the group's K range inside the step, 32 per MMA: plane
                                    // ko / 128 of the token rows, A columns ko / 4
#pragma unroll
                                    for (int kk = 0; kk < GRP / 32; ++kk) {
                                        const int ko = gq * GRP + kk * 32;
                                        mma_i8_ts(dt, tmem_base + kACol0 + (uint32_t)(x * kACols + ko / 4),
                                                  smem_desc_sw128(sB + s * kBStage + (ko >> 7) * BN * 128 + (ko & 127)),
                                                  idesc, 1u);
                                    }
                                }
                            }
                        }
                        // one commit tells the producer (stage s free), the converters (A
                        // slot free) and the epilogue (accumulators ready) at once
                        tc_commit(EMPTY_BAR(s));
                        }
                        __syncwarp();
                    }
                }
                if (elect_one()) tc_commit(FINAL_BAR(mi));
                __syncwarp();
                drain_wait(FINAL_BAR(mi), 0, a.err, a.wait_limit);
            }
            __syncwarp();
        }
    } else if (warp < kEpiWarp0) {
        // ---------------- converters ----------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegConv));
        const int cg = warp >> 2;
        const int r = threadIdx.x & 127;
        // group sums: GQ groups x BN tokens x SP parts; this thread adds part `part` of
        // token m's codes in group gs (with group 128: half a row, 64 bytes)
        constexpr int SP = 128 / (GQ * BN);
        static_assert(SP * GQ * BN == 128 && (SP == 2 || SP == 4), "group-sum split");
        const int gs = r / (BN * SP), m = (r / SP) % BN, part = r % SP;
        uint32_t m28;
        asm volatile("mov.u32 %0, 0x10000000;" : "=r"(m28));  // x * 2^28 >> 32 = x >> 4, on the FMA pipe
        const int nsteps = ((total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * steps_per_item;
        bool full_rdy = false;  // an early test of this step's stage
        for (int j = cg; j < nsteps; j += 2) {
            const int t = j % steps_per_item;
            const int ng = min(PPS, G - t * PPS);  // planes of this step
            const int nq = ng * kGroup / GRP;      // groups of this step
            const int s = j % NS, x = j % NA, slot = j % NSC;
            if (!full_rdy && !wait_bar(FULL_BAR(s), (j / NS) & 1u, abort_flag, a.err, a.wait_limit)) break;
            // A slot x was last read by the MMAs of step j - NA
            // (the MMAs of step j - NA can only finish after this group's previous step, so
            // there is no earlier point at which to test for them)
            if (j >= NA && !wait_bar(EMPTY_BAR((j - NA) % NS), ((j - NA) / NS) & 1u, abort_flag, a.err, a.wait_limit))
                break;
            full_rdy = mbar_test(FULL_BAR((j + 2) % NS), ((j + 2) / NS) & 1u);  // this group's next step
            for (int gq = 0; gq < ng; ++gq) {  // plane gq of the step
                const uint8_t* blk = smA + s * kAStage + gq * kBlk;
                uint4 w[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) w[c] = *reinterpret_cast<const uint4*>(blk + code_chunk_offset(r, c));
                // the scale and zero point of each group the plane starts (group 64: two,
                // the second 512 bytes after the first; group 256: one on even planes)
                const __half* shp = reinterpret_cast<const __half*>(blk + kScaleOff);
                const __half* zhp = reinterpret_cast<const __half*>(blk + kZpOff);
                if constexpr (GRP == 64) {
#pragma unroll
                    for (int sub = 0; sub < 2; ++sub) {
                        sc_ring[(slot * GQ + 2 * gq + sub) * 128 + r] = __half2float(shp[r + sub * 256]);
                        zp_ring[(slot * GQ + 2 * gq + sub) * 128 + r] = __half2float(zhp[r + sub * 256]);
                    }
                } else if constexpr (GRP == 256) {
                    if ((gq & 1) == 0) {
                        sc_ring[(slot * GQ + gq / 2) * 128 + r] = __half2float(shp[r]);
                        zp_ring[(slot * GQ + gq / 2) * 128 + r] = __half2float(zhp[r]);
                    }
                } else {
                    sc_ring[(slot * GQ + gq) * 128 + r] = __half2float(shp[r]);
                    if (!kBf16) zp_ring[(slot * GQ + gq) * 128 + r] = __half2float(zhp[r]);
                }
                if constexpr (kBf16) {
                    // (code - zp) as bf16, exactly: the byte permute puts each code under
                    // the bf16 bits 0x43, giving 128 + code, and one packed bf16 FMA
                    // subtracts 128 + zp (the zero point is an integer 0..15); each 32-bit
                    // tensor-memory column holds two consecutive K
                    const int zi = __half2int_rn(reinterpret_cast<const __half*>(blk + kZpOff)[r]);
                    const uint32_t nz2 = (0xC300u | (uint32_t)zi) * 0x10001u;  // -(128 + zp), twice
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {  // K 64hh .. 64hh + 63: chunks 2hh, 2hh + 1
                        uint32_t v[32];
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const uint4 wc = w[2 * hh + cc];
                            const uint32_t xw[4] = {wc.x, wc.y, wc.z, wc.w};
#pragma unroll
                            for (int qq = 0; qq < 4; ++qq) {
                                const int i = 4 * cc + qq;  // K = 64hh + 8i .. 64hh + 8i + 7
                                const uint32_t lo = xw[qq] & 0x0F0F0F0Fu;
                                const uint32_t hi = __umulhi(xw[qq], m28) & 0x0F0F0F0Fu;
                                v[4 * i] = bf16x2_sub_offset(__byte_perm(lo, 0x43434343u, 0x4140), nz2);
                                v[4 * i + 1] = bf16x2_sub_offset(__byte_perm(lo, 0x43434343u, 0x4342), nz2);
                                v[4 * i + 2] = bf16x2_sub_offset(__byte_perm(hi, 0x43434343u, 0x4140), nz2);
                                v[4 * i + 3] = bf16x2_sub_offset(__byte_perm(hi, 0x43434343u, 0x4342), nz2);
                            }
                        }
                        tmem_st32(tmem_base + lane_base + kACol0 + (uint32_t)(x * kACols + gq * kGCols + hh * 32), v);
                    }
                } else {
                    uint32_t v[32];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t xw[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            const int i = 4 * c + qq;  // word i holds K = 8i .. 8i+7 of the plane
                            v[2 * i] = xw[qq] & 0x0F0F0F0Fu;
                            v[2 * i + 1] = __umulhi(xw[qq], m28) & 0x0F0F0F0Fu;
                        }
                    }
                    tmem_st32(tmem_base + lane_base + kACol0 + (uint32_t)(x * kACols + gq * 32), v);
                }
            }
            if (GRP == 128 && !kBf16 && gs < nq) {
                // S[gs][m] = sum of token m's 128 INT8 codes of group gs (the swizzle only
                // permutes the 16-byte chunks inside the row, so the row sum is unaffected)
                const uint4* rowp = reinterpret_cast<const uint4*>(smB + s * kBStage + gs * BN * kRowBytes + m * 128 + part * 64);
                int sum = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 b4 = rowp[c];
                    sum = __dp4a((int)b4.x, 0x01010101, sum);
                    sum = __dp4a((int)b4.y, 0x01010101, sum);
                    sum = __dp4a((int)b4.z, 0x01010101, sum);
                    sum = __dp4a((int)b4.w, 0x01010101, sum);
                }
                sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                if (part == 0) s_ring[(slot * GQ + gs) * BN + m] = (float)sum;
            } else if (GRP != 128 && gs < nq) {
                // S[gs][m] over the group's K range, SP parts of GRP / SP codes each: logical
                // 16-byte chunk c of token row m sits at chunk position c ^ (m & 7)
                int sum = 0;
#pragma unroll
                for (int c = 0; c < GRP / SP / 16; ++c) {
                    const int k = gs * GRP + part * (GRP / SP) + 16 * c;  // K offset in the step
                    const uint4 b4 = *reinterpret_cast<const uint4*>(smB + s * kBStage + (k >> 7) * BN * 128 + m * 128 +
                                                                     ((((k & 127) >> 4) ^ (m & 7)) << 4));
                    sum = __dp4a((int)b4.x, 0x01010101, sum);
                    sum = __dp4a((int)b4.y, 0x01010101, sum);
                    sum = __dp4a((int)b4.z, 0x01010101, sum);
                    sum = __dp4a((int)b4.w, 0x01010101, sum);
                }
#pragma unroll
                for (int o = 1; o < SP; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (part == 0) s_ring[(slot * GQ + gs) * BN + m] = (float)sum;
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(CONV_BAR(x));
                mbar_arrive(SIDE_BAR(slot));
            }
        }
    } else {
        // ---------------- epilogue ----------------
        // Two groups of 4 warps: group eh folds the step's K groups 2eh and 2eh+1 into
        // its own sums; at the end of a tile group 1 hands its sums to group 0 through
        // shared memory (double-buffered, with bounded mbarrier waits), and group 0
        // adds them and stores the tile.
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegEpi));
        const int eh = (warp - kEpiWarp0) >> 2;
        const int r = q * 32 + lane;
        float* xbuf = reinterpret_cast<float*>(smem + kOffX);
        uint32_t j = 0;
        uint32_t nit = 0;  // tiles done by this CTA
        bool ok = true, acc_rdy = false, side_rdy = false;  // early tests of this step's barriers
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++nit) {
            const Item it = decode_item(u, a);
            // token i's scale in lane i, loaded now so that its latency hides behind the
            // tile's steps (group 0 stores the tile; W4A16 has no token scale)
            const float my_sa = (kBf16 || eh != 0 || lane >= BN) ? 1.f
                                : (lane < it.nrows ? __ldg(a.act_scale + it.row0 + lane) : 0.f);
            uint64_t acc2[BN / 2];  // token pairs, packed fp32x2
#pragma unroll
            for (int i = 0; i < BN / 2; ++i) acc2[i] = 0ull;
            const uint64_t m2 = splat2(kMagicF);
            const int n_out = (a.mode == 1) ? -1 : it.nt * kTileRows + r;
            for (int t = 0; t < steps_per_item; ++t, ++j) {
                const int nq = min(PPS, G - t * PPS) * kGroup / GRP;  // groups of this step
                const int b = j % ND, slot = j % NSC;
                if (!acc_rdy && !wait_bar(EMPTY_BAR(j % NS), (j / NS) & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                acc_rdy = mbar_test(EMPTY_BAR((j + 1) % NS), ((j + 1) / NS) & 1u);
                tc_fence_after();
                const uint32_t taddr = tmem_base + lane_base + kDCol0 + (uint32_t)(b * kDCols);
                uint32_t v[GQ / 2][BN];
#pragma unroll
                for (int gh = 0; gh < GQ / 2; ++gh)
                    if (eh * (GQ / 2) + gh < nq) tmem_ld16(taddr + (eh * (GQ / 2) + gh) * BN, v[gh]);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(DEMPTY_BAR(b));
                if (!side_rdy && !wait_bar(SIDE_BAR(slot), (j / NSC) & 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
                side_rdy = mbar_test(SIDE_BAR((j + 1) % NSC), ((j + 1) / NSC) & 1u);
#pragma unroll
                for (int gh = 0; gh < GQ / 2; ++gh) {
                    const int gq = eh * (GQ / 2) + gh;
                    if (kBf16 && gq < nq) {
                        // fp32 partials: acc += scale * D
                        const uint64_t sc2 = splat2(sc_ring[(slot * GQ + gq) * 128 + r]);
#pragma unroll
                        for (int i = 0; i < BN; i += 2) fold2_f32(acc2[i / 2], sc2, v[gh][i], v[gh][i + 1]);
                    } else if (!kBf16 && gq < nq) {
                        const float zpf = zp_ring[(slot * GQ + gq) * 128 + r];
                        const uint64_t sc2 = splat2(sc_ring[(slot * GQ + gq) * 128 + r]);
                        const uint64_t nzp2 = splat2(-zpf);
                        const float4* sp = reinterpret_cast<const float4*>(s_ring + (slot * GQ + gq) * BN);
                        float sg[BN];
#pragma unroll
                        for (int i = 0; i < BN / 4; ++i) {
                            const float4 f4 = sp[i];
                            sg[4 * i] = f4.x; sg[4 * i + 1] = f4.y; sg[4 * i + 2] = f4.z; sg[4 * i + 3] = f4.w;
                        }
                        if (a.partials != nullptr && n_out < a.nvalid) {
                            int32_t* pp = a.partials + ((size_t)it.row0 * a.nvalid + n_out) * Gq + t * GQ + gq;
                            const size_t pstride = (size_t)a.nvalid * Gq;
#pragma unroll
                            for (int i = 0; i < BN; ++i)
                                if (i < it.nrows)
                                    pp[i * pstride] = (int32_t)(v[gh][i] - kMagicBits) - (int32_t)zpf * (int32_t)sg[i];
                        }
#pragma unroll
                        for (int i = 0; i < BN; i += 2)
                            fold2_packed_zp(acc2[i / 2], sc2, m2, nzp2, pack2(sg[i], sg[i + 1]), v[gh][i], v[gh][i + 1]);
                    }
                }
            }
            if (!ok) break;
            const int xp = nit & 1;
            const uint32_t xpar = (nit >> 1) & 1u;
            float* xrow = xbuf + (xp * 128 + r) * BN;
            if (eh == 1) {
                // hand the sums to group 0 and go on with the next tile
                if (!wait_bar(XEMPTY_BAR(xp), xpar ^ 1u, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
#pragma unroll
                for (int i = 0; i < BN / 2; ++i) reinterpret_cast<uint64_t*>(xrow)[i] = acc2[i];
                __syncwarp();
                if (lane == 0) mbar_arrive(XFULL_BAR(xp));
                continue;
            }
            if (!wait_bar(XFULL_BAR(xp), xpar, abort_flag, a.err, a.wait_limit)) { ok = false; break; }
            float acc[BN];
#pragma unroll
            for (int i = 0; i < BN; i += 2) {
                float o0, o1;
                unpack2(reinterpret_cast<const uint64_t*>(xrow)[i / 2], o0, o1);
                unpack2(acc2[i / 2], acc[i], acc[i + 1]);
                acc[i] += o0;
                acc[i + 1] += o1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(XEMPTY_BAR(xp));

            float sa[BN];
#pragma unroll
            for (int i = 0; i < BN; ++i) sa[i] = kBf16 ? 1.f : __shfl_sync(0xffffffffu, my_sa, i);
            // mode 1 with out_bf16: h as bf16 (RNE of the fp32 result)
            const bool obf = a.out_bf16 != 0 && a.mode == 1;
            uint16_t* out16 = reinterpret_cast<uint16_t*>(a.out);
            if (a.mode != 1) {
                const bool valid = n_out < a.nvalid;
                float* op = a.out + (size_t)it.row0 * a.ldo + (valid ? n_out : 0);
#pragma unroll
                for (int i = 0; i < BN; ++i) {
                    if (valid && i < it.nrows) *op = acc[i] * sa[i];
                    op += a.ldo;
                }
            } else {
                // SwiGLU: even tile rows hold gate channel f, odd rows the matching up
                // channel.  Per pair of tokens (i, i+1) the lanes of a pair swap one value:
                // the even lane finishes token i, the odd lane token i+1.
                const int f = it.nt * (kTileRows / 2) + (r >> 1);
                const int odd = r & 1;
                const bool valid = f < a.nvalid;
                const size_t o0 = (size_t)(it.row0 + odd) * a.ldo + f;
#pragma unroll
                for (int i = 0; i < BN; i += 2) {
                    // even lane: own gate_i, needs the partner's up_i; odd lane: own up_{i+1},
                    // needs the partner's gate_{i+1}
                    const float send = odd ? acc[i] : acc[i + 1];
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                    const float si = odd ? sa[i + 1] : sa[i];
                    const float g = (odd ? recv : acc[i]) * si;
                    const float u = (odd ? acc[i + 1] : recv) * si;
                    if constexpr (kBf16) {
                        // h rounded to bf16, straight into the down projection's token rows
                        if (valid && i + odd < it.nrows)
                            *reinterpret_cast<__nv_bfloat16*>(a.out16 + act16_offset(it.row0 + i + odd, f, a.out16_G, BN)) =
                                __float2bfloat16_rn(silu_mul(g, u));
                    } else if (valid && i + odd < it.nrows) {
                        if (obf)
                            out16[o0 + (size_t)i * a.ldo] = bf16_bits(silu_mul(g, u));
                        else
                            a.out[o0 + (size_t)i * a.ldo] = silu_mul(g, u);
                    }
                }
            }
        }
    }

    __syncthreads();
    if (warp == kCtrlWarp0 + 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

#undef FULL_BAR
#undef EMPTY_BAR
#undef CONV_BAR
#undef DEMPTY_BAR
#undef SIDE_BAR
#undef FINAL_BAR
#undef XFULL_BAR
#undef XEMPTY_BAR

}  // namespace

int gemm_decode_tile_tokens() { return BN; }

namespace {
template <bool kBf16, int GRP>
cudaError_t launch_decode(const GemmArgs& a, int num_ctas, cudaStream_t stream) {
    constexpr int kSmem = DecLayout<kBf16, GRP>::kSmemBytes;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        // the register split assumes kRegLaunch registers per thread at launch
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, gemm_decode_kernel<kBf16, GRP>);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != kRegLaunch) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(gemm_decode_kernel<kBf16, GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = 1;
    }
    return launch_pdl(gemm_decode_kernel<kBf16, GRP>, num_ctas, kThreads, kSmem, stream, a);
}
}  // namespace

cudaError_t launch_gemm_decode(const GemmArgs& a, int num_ctas, cudaStream_t stream) {
    if (a.group == 64) return launch_decode<false, 64>(a, num_ctas, stream);
    if (a.group == 256) return launch_decode<false, 256>(a, num_ctas, stream);
    return launch_decode<false, 128>(a, num_ctas, stream);
}

cudaError_t launch_gemm_w4a16(const GemmArgs& a, int num_ctas, cudaStream_t stream) {
    if (a.partials != nullptr || (a.mode == 1 && a.out16 == nullptr) || (a.group != 0 && a.group != 128))
        return cudaErrorInvalidValue;
    return launch_decode<true, 128>(a, num_ctas, stream);
}

}  // namespace w4a8

// Shared device-side definitions of libw4a8: layout constants, the tiled
// layouts' index arithmetic, and inline-PTX wrappers for mbarriers, bulk copies
// and the sm_100a tensor-core (tcgen05) instructions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace w4a8 {

// ---------------------------------------------------------------------------
// Format constants
// ---------------------------------------------------------------------------
constexpr int kGroup = 128;           // weights per quantisation group along K
constexpr int kTileRows = 128;        // weight rows per packed tile (= MMA M)
constexpr int kCodeBytes = kTileRows * kGroup / 2;   // 8192: 4-bit codes of one block
constexpr int kScaleOff = kCodeBytes;                // fp16 scales of the 128 rows
constexpr int kZpOff = kCodeBytes + kTileRows * 2;   // fp16 zero points of the 128 rows
constexpr int kBlockBytes = kZpOff + kTileRows * 2;  // 8704 bytes per (tile, group) block
constexpr int kHeaderBytes = 256;
// Other group sizes along K (64 and 256; 128 is the default).  The packed blocks stay
// one per 128-wide K plane (kGroup above is that plane): 8192 bytes of codes, then per
// row the fp16 scale and zero point of each group the plane holds.  Group 64: two
// groups, the second pair after the first (block of 9216 bytes); group 256: the plane
// is half of a group whose scale and zero point both of its planes carry (8704 bytes),
// so that every block is self-contained.  K is padded to a whole number of groups and
// of planes.
__host__ __device__ constexpr int block_bytes_for(int group) { return group == 64 ? kBlockBytes + 512 : kBlockBytes; }
__host__ __device__ constexpr int k_padded_for(int K, int group) {
    return (K + (group > 128 ? group : 128) - 1) / (group > 128 ? group : 128) * (group > 128 ? group : 128);
}
constexpr uint32_t kPackMagic = 0x38413457u;         // "W4A8"
constexpr int kRowPad = 16;           // each expert's row segment is padded to 16 rows
constexpr int kMaxExperts = 1024;

// device error word bits
constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrBadExpert = 2u;

// how long a bounded mbarrier wait may last before it gives up (clock cycles, ~2 s)
constexpr long long kWaitLimitCycles = 4000000000ll;
// debug word bit: CTA 0's producer issues no copy for its first pipeline step, so the
// consumers' bounded waits run out (a test of the failure-detection path)
constexpr uint32_t kDebugSkipFirstCopy = 1u;

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline int round_up(int a, int b) { return ceil_div(a, b) * b; }

// Byte offset of (row r, column k) inside one 128-column plane of the tiled INT8
// activation layout: 128 bytes per row, 16-byte chunk c of row r stored at chunk
// position c ^ (r & 7).  This is the 128-byte-swizzled K-major arrangement that the
// tensor-core shared-memory descriptor (SWIZZLE_128B) reads, so a run of rows can
// be moved into shared memory with one plain bulk copy.
__host__ __device__ inline uint32_t act_tiled_offset(int r, int k) {
    return (uint32_t)r * 128u + ((uint32_t)(((k >> 4) ^ (r & 7)) & 7) << 4) + (uint32_t)(k & 15);
}

// Byte offset of (row r, column k) in the whole tiled activation buffer of G planes:
// rows are grouped in blocks of RB rows, each block stores its G planes one after the
// other ([rows/RB][G][RB][128]).  RB = 16 lets one copy fetch several K groups of a
// 16-row tile; RB = all rows gives plain planes [G][rows][128].
__host__ __device__ inline size_t act_offset(int r, int k, int G, int RB) {
    return ((size_t)(r / RB) * G + (size_t)(k >> 7)) * (size_t)RB * 128u + act_tiled_offset(r % RB, k & 127);
}

// Byte offset of (row r, column k) in a tiled bf16 token-row buffer: per block of RB
// rows and 128-wide K group, two planes of 64 columns (128 bytes per row), each in the
// swizzled arrangement of act_tiled_offset ([rows/RB][G][2][RB][128 bytes]).  A
// 16-bit tensor-core step (K = 16, 32 bytes) then reads inside one plane.
__host__ __device__ inline size_t act16_offset(int r, int k, int G, int RB) {
    return (((size_t)(r / RB) * G + (size_t)(k >> 7)) * 2u + (size_t)((k >> 6) & 1)) * (size_t)RB * 128u +
           act_tiled_offset(r % RB, (k & 63) * 2);
}

// Byte offset of 16-byte chunk c (K columns 32c..32c+31 of the group) of tiled row r
// inside a code block: rows of 64 bytes, chunk swizzled with (r >> 1) & 3 so that
// eight consecutive rows reading the same chunk hit distinct shared-memory banks.
__host__ __device__ inline uint32_t code_chunk_offset(int r, int c) {
    return (uint32_t)r * 64u + ((uint32_t)((c ^ (r >> 1)) & 3) << 4);
}

// G counts 128-wide planes (blocks per tile), `group` the weights per scale along K
struct PackHeader {
    uint32_t magic, version, layout, E, N, K, Kp, G, NT, rows_per_tile, block_bytes, group;
};

// ---------------------------------------------------------------------------
// small PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// Test an mbarrier phase.  A thread whose phase is not complete yet is suspended
// by the hardware until it completes or about `suspend_ns` pass, so waiting warps
// do not spin on the issue slots that working warps on the same SM need.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity, uint32_t suspend_ns = 20000u) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(suspend_ns)
        : "memory");
    return ok != 0;
}

// Non-blocking test of an mbarrier phase (acquire semantics when it reports completion).
// The result arrives with a latency of a few hundred cycles, so the pipelines test the
// barrier of their next step early, while they work on the current one, and only fall
// back to a blocking wait when that test found the phase incomplete.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// one thread of the (converged) warp, the same one every time
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// 1-D bulk copy global -> shared (no tensor map, no multicast); completion is
// reported to mbarrier `bar` as transaction bytes.  dst, src 16-B aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// 1-D bulk copy shared -> global (no tensor map), tracked per issuing thread in a
// bulk group.  dst, src 16-B aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_s2g(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until this thread's committed bulk copies have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// wait until this thread's committed bulk copies are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// make this thread's generic-proxy shared-memory writes visible to the async proxy
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- tcgen05 (5th-generation tensor core, tensor memory) ----
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
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// arrive (once) on `bar` when every tcgen05 op issued so far by this thread completes
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, s8 x s8 -> s32; M = 128, N from idesc, K = 32
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> f32; M = 128, N from idesc, K = 16
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 x bf16 -> f32; M = 128, N from idesc, K = 16
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor for kind::f16 with bf16 A and B and an f32 D (bits 4-5 = 1,
// bits 7-9 = 1, bits 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor without swizzling: 8-row x 16-byte core matrices,
// `lbo` bytes apart along K and `sbo` bytes apart along M / N, descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_noswz(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    return d;
}

// Accumulator reset by the tensor core.  The W4A8 GEMMs keep every INT32 accumulator
// at the bit pattern 0x4B400000 (the fp32 value 1.5 * 2^23) before a K group's INT8
// MMAs add the partial P on top, so that the bits read back as fp32 are exactly
// 1.5 * 2^23 + P.  One bf16 MMA with accumulate = 0 writes that pattern into a whole
// accumulator: A is all ones, B holds 1.5 * 2^19 everywhere, and the K = 16 products sum
// to 16 * 1.5 * 2^19 = 1.5 * 2^23 exactly (every partial sum is a multiple of 1.5 * 2^19
// below 2^24).  Both operands are uniform tiles, so the result does not depend on how
// the descriptor's strides walk them; kResetTileBytes of each cover every address a
// 128 x 16 operand with 128-byte strides can reach.
constexpr int kResetTileBytes = 2304;
constexpr uint32_t kResetOneBits = 0x3F80u;   // bf16 1.0
constexpr uint32_t kResetBBits = 0x4940u;     // bf16 1.5 * 2^19
constexpr uint32_t kResetStride = 128u;

// fill the two reset operand tiles (A at `a`, B at `a + kResetTileBytes`); every thread
// of the block takes part, then the writes are made visible to the tensor core
__device__ __forceinline__ void fill_reset_tiles(uint8_t* a) {
    uint32_t* w = reinterpret_cast<uint32_t*>(a);
    for (int i = threadIdx.x; i < 2 * kResetTileBytes / 4; i += blockDim.x) {
        const uint32_t h = i < kResetTileBytes / 4 ? kResetOneBits : kResetBBits;
        w[i] = h | (h << 16);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// the reset MMA for an accumulator of n columns (n a multiple of 16, 16..256) at d_tmem
__device__ __forceinline__ void mma_reset_acc(uint32_t d_tmem, uint32_t reset_smem, int n) {
    mma_bf16_ss(d_tmem, smem_desc_noswz(reset_smem, kResetStride, kResetStride),
                smem_desc_noswz(reset_smem + kResetTileBytes, kResetStride, kResetStride), idesc_bf16(128, n), 0u);
}

// Instruction descriptor for kind::i8: D = s32 (bits 4-5 = 2), A = s8 or u8 (bits 7-9),
// B = s8 (bits 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
// a_signed = false selects unsigned 8-bit A (bits 7-9 = 0).
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N, bool a_signed = true) {
    return (2u << 4) | ((a_signed ? 1u : 0u) << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 bytes,
// 8-row groups 1024 bytes apart (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;            // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024u >> 4) << 32;  // stride byte offset
    d |= (uint64_t)1u << 46;            // version
    d |= (uint64_t)2u << 61;            // SWIZZLE_128B
    return d;
}

// 32 lanes x 32 bits, 16 consecutive columns per thread
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 32 consecutive columns per thread
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

// 32 lanes x 32 bits, 32 consecutive columns per thread
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier over `nthreads` threads (whole warps) that also ORs a predicate across
// them: every participant gets the same result.  A group of warps uses it to follow
// one leader warp that did the group's mbarrier waits: mbarrier waits are costly (each
// warp-level wait occupies the SM's barrier unit for tens of cycles, even on a phase
// that has completed), a named barrier is not.  The leader passes "my wait failed"
// as the predicate, so the whole group leaves together and no warp is left waiting
// at a barrier that the others skipped.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %3, 0;\n\t"
        "bar.red.or.pred p, %1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(id), "r"(nthreads), "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  The kernels of a forward pass are launched with
// launch_pdl(): each may start (barrier and tensor-memory set-up) while the previous
// kernel on the stream drains, and calls grid_dep_wait() before it touches global
// memory -- reads of the previous kernels' results and every write.  Launched
// without the attribute, the wait returns at once.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// bf16 bit pattern of an fp32 value, rounded to nearest even
__device__ __forceinline__ uint16_t bf16_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// ---------------------------------------------------------------------------
// quantisation arithmetic (IEEE fp32, round half to even, no contraction)
// ---------------------------------------------------------------------------
// symmetric INT8 of one value with scale s > 0
__device__ __forceinline__ int quant_i8(float x, float s) {
    float r = rintf(__fdiv_rn(x, s));
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    return (int)r;
}

// The same code, bit for bit, with a multiply by inv = RN(1/s) in the common case.
// With v = x/s exact, d = RN(v) (what quant_i8 rounds) and y = RN(x * inv):
// |y - d| <= 3 * 2^-24 * |v| < 2.3e-5 for |v| < 128, so rint(y) and rint(d) can only
// differ when y is that close to a half-integer (a rounding boundary, including the
// ties that rint(d) sends to even); those values, and a y that is not finite, take
// the exact division.  Beyond |v| = 128 both saturate to +-127.
__device__ __forceinline__ int quant_i8_fast(float x, float s, float inv) {
    const float y = __fmul_rn(x, inv);
    const float f = __fsub_rn(y, floorf(y));
    if (!(fabsf(y) <= 1.0e30f) || fabsf(__fsub_rn(f, 0.5f)) <= 6.103515625e-05f) return quant_i8(x, s);
    float r = rintf(y);
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    return (int)r;
}

}  // namespace w4a8

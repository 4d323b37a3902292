// C ABI of libw4a8.so: argument validation, workspace carve-up and the launch
// sequence of the W4A8 MoE expert FFN.  Declarations and the contract of every
// entry point are in include/w4a8.h.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "../../include/w4a8.h"
#include "w4a8_common.cuh"
#include "w4a8_internal.h"

#define W4A8_EXPORT extern "C" __attribute__((visibility("default")))

namespace w4a8 {
namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count() {
    static int counts[64] = {0};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (counts[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

// Row capacity of the expert-grouped layout: every non-empty expert's segment is
// padded up to a multiple of 16 rows.
int rows_capacity(int T, int E, int k) {
    const long long nslots = (long long)T * k;
    if (nslots <= 0) return 0;
    const long long pad = (long long)(kRowPad - 1) * (nslots < E ? nslots : E);
    return (int)(((nslots + pad + kRowPad - 1) / kRowPad) * kRowPad);
}

// Workspace of w4a8_moe_forward: regions in the order of the enum below.
enum Region {
    R_ERR, R_CHIST, R_COUNTS, R_OFFS, R_POFFS, R_MTSTART, R_MTTAB, R_PERM, R_INV, R_ROWSRC,
    R_ACT1, R_S1, R_H, R_ACT2, R_S2, R_Y2,
    R_XIN, R_IDSIN, R_WIN, R_OUT, R_LOGITS,  // host-buffer variants only
    R_COUNT
};

struct MoeLayout {
    size_t off[R_COUNT + 1];
    size_t bytes[R_COUNT];
    int nslots, nchunk, R, Hp, Fp, G1, G2;
};

// w4a16: the W4A16 layer's workspace, in which ACT1 and ACT2 hold bf16 token rows
// (act16_offset, 16-row blocks) and the INT8 scales and the fp32 h are absent
// group: weights per scale of the packed weights (64, 128, 256): the token rows are
// padded to whole groups
bool moe_layout(int T, int E, int k, int H, int F, bool host_io, MoeLayout* L, bool w4a16 = false, int group = 128) {
    if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > 32 || k > E || H < 1 || F < 1) return false;
    if ((long long)T * k >= (1ll << 31)) return false;
    if (group != 64 && group != 128 && group != 256) return false;
    L->nslots = T * k;
    L->nchunk = ceil_div(L->nslots, kPermChunk);
    L->R = rows_capacity(T, E, k);
    L->Hp = k_padded_for(H, group);
    L->Fp = k_padded_for(F, group);
    L->G1 = L->Hp / kGroup;
    L->G2 = L->Fp / kGroup;
    const size_t R = (size_t)L->R;
    size_t* b = L->bytes;
    b[R_ERR] = 16;
    b[R_CHIST] = (size_t)L->nchunk * E * 4;
    b[R_COUNTS] = (size_t)E * 4;
    b[R_OFFS] = (size_t)(E + 1) * 4;
    b[R_POFFS] = (size_t)(E + 1) * 4;
    b[R_MTSTART] = (size_t)(E + 1) * 4;
    b[R_MTTAB] = (size_t)mt_tab_capacity(L->nslots, E) * 16;
    b[R_PERM] = (size_t)L->nslots * 4;
    b[R_INV] = (size_t)L->nslots * 4;
    b[R_ROWSRC] = R * 4;
    const size_t row_bytes = w4a16 ? 256 : 128;  // token row bytes per K group
    b[R_ACT1] = (size_t)L->G1 * R * row_bytes;
    b[R_S1] = w4a16 ? 0 : R * 4;
    b[R_H] = w4a16 ? 0 : R * (size_t)L->Fp * 2;  // bf16
    b[R_ACT2] = (size_t)L->G2 * R * row_bytes;
    b[R_S2] = w4a16 ? 0 : R * 4;
    b[R_Y2] = R * (size_t)H * 4;
    b[R_XIN] = host_io ? (size_t)T * H * 2 : 0;
    b[R_IDSIN] = host_io ? (size_t)L->nslots * 4 : 0;
    b[R_WIN] = host_io ? (size_t)L->nslots * 4 : 0;
    b[R_OUT] = host_io ? (size_t)T * H * 2 : 0;
    b[R_LOGITS] = host_io ? (size_t)T * E * 2 : 0;
    size_t o = 0;
    for (int r = 0; r < R_COUNT; ++r) {
        L->off[r] = o;
        o += align_up(b[r]);
    }
    L->off[R_COUNT] = o;
    return true;
}

int to_status(cudaError_t e) { return e == cudaSuccess ? W4A8_OK : W4A8_ECUDA; }

thread_local DebugInject g_debug;

// the test hook of w4a8_debug_inject, copied into every GEMM launch
void apply_debug(GemmArgs& a) {
    a.wait_limit = g_debug.wait_limit > 0 ? g_debug.wait_limit : kWaitLimitCycles;
    a.debug = g_debug.flags;
}

// Optional per-kernel event timing (w4a8_profile_start / w4a8_profile_stop),
// kept per host thread.
struct Profiler {
    bool on = false;
    struct Rec {
        int kind;
        cudaEvent_t a, b;
    };
    std::vector<cudaEvent_t> pool;
    std::vector<Rec> recs;
    int launches[W4A8_KERNEL_KINDS] = {0};
};
thread_local Profiler g_prof;

cudaEvent_t prof_event() {
    if (!g_prof.pool.empty()) {
        cudaEvent_t e = g_prof.pool.back();
        g_prof.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// RAII: records an event pair around the kernels launched in its scope
struct ProfScope {
    int kind, nlaunch;
    cudaStream_t st;
    cudaEvent_t a = nullptr;
    ProfScope(int k, int n, cudaStream_t s) : kind(k), nlaunch(n), st(s) {
        if (g_prof.on && (a = prof_event()) != nullptr) cudaEventRecord(a, st);
    }
    ~ProfScope() {
        if (a == nullptr) return;
        cudaEvent_t b = prof_event();
        if (b == nullptr) return;
        cudaEventRecord(b, st);
        g_prof.recs.push_back({kind, a, b});
        g_prof.launches[kind] += nlaunch;
    }
};

#define W4A8_TRY(expr)                                  \
    do {                                                \
        cudaError_t _e = (expr);                        \
        if (_e != cudaSuccess) return W4A8_ECUDA;       \
    } while (0)

int packed_tiles(int N, int layout) {
    return layout == W4A8_LAYOUT_GATEUP ? ceil_div(N / 2, kTileRows / 2) : ceil_div(N, kTileRows);
}

template <typename T>
T* at(void* base, const MoeLayout& L, Region r) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + L.off[r]);
}

// the forward on device buffers, workspace already validated
int moe_forward_impl(const void* packed_up, const void* packed_down, int E, int H, int F, const uint16_t* x, int T,
                     const int32_t* ids, const float* w, int k, uint16_t* out, void* ws, const MoeLayout& L,
                     cudaStream_t st, int group = 128) {
    uint32_t* err = at<uint32_t>(ws, L, R_ERR);
    W4A8_TRY(cudaMemsetAsync(err, 0, 16, st));
    if (T == 0) return W4A8_OK;
    int* counts = at<int>(ws, L, R_COUNTS);
    int* offs = at<int>(ws, L, R_OFFS);
    int* poffs = at<int>(ws, L, R_POFFS);
    int* mtstart = at<int>(ws, L, R_MTSTART);
    int4* mt_tab = at<int4>(ws, L, R_MTTAB);
    int* row_src = at<int>(ws, L, R_ROWSRC);
    int* inv = at<int>(ws, L, R_INV);
    float* s1 = at<float>(ws, L, R_S1);
    float* s2 = at<float>(ws, L, R_S2);
    uint16_t* h = at<uint16_t>(ws, L, R_H);
    float* y2 = at<float>(ws, L, R_Y2);
    int8_t* act1 = at<int8_t>(ws, L, R_ACT1);
    int8_t* act2 = at<int8_t>(ws, L, R_ACT2);
    // tokens per GEMM tile from the mean tokens per expert (decode-like layers use the
    // decode kernel with 16-token tiles and 16-row blocks of token rows)
    const int tile = gemm_tile_tokens(L.nslots / E);
    const int rb = act_block_rows(tile, L.R);

    {
        ProfScope p(W4A8_KERNEL_PERM, perm_launch_count(L.nslots), st);
        W4A8_TRY(launch_perm(ids, L.nslots, E, tile, at<int>(ws, L, R_CHIST), L.nchunk, counts, offs, poffs, mtstart,
                             mt_tab, at<int>(ws, L, R_PERM), inv, row_src, err, st));
    }
    {
        ProfScope p(W4A8_KERNEL_ACT_QUANT, 1, st);
        W4A8_TRY(launch_act_scatter(x, T, H, L.Hp, k, inv, offs, poffs, E, rb, act1, s1, st));
    }

    GemmArgs up{};
    up.wblocks = static_cast<const uint8_t*>(packed_up) + kHeaderBytes;
    up.NT = packed_tiles(2 * F, W4A8_LAYOUT_GATEUP);
    up.G = L.G1;
    up.act = act1;
    up.act_plane = (size_t)rb * 128;
    up.act_rb_stride = (size_t)L.G1 * rb * 128;
    up.act_scale = s1;
    up.mt_tab = mt_tab;
    up.n_mtiles = mtstart + E;
    up.mode = 1;
    up.out = reinterpret_cast<float*>(h);
    up.out_bf16 = 1;
    up.ldo = L.Fp;
    up.nvalid = F;
    up.partials = nullptr;
    up.err = err;
    up.group = group;
    apply_debug(up);
    {
        ProfScope p(W4A8_KERNEL_GEMM_UP, 1, st);
        W4A8_TRY(launch_gemm(up, tile, sm_count(), st));
    }
    {
        ProfScope p(W4A8_KERNEL_REQUANT, 1, st);
        W4A8_TRY(launch_requant(h, L.Fp, F, L.Fp, row_src, poffs, E, L.R, rb, act2, s2, st));
    }

    GemmArgs dn = up;
    dn.wblocks = static_cast<const uint8_t*>(packed_down) + kHeaderBytes;
    dn.NT = packed_tiles(H, W4A8_LAYOUT_PLAIN);
    dn.G = L.G2;
    dn.act = act2;
    dn.act_rb_stride = (size_t)L.G2 * rb * 128;
    dn.act_scale = s2;
    dn.mode = 2;
    dn.out = y2;  // fp32
    dn.out_bf16 = 0;
    dn.ldo = H;
    dn.nvalid = H;
    {
        ProfScope p(W4A8_KERNEL_GEMM_DOWN, 1, st);
        W4A8_TRY(launch_gemm(dn, tile, sm_count(), st));
    }
    {
        ProfScope p(W4A8_KERNEL_COMBINE, 1, st);
        W4A8_TRY(launch_combine(y2, H, inv, w, T, k, out, st));
    }
    return W4A8_OK;
}

// The W4A16 comparison layer on the same packed weights: the same routing,
// permutation and combine, 16-bit token rows into both projections (16-token tiles of
// the decode-shaped kernel), h rounded to bf16 between them.
int moe_forward_w4a16_impl(const void* packed_up, const void* packed_down, int E, int H, int F, const uint16_t* x,
                           int T, const int32_t* ids, const float* w, int k, uint16_t* out, void* ws,
                           const MoeLayout& L, cudaStream_t st) {
    uint32_t* err = at<uint32_t>(ws, L, R_ERR);
    W4A8_TRY(cudaMemsetAsync(err, 0, 16, st));
    if (T == 0) return W4A8_OK;
    int* mtstart = at<int>(ws, L, R_MTSTART);
    int4* mt_tab = at<int4>(ws, L, R_MTTAB);
    int* inv = at<int>(ws, L, R_INV);
    float* y2 = at<float>(ws, L, R_Y2);
    uint8_t* x16 = at<uint8_t>(ws, L, R_ACT1);
    uint8_t* h16 = at<uint8_t>(ws, L, R_ACT2);
    constexpr int tile = 16;
    {
        ProfScope p(W4A8_KERNEL_PERM, perm_launch_count(L.nslots), st);
        W4A8_TRY(launch_perm(ids, L.nslots, E, tile, at<int>(ws, L, R_CHIST), L.nchunk, at<int>(ws, L, R_COUNTS),
                             at<int>(ws, L, R_OFFS), at<int>(ws, L, R_POFFS), mtstart, mt_tab, at<int>(ws, L, R_PERM),
                             inv, at<int>(ws, L, R_ROWSRC), err, st));
    }
    {
        ProfScope p(W4A8_KERNEL_ACT_QUANT, 1, st);
        W4A8_TRY(launch_act_gather_bf16(x, T, H, k, inv, x16, h16, F, st));
    }
    GemmArgs up{};
    up.wblocks = static_cast<const uint8_t*>(packed_up) + kHeaderBytes;
    up.NT = packed_tiles(2 * F, W4A8_LAYOUT_GATEUP);
    up.G = L.G1;
    up.act = reinterpret_cast<const int8_t*>(x16);
    up.act_rb_stride = (size_t)L.G1 * tile * 256;
    up.mt_tab = mt_tab;
    up.n_mtiles = mtstart + E;
    up.mode = 1;
    up.nvalid = F;
    up.out16 = h16;
    up.out16_G = L.G2;
    up.err = err;
    apply_debug(up);
    {
        ProfScope p(W4A8_KERNEL_GEMM_UP, 1, st);
        W4A8_TRY(launch_gemm_w4a16(up, sm_count(), st));
    }
    GemmArgs dn = up;
    dn.wblocks = static_cast<const uint8_t*>(packed_down) + kHeaderBytes;
    dn.NT = packed_tiles(H, W4A8_LAYOUT_PLAIN);
    dn.G = L.G2;
    dn.act = reinterpret_cast<const int8_t*>(h16);
    dn.act_rb_stride = (size_t)L.G2 * tile * 256;
    dn.mode = 2;
    dn.out = y2;  // fp32
    dn.ldo = H;
    dn.nvalid = H;
    dn.out16 = nullptr;
    {
        ProfScope p(W4A8_KERNEL_GEMM_DOWN, 1, st);
        W4A8_TRY(launch_gemm_w4a16(dn, sm_count(), st));
    }
    {
        ProfScope p(W4A8_KERNEL_COMBINE, 1, st);
        W4A8_TRY(launch_combine(y2, H, inv, w, T, k, out, st));
    }
    return W4A8_OK;
}

int check_moe_args(const void* packed_up, const void* packed_down, int E, int H, int F, int T, int k, void* ws,
                   size_t ws_bytes, bool host_io, MoeLayout* L, bool w4a16 = false, int group = 128) {
    if (!moe_layout(T, E, k, H, F, host_io, L, w4a16, group)) {
        if (E > kMaxExperts || k > 32) return W4A8_EUNSUPPORTED;
        return W4A8_EINVAL;
    }
    if (packed_up == nullptr || packed_down == nullptr || ws == nullptr) return W4A8_EINVAL;
    if (!aligned(packed_up, kAlign) || !aligned(packed_down, kAlign) || !aligned(ws, kAlign)) return W4A8_EALIGN;
    if (ws_bytes < L->off[R_COUNT]) return W4A8_ENOSPACE;
    return W4A8_OK;
}

}  // namespace
}  // namespace w4a8

using namespace w4a8;

W4A8_EXPORT int w4a8_version(void) { return 100; }

W4A8_EXPORT const char* w4a8_status_string(int status) {
    switch (status) {
        case W4A8_OK: return "ok";
        case W4A8_EINVAL: return "invalid argument";
        case W4A8_EALIGN: return "misaligned pointer";
        case W4A8_ENOSPACE: return "buffer or workspace too small";
        case W4A8_ECUDA: return "CUDA error";
        case W4A8_EUNSUPPORTED: return "unsupported shape";
        case W4A8_ETIMEOUT: return "device wait timed out";
        case W4A8_EDEVICE: return "bad data on device";
        default: return "unknown status";
    }
}

namespace w4a8 {
namespace {
// Split the packer's `layout` argument into the row layout, the quantisation scheme
// (0 asymmetric, 1 symmetric, 2 percentile range) and the group size; false for an
// unknown flag or combination (two schemes, two group sizes, the percentile range
// with a group other than 128).
bool parse_layout(int layout, int* base, int* scheme, int* group) {
    const int flags = layout & ~0xFF;
    if (flags & ~(W4A8_PACK_SYMMETRIC | W4A8_PACK_CLIP999 | W4A8_PACK_GROUP64 | W4A8_PACK_GROUP256)) return false;
    if ((flags & W4A8_PACK_SYMMETRIC) && (flags & W4A8_PACK_CLIP999)) return false;
    if ((flags & W4A8_PACK_GROUP64) && (flags & W4A8_PACK_GROUP256)) return false;
    *base = layout & 0xFF;
    if (*base != W4A8_LAYOUT_PLAIN && *base != W4A8_LAYOUT_GATEUP) return false;
    *scheme = (flags & W4A8_PACK_SYMMETRIC) ? 1 : (flags & W4A8_PACK_CLIP999) ? 2 : 0;
    *group = (flags & W4A8_PACK_GROUP64) ? 64 : (flags & W4A8_PACK_GROUP256) ? 256 : 128;
    return !(*scheme == 2 && *group != 128);
}

size_t packed_bytes_of(int E, int N, int K, int base, int group) {
    if (E < 1 || N < 1 || K < 1) return 0;
    if (base == W4A8_LAYOUT_GATEUP && (N & 1)) return 0;
    const size_t G = (size_t)k_padded_for(K, group) / kGroup;
    return (size_t)kHeaderBytes + (size_t)E * packed_tiles(N, base) * G * block_bytes_for(group);
}

bool valid_group(int group) { return group == 64 || group == 128 || group == 256; }
}  // namespace
}  // namespace w4a8

W4A8_EXPORT size_t w4a8_packed_bytes(int E, int N, int K, int layout) {
    int base, scheme, group;
    if (!parse_layout(layout, &base, &scheme, &group)) return 0;
    return packed_bytes_of(E, N, K, base, group);
}

W4A8_EXPORT int w4a8_pack_weights(const void* w_bf16, int E, int N, int K, int layout, void* packed,
                                  size_t packed_bytes, uint8_t* codes_opt, uint16_t* scale_f16_opt,
                                  uint16_t* zp_f16_opt, void* stream) {
    int base, scheme, group;
    if (!parse_layout(layout, &base, &scheme, &group)) return W4A8_EINVAL;
    const size_t need = packed_bytes_of(E, N, K, base, group);
    if (need == 0 || w_bf16 == nullptr || packed == nullptr) return W4A8_EINVAL;
    if (E > 65535) return W4A8_EUNSUPPORTED;
    if (!aligned(w_bf16, 16) || !aligned(packed, kAlign)) return W4A8_EALIGN;
    if ((codes_opt && !aligned(codes_opt, 16)) || (scale_f16_opt && !aligned(scale_f16_opt, 2)) ||
        (zp_f16_opt && !aligned(zp_f16_opt, 2)))
        return W4A8_EALIGN;
    if (packed_bytes < need) return W4A8_ENOSPACE;
    return to_status(launch_pack(static_cast<const uint16_t*>(w_bf16), E, N, K, base, scheme, group,
                                 static_cast<uint8_t*>(packed), codes_opt, scale_f16_opt, zp_f16_opt,
                                 static_cast<cudaStream_t>(stream)));
}

namespace {
int kv_check(int T, int H, int D) {
    if (T < 0 || H < 1 || D < 16) return W4A8_EINVAL;
    if (D % 16 != 0 || H > kv_max_heads()) return W4A8_EUNSUPPORTED;
    return W4A8_OK;
}
}  // namespace

W4A8_EXPORT int w4a8_kv_calibrate(const void* x_bf16, int T, int H, int D, float* scale, void* stream) {
    const int c = kv_check(T, H, D);
    if (c != W4A8_OK) return c;
    if (scale == nullptr || (T > 0 && x_bf16 == nullptr)) return W4A8_EINVAL;
    if (!aligned(x_bf16, 16) || !aligned(scale, 4)) return W4A8_EALIGN;
    return to_status(launch_kv_calibrate(static_cast<const uint16_t*>(x_bf16), T, H, D, scale, sm_count(),
                                         static_cast<cudaStream_t>(stream)));
}

W4A8_EXPORT int w4a8_kv_quant(const void* x_bf16, int T, int H, int D, const float* scale, int8_t* q,
                              void* stream) {
    const int c = kv_check(T, H, D);
    if (c != W4A8_OK) return c;
    if (T == 0) return W4A8_OK;
    if (x_bf16 == nullptr || scale == nullptr || q == nullptr) return W4A8_EINVAL;
    if (!aligned(x_bf16, 16) || !aligned(q, 16) || !aligned(scale, 4)) return W4A8_EALIGN;
    return to_status(launch_kv_quant(static_cast<const uint16_t*>(x_bf16), T, H, D, scale, q, sm_count(),
                                     static_cast<cudaStream_t>(stream)));
}

W4A8_EXPORT int w4a8_kv_dequant(const int8_t* q, int T, int H, int D, const float* scale, void* x_bf16,
                                void* stream) {
    const int c = kv_check(T, H, D);
    if (c != W4A8_OK) return c;
    if (T == 0) return W4A8_OK;
    if (x_bf16 == nullptr || scale == nullptr || q == nullptr) return W4A8_EINVAL;
    if (!aligned(x_bf16, 16) || !aligned(q, 16) || !aligned(scale, 4)) return W4A8_EALIGN;
    return to_status(launch_kv_dequant(q, T, H, D, scale, static_cast<uint16_t*>(x_bf16), sm_count(),
                                       static_cast<cudaStream_t>(stream)));
}

W4A8_EXPORT int w4a8_quant_act(const void* x_bf16, int T, int K, int8_t* q, float* s, void* stream) {
    if (T < 0 || K < 1) return W4A8_EINVAL;
    if (T == 0) return W4A8_OK;
    if (x_bf16 == nullptr || q == nullptr || s == nullptr) return W4A8_EINVAL;
    if (!aligned(x_bf16, 16) || !aligned(q, 16) || !aligned(s, 16)) return W4A8_EALIGN;
    ProfScope prof(W4A8_KERNEL_ACT_QUANT, 1, static_cast<cudaStream_t>(stream));
    return to_status(launch_quant_act(static_cast<const uint16_t*>(x_bf16), T, K, q, s,
                                      static_cast<cudaStream_t>(stream)));
}

W4A8_EXPORT int w4a8_route_topk(const void* logits_bf16, int T, int E, int k, int32_t* ids, float* w,
                                void* stream) {
    if (T < 0 || E < 1 || k < 1 || k > E) return W4A8_EINVAL;
    if (E > kMaxExperts || k > 32) return W4A8_EUNSUPPORTED;
    if (T == 0) return W4A8_OK;
    if (logits_bf16 == nullptr || ids == nullptr || w == nullptr) return W4A8_EINVAL;
    if (!aligned(logits_bf16, 16) || !aligned(ids, 16) || !aligned(w, 16)) return W4A8_EALIGN;
    ProfScope prof(W4A8_KERNEL_ROUTE, 1, static_cast<cudaStream_t>(stream));
    return to_status(launch_route_topk(static_cast<const uint16_t*>(logits_bf16), T, E, k, ids, w,
                                       static_cast<cudaStream_t>(stream)));
}

W4A8_EXPORT int w4a8_moe_rows_capacity(int T, int E, int k) { return rows_capacity(T, E, k); }

W4A8_EXPORT int w4a8_moe_act_block_rows(int T, int E, int k) {
    if (T < 0 || E < 1 || k < 1) return 0;
    return act_block_rows(gemm_tile_tokens((int)((long long)T * k / E)), rows_capacity(T, E, k));
}

W4A8_EXPORT size_t w4a8_moe_workspace_bytes(int T, int E, int k, int H, int F) {
    MoeLayout L;
    if (!moe_layout(T, E, k, H, F, false, &L)) return 0;
    return L.off[R_COUNT];
}

W4A8_EXPORT size_t w4a8_moe_host_workspace_bytes(int T, int E, int k, int H, int F) {
    MoeLayout L;
    if (!moe_layout(T, E, k, H, F, true, &L)) return 0;
    return L.off[R_COUNT];
}

W4A8_EXPORT int w4a8_moe_forward(const void* packed_up, const void* packed_down, int E, int H, int F,
                                 const void* x_bf16, int T, const int32_t* ids, const float* w, int k,
                                 void* out_bf16, void* ws, size_t ws_bytes, void* stream) {
    MoeLayout L;
    const int st = check_moe_args(packed_up, packed_down, E, H, F, T, k, ws, ws_bytes, false, &L);
    if (st != W4A8_OK) return st;
    if (T > 0) {
        if (x_bf16 == nullptr || ids == nullptr || w == nullptr || out_bf16 == nullptr) return W4A8_EINVAL;
        if (!aligned(x_bf16, 16) || !aligned(ids, 16) || !aligned(w, 16) || !aligned(out_bf16, 16))
            return W4A8_EALIGN;
    }
    return moe_forward_impl(packed_up, packed_down, E, H, F, static_cast<const uint16_t*>(x_bf16), T, ids, w, k,
                            static_cast<uint16_t*>(out_bf16), ws, L, static_cast<cudaStream_t>(stream));
}

W4A8_EXPORT size_t w4a8_moe_workspace_bytes_g(int T, int E, int k, int H, int F, int group) {
    MoeLayout L;
    if (!moe_layout(T, E, k, H, F, false, &L, false, group)) return 0;
    return L.off[R_COUNT];
}

W4A8_EXPORT int w4a8_moe_forward_g(const void* packed_up, const void* packed_down, int E, int H, int F, int group,
                                   const void* x_bf16, int T, const int32_t* ids, const float* w, int k,
                                   void* out_bf16, void* ws, size_t ws_bytes, void* stream) {
    if (!valid_group(group)) return W4A8_EINVAL;
    MoeLayout L;
    const int st = check_moe_args(packed_up, packed_down, E, H, F, T, k, ws, ws_bytes, false, &L, false, group);
    if (st != W4A8_OK) return st;
    if (T > 0) {
        if (x_bf16 == nullptr || ids == nullptr || w == nullptr || out_bf16 == nullptr) return W4A8_EINVAL;
        if (!aligned(x_bf16, 16) || !aligned(ids, 16) || !aligned(w, 16) || !aligned(out_bf16, 16))
            return W4A8_EALIGN;
    }
    return moe_forward_impl(packed_up, packed_down, E, H, F, static_cast<const uint16_t*>(x_bf16), T, ids, w, k,
                            static_cast<uint16_t*>(out_bf16), ws, L, static_cast<cudaStream_t>(stream), group);
}

W4A8_EXPORT size_t w4a16_moe_workspace_bytes(int T, int E, int k, int H, int F) {
    MoeLayout L;
    if (!moe_layout(T, E, k, H, F, false, &L, true)) return 0;
    return L.off[R_COUNT];
}

W4A8_EXPORT int w4a16_moe_forward(const void* packed_up, const void* packed_down, int E, int H, int F,
                                  const void* x_bf16, int T, const int32_t* ids, const float* w, int k,
                                  void* out_bf16, void* ws, size_t ws_bytes, void* stream) {
    MoeLayout L;
    const int st = check_moe_args(packed_up, packed_down, E, H, F, T, k, ws, ws_bytes, false, &L, true);
    if (st != W4A8_OK) return st;
    if (T > 0) {
        if (x_bf16 == nullptr || ids == nullptr || w == nullptr || out_bf16 == nullptr) return W4A8_EINVAL;
        if (!aligned(x_bf16, 16) || !aligned(ids, 16) || !aligned(w, 16) || !aligned(out_bf16, 16))
            return W4A8_EALIGN;
    }
    return moe_forward_w4a16_impl(packed_up, packed_down, E, H, F, static_cast<const uint16_t*>(x_bf16), T, ids, w,
                                  k, static_cast<uint16_t*>(out_bf16), ws, L, static_cast<cudaStream_t>(stream));
}

W4A8_EXPORT int w4a8_moe_forward_host(const void* packed_up, const void* packed_down, int E, int H, int F,
                                      const void* x_bf16_host, int T, const int32_t* ids_host, const float* w_host,
                                      int k, void* out_bf16_host, void* ws, size_t ws_bytes, void* stream) {
    MoeLayout L;
    const int st = check_moe_args(packed_up, packed_down, E, H, F, T, k, ws, ws_bytes, true, &L);
    if (st != W4A8_OK) return st;
    if (T == 0) return W4A8_OK;
    if (x_bf16_host == nullptr || ids_host == nullptr || w_host == nullptr || out_bf16_host == nullptr)
        return W4A8_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint16_t* x = at<uint16_t>(ws, L, R_XIN);
    int32_t* ids = at<int32_t>(ws, L, R_IDSIN);
    float* w = at<float>(ws, L, R_WIN);
    uint16_t* out = at<uint16_t>(ws, L, R_OUT);
    W4A8_TRY(cudaMemcpyAsync(x, x_bf16_host, L.bytes[R_XIN], cudaMemcpyHostToDevice, s));
    W4A8_TRY(cudaMemcpyAsync(ids, ids_host, L.bytes[R_IDSIN], cudaMemcpyHostToDevice, s));
    W4A8_TRY(cudaMemcpyAsync(w, w_host, L.bytes[R_WIN], cudaMemcpyHostToDevice, s));
    const int r = moe_forward_impl(packed_up, packed_down, E, H, F, x, T, ids, w, k, out, ws, L, s);
    if (r != W4A8_OK) return r;
    W4A8_TRY(cudaMemcpyAsync(out_bf16_host, out, L.bytes[R_OUT], cudaMemcpyDeviceToHost, s));
    return W4A8_OK;
}

W4A8_EXPORT int w4a8_moe_forward_logits_host(const void* packed_up, const void* packed_down, int E, int H, int F,
                                             const void* x_bf16_host, int T, const void* logits_bf16_host, int k,
                                             void* out_bf16_host, void* ws, size_t ws_bytes, void* stream) {
    MoeLayout L;
    const int st = check_moe_args(packed_up, packed_down, E, H, F, T, k, ws, ws_bytes, true, &L);
    if (st != W4A8_OK) return st;
    if (T == 0) return W4A8_OK;
    if (x_bf16_host == nullptr || logits_bf16_host == nullptr || out_bf16_host == nullptr) return W4A8_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint16_t* x = at<uint16_t>(ws, L, R_XIN);
    uint16_t* logits = at<uint16_t>(ws, L, R_LOGITS);
    int32_t* ids = at<int32_t>(ws, L, R_IDSIN);
    float* w = at<float>(ws, L, R_WIN);
    uint16_t* out = at<uint16_t>(ws, L, R_OUT);
    W4A8_TRY(cudaMemcpyAsync(x, x_bf16_host, L.bytes[R_XIN], cudaMemcpyHostToDevice, s));
    W4A8_TRY(cudaMemcpyAsync(logits, logits_bf16_host, L.bytes[R_LOGITS], cudaMemcpyHostToDevice, s));
    {
        ProfScope p(W4A8_KERNEL_ROUTE, 1, s);
        W4A8_TRY(launch_route_topk(logits, T, E, k, ids, w, s));
    }
    const int r = moe_forward_impl(packed_up, packed_down, E, H, F, x, T, ids, w, k, out, ws, L, s);
    if (r != W4A8_OK) return r;
    W4A8_TRY(cudaMemcpyAsync(out_bf16_host, out, L.bytes[R_OUT], cudaMemcpyDeviceToHost, s));
    return W4A8_OK;
}

namespace w4a8 {
namespace {
struct GemmLayout {
    size_t err, nmt, mttab, act, total;
    int Mp, G;
};
bool gemm_layout(int M, int N, int K, GemmLayout* L, bool bf16 = false, int group = 128) {
    if (M < 0 || N < 1 || K < 1 || !valid_group(group)) return false;
    L->Mp = round_up(M, kRowPad);
    L->G = k_padded_for(K, group) / kGroup;  // 128-wide planes
    size_t o = 0;
    L->err = o; o += align_up(16);
    L->nmt = o; o += align_up(4);
    L->mttab = o; o += align_up((size_t)(M / 16 + 2) * 16);
    L->act = o; o += align_up((size_t)L->G * L->Mp * (bf16 ? 256 : 128));
    L->total = o;
    return true;
}
}  // namespace
}  // namespace w4a8

W4A8_EXPORT size_t w4a8_gemm_workspace_bytes(int M, int N, int K) {
    GemmLayout L;
    if (!gemm_layout(M, N, K, &L)) return 0;
    return L.total;
}

W4A8_EXPORT size_t w4a8_gemm_workspace_bytes_g(int M, int N, int K, int group) {
    GemmLayout L;
    if (!gemm_layout(M, N, K, &L, false, group)) return 0;
    return L.total;
}

W4A8_EXPORT int w4a8_gemm_g(const int8_t* qa, const float* sa, int M, const void* packed, int N, int K, int group,
                            float* y, int32_t* partials_opt, void* ws, size_t ws_bytes, void* stream) {
    GemmLayout L;
    if (!gemm_layout(M, N, K, &L, false, group)) return W4A8_EINVAL;
    if (packed == nullptr || ws == nullptr) return W4A8_EINVAL;
    if (!aligned(packed, kAlign) || !aligned(ws, kAlign)) return W4A8_EALIGN;
    if (ws_bytes < L.total) return W4A8_ENOSPACE;
    uint8_t* base = static_cast<uint8_t*>(ws);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* err = reinterpret_cast<uint32_t*>(base + L.err);
    W4A8_TRY(cudaMemsetAsync(err, 0, 16, s));
    if (M == 0) return W4A8_OK;
    if (qa == nullptr || sa == nullptr || y == nullptr) return W4A8_EINVAL;
    if (!aligned(qa, 16) || !aligned(sa, 4) || !aligned(y, 4) || (partials_opt && !aligned(partials_opt, 4)))
        return W4A8_EALIGN;
    int* n_mtiles = reinterpret_cast<int*>(base + L.nmt);
    int4* mt_tab = reinterpret_cast<int4*>(base + L.mttab);
    int8_t* act = reinterpret_cast<int8_t*>(base + L.act);
    ProfScope prof(W4A8_KERNEL_GEMM_DENSE, 2, s);
    const int tile = gemm_tile_tokens(M);
    const int rb = act_block_rows(tile, L.Mp);
    W4A8_TRY(launch_dense_prep(qa, M, round_up(K, kGroup), L.G * kGroup, tile, rb, act, mt_tab, n_mtiles, s));
    GemmArgs a{};
    a.wblocks = static_cast<const uint8_t*>(packed) + kHeaderBytes;
    a.NT = packed_tiles(N, W4A8_LAYOUT_PLAIN);
    a.G = L.G;
    a.act = act;
    a.act_plane = (size_t)rb * 128;
    a.act_rb_stride = (size_t)L.G * rb * 128;
    a.act_scale = sa;
    a.mt_tab = mt_tab;
    a.n_mtiles = n_mtiles;
    a.mode = 0;
    a.out = y;
    a.ldo = N;
    a.nvalid = N;
    a.partials = partials_opt;
    a.err = err;
    a.group = group;
    apply_debug(a);
    W4A8_TRY(launch_gemm(a, tile, sm_count(), s));
    return W4A8_OK;
}

W4A8_EXPORT int w4a8_gemm(const int8_t* qa, const float* sa, int M, const void* packed, int N, int K, float* y,
                          int32_t* partials_opt, void* ws, size_t ws_bytes, void* stream) {
    return w4a8_gemm_g(qa, sa, M, packed, N, K, 128, y, partials_opt, ws, ws_bytes, stream);
}

W4A8_EXPORT size_t w4a16_gemm_workspace_bytes(int M, int N, int K) {
    GemmLayout L;
    if (!gemm_layout(M, N, K, &L, true)) return 0;
    return L.total;
}

W4A8_EXPORT int w4a16_gemm(const void* x_bf16, int M, const void* packed, int N, int K, float* y, void* ws,
                           size_t ws_bytes, void* stream) {
    GemmLayout L;
    if (!gemm_layout(M, N, K, &L, true)) return W4A8_EINVAL;
    if (packed == nullptr || ws == nullptr) return W4A8_EINVAL;
    if (!aligned(packed, kAlign) || !aligned(ws, kAlign)) return W4A8_EALIGN;
    if (ws_bytes < L.total) return W4A8_ENOSPACE;
    uint8_t* base = static_cast<uint8_t*>(ws);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* err = reinterpret_cast<uint32_t*>(base + L.err);
    W4A8_TRY(cudaMemsetAsync(err, 0, 16, s));
    if (M == 0) return W4A8_OK;
    if (x_bf16 == nullptr || y == nullptr) return W4A8_EINVAL;
    if (!aligned(x_bf16, 2) || !aligned(y, 4)) return W4A8_EALIGN;
    int* n_mtiles = reinterpret_cast<int*>(base + L.nmt);
    int4* mt_tab = reinterpret_cast<int4*>(base + L.mttab);
    uint8_t* act = base + L.act;
    ProfScope prof(W4A8_KERNEL_GEMM_DENSE, 2, s);
    W4A8_TRY(launch_dense_prep_bf16(static_cast<const uint16_t*>(x_bf16), M, K, act, mt_tab, n_mtiles, s));
    GemmArgs a{};
    a.wblocks = static_cast<const uint8_t*>(packed) + kHeaderBytes;
    a.NT = packed_tiles(N, W4A8_LAYOUT_PLAIN);
    a.G = L.G;
    a.act = reinterpret_cast<const int8_t*>(act);
    a.act_rb_stride = (size_t)L.G * 16 * 256;
    a.mt_tab = mt_tab;
    a.n_mtiles = n_mtiles;
    a.mode = 0;
    a.out = y;
    a.ldo = N;
    a.nvalid = N;
    a.err = err;
    apply_debug(a);
    W4A8_TRY(launch_gemm_w4a16(a, sm_count(), s));
    return W4A8_OK;
}

W4A8_EXPORT int w4a8_debug_region(int T, int E, int k, int H, int F, int what, size_t* offset, size_t* bytes) {
    MoeLayout L;
    const bool w4a16 = (what & W4A8_DUMP_W4A16) != 0;
    const int group = (what & W4A8_DUMP_GROUP64) ? 64 : (what & W4A8_DUMP_GROUP256) ? 256 : 128;
    what &= ~(W4A8_DUMP_W4A16 | W4A8_DUMP_GROUP64 | W4A8_DUMP_GROUP256);
    if (!moe_layout(T, E, k, H, F, false, &L, w4a16, group) || offset == nullptr || bytes == nullptr)
        return W4A8_EINVAL;
    static const Region map[] = {R_COUNTS, R_OFFS, R_PERM, R_INV, R_POFFS, R_ACT1,
                                 R_S1,     R_H,    R_ACT2, R_S2,  R_Y2,    R_ERR};
    if (what < 0 || what >= (int)(sizeof(map) / sizeof(map[0]))) return W4A8_EINVAL;
    *offset = L.off[map[what]];
    *bytes = what == W4A8_DUMP_ERR ? 4 : L.bytes[map[what]];
    return W4A8_OK;
}

W4A8_EXPORT int w4a8_debug_dump(const void* ws, int T, int E, int k, int H, int F, int what, void* dst,
                                size_t bytes, void* stream) {
    size_t off = 0, n = 0;
    const int r = w4a8_debug_region(T, E, k, H, F, what, &off, &n);
    if (r != W4A8_OK) return r;
    if (ws == nullptr || dst == nullptr) return W4A8_EINVAL;
    if (bytes < n) n = bytes;
    if (n == 0) return W4A8_OK;
    return to_status(cudaMemcpyAsync(dst, static_cast<const uint8_t*>(ws) + off, n, cudaMemcpyDefault,
                                     static_cast<cudaStream_t>(stream)));
}

W4A8_EXPORT int w4a8_last_device_error(const void* ws, void* stream) {
    if (ws == nullptr) return W4A8_EINVAL;
    uint32_t v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return W4A8_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return W4A8_ECUDA;
    return (int)v;
}

W4A8_EXPORT int w4a8_debug_inject(unsigned int flags, long long wait_limit_cycles) {
    if ((flags & ~kDebugSkipFirstCopy) != 0 || wait_limit_cycles < 0) return W4A8_EINVAL;
    g_debug.flags = flags;
    g_debug.wait_limit = wait_limit_cycles;
    return W4A8_OK;
}

W4A8_EXPORT int w4a8_profile_start(void) {
    g_prof.on = true;
    return W4A8_OK;
}

W4A8_EXPORT int w4a8_profile_stop(int* launches, float* total_ms, int n) {
    float ms[W4A8_KERNEL_KINDS] = {0.f};
    int rc = W4A8_OK;
    for (auto& r : g_prof.recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            rc = W4A8_ECUDA;
        ms[r.kind] += t;
        g_prof.pool.push_back(r.a);
        g_prof.pool.push_back(r.b);
    }
    for (int i = 0; i < n && i < W4A8_KERNEL_KINDS; ++i) {
        if (launches) launches[i] = g_prof.launches[i];
        if (total_ms) total_ms[i] = ms[i];
    }
    g_prof.recs.clear();
    for (int i = 0; i < W4A8_KERNEL_KINDS; ++i) g_prof.launches[i] = 0;
    g_prof.on = false;
    return rc;
}

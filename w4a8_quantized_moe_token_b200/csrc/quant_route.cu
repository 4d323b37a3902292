// Quantisation, routing, permutation and combine kernels of the W4A8 MoE layer.
//
// Sources of the arithmetic:
//   weight INT4 (group 128, asymmetric, low nibble first):
//       «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» (pptc.cn) sections 2.1 and 2.2;
//   activation INT8 (per token, symmetric, scale = max|x| / (2^(b-1) - 1)):
//       LLM quantisation primer (hotelren.com 5982361) section 2.1 and the Kimi 2.7T
//       MoE W4A8 article (hotelren.com 5173946) section 4.3, step 3;
//   routing kept in 16-bit float: the Kimi 2.7T MoE W4A8 article, section 5.2.
// Every "round" is round-half-to-even, every division a correctly rounded fp32
// division, so codes agree bit for bit with any other IEEE implementation.
#include <climits>

#include "w4a8_common.cuh"
#include "w4a8_internal.h"

namespace w4a8 {

namespace {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// a1: weight quantisation + packing.  One block per (group gq, tile t, matrix e);
// thread r quantises tiled row r's GRP weights of group gq, 64 at a time: a first
// pass over the group finds its range, a second one (re-reading the row from cache)
// computes the codes and writes them into the group's 128-wide plane blocks.
// ---------------------------------------------------------------------------
// 64 weights of a row from K index k0 on (zero past K and for rows past N)
__device__ __forceinline__ void load_w64(const uint16_t* row, int K, int k0, float (&v)[64]) {
    if (row != nullptr && (K & 7) == 0 && k0 + 64 <= K) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 p = *reinterpret_cast<const uint4*>(row + k0 + 8 * i);
            const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                v[8 * i + 2 * h] = bf16_to_f32((uint16_t)(pw[h] & 0xFFFFu));
                v[8 * i + 2 * h + 1] = bf16_to_f32((uint16_t)(pw[h] >> 16));
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) v[i] = (row != nullptr && k0 + i < K) ? bf16_to_f32(row[k0 + i]) : 0.f;
    }
}

// sym: 0 asymmetric min/max, 1 symmetric, 2 asymmetric on the 0.1th..99.9th percentile
// range (128-value groups only); G = 128-wide planes per row
template <int GRP>
__global__ void __launch_bounds__(128) pack_kernel(const uint16_t* __restrict__ w, int N, int K, int layout, int sym,
                                                   int NT, int G, uint8_t* __restrict__ blocks,
                                                   uint8_t* __restrict__ codes_out, uint16_t* __restrict__ scale_out,
                                                   uint16_t* __restrict__ zp_out) {
    constexpr int kChunks = GRP / 64;
    constexpr int kBB = block_bytes_for(GRP);
    const int gq = blockIdx.x, t = blockIdx.y, e = blockIdx.z;
    const int Gq = G * kGroup / GRP;
    const int r = threadIdx.x;
    int src;
    bool valid;
    if (layout == 1) {  // gate|up interleave: even tiled rows gate channel f, odd rows up channel f
        const int F = N / 2;
        const int f = t * (kTileRows / 2) + (r >> 1);
        valid = f < F;
        src = (r & 1) ? F + f : f;
    } else {
        src = t * kTileRows + r;
        valid = src < N;
    }
    const uint16_t* row = valid ? w + ((size_t)e * N + src) * (size_t)K : nullptr;
    float v[64];
    __half sh;
    int zp;
    if (sym != 1) {
        float lo, hi;
        // min / max, and the two smallest and two largest values (a0 <= a1, b0 >= b1)
        float mn0 = INFINITY, mx0 = -INFINITY;
        float a0 = INFINITY, a1 = INFINITY, b0 = -INFINITY, b1 = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < kChunks; ++c) {
            load_w64(row, K, gq * GRP + c * 64, v);
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                mn0 = fminf(mn0, v[i]);
                mx0 = fmaxf(mx0, v[i]);
                if (sym == 2) {
                    a1 = fminf(a1, fmaxf(v[i], a0));
                    a0 = fminf(a0, v[i]);
                    b1 = fmaxf(b1, fminf(v[i], b0));
                    b0 = fmaxf(b0, v[i]);
                }
            }
        }
        if (sym == 2) {
            // the 0.1th and 99.9th percentiles of a 128-value group: linear interpolation
            // between the order statistics around positions 0.127 and 126.873
            lo = __fadd_rn(a0, __fmul_rn(0.127f, __fsub_rn(a1, a0)));
            hi = __fadd_rn(b1, __fmul_rn(0.873f, __fsub_rn(b0, b1)));
        } else {
            lo = mn0;
            hi = mx0;
        }
        // range widened to contain 0
        const float mn = fminf(lo, 0.f), mx = fmaxf(hi, 0.f);
        // scale = (max - min) / (2^4 - 1), stored as fp16; the fp16 value is the one used
        sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
        if (__half2float(sh) == 0.f) sh = __float2half_rn(1.0f);
        // zero_point = round(-min / scale)
        zp = (int)fminf(fmaxf(rintf(__fdiv_rn(-mn, __half2float(sh))), 0.f), 15.f);
    } else {
        // symmetric (b = 4): scale = max|w| / (2^3 - 1), stored as code q + 8 with zero point 8
        float amax = 0.f;
#pragma unroll 1
        for (int c = 0; c < kChunks; ++c) {
            load_w64(row, K, gq * GRP + c * 64, v);
#pragma unroll
            for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
        sh = __float2half_rn(__fdiv_rn(amax, 7.0f));
        if (__half2float(sh) == 0.f) sh = __float2half_rn(1.0f);
        zp = 8;
    }
    const float shf = __half2float(sh);
    const size_t tile_blk = (size_t)(e * NT + t) * G;
#pragma unroll 1
    for (int c = 0; c < kChunks; ++c) {
        const int k0 = gq * GRP + c * 64;  // K index of this chunk's first weight
        load_w64(row, K, k0, v);
        uint32_t code[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if (sym != 1) {
                // index = clamp(round(w / scale) + zero_point, 0, 15)
                const int cc = (int)rintf(__fdiv_rn(v[i], shf)) + zp;
                code[i] = (uint32_t)min(max(cc, 0), 15);
            } else {
                // q = clamp(round(w / scale), -7, 7)
                const int q = (int)rintf(__fdiv_rn(v[i], shf));
                code[i] = (uint32_t)(min(max(q, -7), 7) + 8);
            }
        }
        // tiled block of plane k0 / 128: word i of the plane (K = 8i .. 8i+7):
        // byte b = code[8i+b] | code[8i+4+b] << 4; this chunk is the plane's half k0 / 64 % 2
        uint8_t* blk = blocks + (tile_blk + (size_t)(k0 / kGroup)) * kBB;
        const int hh = (k0 / 64) & 1;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            uint32_t wd[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int l = 32 * cc + 8 * q;  // chunk-local index of the word's first code
                uint32_t x = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) x |= (code[l + b] | (code[l + 4 + b] << 4)) << (8 * b);
                wd[q] = x;
            }
            *reinterpret_cast<uint4*>(blk + code_chunk_offset(r, 2 * hh + cc)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
        if (valid && codes_out != nullptr) {
            // canonical order: byte j = code[2j] | code[2j+1] << 4
            uint8_t* dst = codes_out + ((size_t)e * N + src) * (size_t)(G * kGroup / 2) + (size_t)k0 / 2;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t wd[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t x = 0;
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const int j = 16 * cc + 4 * q + b;
                        x |= (code[2 * j] | (code[2 * j + 1] << 4)) << (8 * b);
                    }
                    wd[q] = x;
                }
                *reinterpret_cast<uint4*>(dst + 16 * cc) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            }
        }
    }
    // scale and zero point: in the plane block (group 64: the plane's sub-group slot;
    // group 256: both of the group's planes)
    const __half zh = __float2half_rn((float)zp);
#pragma unroll
    for (int pp = 0; pp < (GRP > kGroup ? GRP / kGroup : 1); ++pp) {
        const int plane = GRP > kGroup ? gq * (GRP / kGroup) + pp : gq * GRP / kGroup;
        const int sub = GRP < kGroup ? (gq & 1) : 0;
        uint8_t* blk = blocks + (tile_blk + (size_t)plane) * kBB + sub * 512;
        reinterpret_cast<__half*>(blk + kScaleOff)[r] = sh;
        reinterpret_cast<__half*>(blk + kZpOff)[r] = zh;
    }
    if (valid) {
        if (scale_out != nullptr) scale_out[((size_t)e * N + src) * Gq + gq] = __half_as_ushort(sh);
        if (zp_out != nullptr) zp_out[((size_t)e * N + src) * Gq + gq] = __half_as_ushort(zh);
    }
    if (e == 0 && t == 0 && gq == 0 && r == 0) {
        PackHeader* h = reinterpret_cast<PackHeader*>(blocks - kHeaderBytes);
        h->magic = kPackMagic;
        h->version = 2;
        h->layout = (uint32_t)layout | (sym == 1 ? 0x100u : sym == 2 ? 0x200u : 0u);
        h->E = gridDim.z;
        h->N = (uint32_t)N;
        h->K = (uint32_t)K;
        h->Kp = (uint32_t)(G * kGroup);
        h->G = (uint32_t)G;
        h->NT = (uint32_t)NT;
        h->rows_per_tile = kTileRows;
        h->block_bytes = kBB;
        h->group = GRP;
    }
}

// ---------------------------------------------------------------------------
// a2: per-token INT8, natural layout [T][Kp].  One warp per row.  With K a multiple
// of 8 the row is read in 16-byte vectors (8 bf16 per lane and step) and the codes are
// written 8 bytes at a time; other K take the scalar path.  The codes are the same.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_act_kernel(const uint16_t* __restrict__ x, int T, int K, int Kp,
                                                        int8_t* __restrict__ q, float* __restrict__ s) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= T) return;
    const uint16_t* xr = x + (size_t)row * K;
    int8_t* qr = q + (size_t)row * Kp;
    float amax = 0.f;
    if ((K & 7) == 0) {
        const uint4* xv = reinterpret_cast<const uint4*>(xr);
        for (int c = lane; c < K / 8; c += 32) {
            const uint4 p = __ldg(xv + c);
            const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int h = 0; h < 4; ++h)
                amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(pw[h] << 16)), fabsf(__uint_as_float(pw[h] & 0xFFFF0000u))));
        }
        amax = warp_max(amax);
        const float sc = __fdiv_rn(amax, 127.0f);
        const float rinv = __fdiv_rn(1.0f, sc);
        for (int c = lane; c < Kp / 8; c += 32) {
            uint32_t out[2] = {0u, 0u};
            if (c < K / 8 && amax > 0.f) {
                const uint4 p = __ldg(xv + c);
                const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint32_t lo = (uint32_t)(quant_i8_fast(__uint_as_float(pw[h] << 16), sc, rinv) & 0xFF);
                    const uint32_t hi = (uint32_t)(quant_i8_fast(__uint_as_float(pw[h] & 0xFFFF0000u), sc, rinv) & 0xFF);
                    out[h >> 1] |= (lo | (hi << 8)) << (16 * (h & 1));
                }
            }
            *reinterpret_cast<uint2*>(qr + 8 * c) = make_uint2(out[0], out[1]);
        }
        if (lane == 0) s[row] = sc;
        return;
    }
    for (int k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(bf16_to_f32(xr[k])));
    amax = warp_max(amax);
    const float sc = __fdiv_rn(amax, 127.0f);
    const float rinv = __fdiv_rn(1.0f, sc);
    for (int k = lane; k < Kp; k += 32) {
        int c = 0;
        if (k < K && amax > 0.f) c = quant_i8_fast(bf16_to_f32(xr[k]), sc, rinv);
        qr[k] = (int8_t)c;
    }
    if (lane == 0) s[row] = sc;
}

// ---------------------------------------------------------------------------
// a3: top-k softmax routing.  One warp per token; lane l owns experts l, l+32, ...
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) route_topk_kernel(const uint16_t* __restrict__ logits, int T, int E, int k,
                                                         int32_t* __restrict__ ids, float* __restrict__ wout) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const uint16_t* lr = logits + (size_t)t * E;
    const int per_lane = (E + 31) >> 5;
    uint32_t taken = 0;
    float top = -INFINITY;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = INT_MAX;
        for (int i = 0; i < per_lane; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u)) {
                float v = bf16_to_f32(lr[e]);
                if (isnan(v)) v = -INFINITY;
                if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
        }
        if (lane == (be & 31)) taken |= 1u << (be >> 5);
        if (j == 0) top = bv;
        if (lane == 0) {
            ids[(size_t)t * k + j] = be;
            wout[(size_t)t * k + j] = bv;  // logit for now, turned into a probability below
        }
    }
    float sum = 0.f;
    for (int i = 0; i < per_lane; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            const float v = bf16_to_f32(lr[e]);
            if (!isnan(v)) sum += expf(v - top);
        }
    }
    sum = warp_sum(sum);
    __syncwarp();
    if (lane < k) {
        const float lv = wout[(size_t)t * k + lane];
        wout[(size_t)t * k + lane] = expf(lv - top) / sum;
    }
}

// ---------------------------------------------------------------------------
// a4: stable grouping of slots by expert (counting sort in three passes)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPermChunk) perm_hist_kernel(const int32_t* __restrict__ ids, int nslots, int E,
                                                              int* __restrict__ chist, uint32_t* err) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    __shared__ int h[kMaxExperts];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int i = blockIdx.x * kPermChunk + threadIdx.x;
    if (i < nslots) {
        const int e = ids[i];
        if (e >= 0 && e < E) atomicAdd(&h[e], 1);
        else atomicOr(err, kErrBadExpert);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chist[(size_t)blockIdx.x * E + e] = h[e];
}

// block-wide exclusive scan (blockDim.x == 1024) of one int per thread
__device__ int block_exclusive_scan(int v, int* sh, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) sh[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = sh[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        sh[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int before = (warp > 0 ? sh[warp - 1] : 0) + incl - v;
    *total = sh[31];
    __syncthreads();
    return before;
}

__global__ void __launch_bounds__(1024) perm_scan_kernel(int* __restrict__ chist, int nchunk, int E, int tile_tokens,
                                                        int* __restrict__ counts, int* __restrict__ offs,
                                                        int* __restrict__ poffs, int* __restrict__ mtstart,
                                                        int4* __restrict__ mt_tab, int* __restrict__ row_src) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    __shared__ int sh[32];
    const int e = threadIdx.x;
    int c_e = 0;
    if (e < E) {
        // per-chunk histogram -> slots of e in all earlier chunks (in place)
        for (int c = 0; c < nchunk; ++c) {
            const int v = chist[(size_t)c * E + e];
            chist[(size_t)c * E + e] = c_e;
            c_e += v;
        }
    }
    int t0, t1, t2;
    const int o0 = block_exclusive_scan(c_e, sh, &t0);
    const int o1 = block_exclusive_scan(round_up(c_e, kRowPad), sh, &t1);
    const int o2 = block_exclusive_scan(ceil_div(c_e, tile_tokens), sh, &t2);
    if (e < E) {
        counts[e] = c_e;
        offs[e] = o0;
        poffs[e] = o1;
        mtstart[e] = o2;
        for (int rr = o1 + c_e; rr < o1 + round_up(c_e, kRowPad); ++rr) row_src[rr] = -1;
        // one entry per row tile of this expert: (expert, first row, rows)
        for (int t = 0; t < ceil_div(c_e, tile_tokens); ++t)
            mt_tab[o2 + t] = make_int4(e, o1 + t * tile_tokens, min(tile_tokens, c_e - t * tile_tokens), 0);
    }
    if (e == 0) {
        offs[E] = t0;
        poffs[E] = t1;
        mtstart[E] = t2;
    }
}

__global__ void __launch_bounds__(kPermChunk) perm_scatter_kernel(const int32_t* __restrict__ ids, int nslots, int E,
                                                                 const int* __restrict__ chist,
                                                                 const int* __restrict__ offs,
                                                                 const int* __restrict__ poffs, int* __restrict__ perm,
                                                                 int* __restrict__ inv, int* __restrict__ row_src) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    constexpr int kWarps = kPermChunk / 32;
    __shared__ int wcnt[kWarps][kMaxExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int idx = threadIdx.x; idx < kWarps * E; idx += blockDim.x) wcnt[idx / E][idx % E] = 0;
    __syncthreads();
    const int i = blockIdx.x * kPermChunk + threadIdx.x;
    const bool valid = i < nslots;
    const int e = valid ? ids[i] : -1;
    const bool good = valid && e >= 0 && e < E;
    const int key = good ? e : E + lane;  // unmatched keys for slots that take no part
    const uint32_t mask = __match_any_sync(0xffffffffu, key);
    const int rank_w = __popc(mask & ((1u << lane) - 1u));
    if (good && lane == __ffs(mask) - 1) wcnt[warp][e] = __popc(mask);
    __syncthreads();
    if (good) {
        int p = chist[(size_t)blockIdx.x * E + e] + rank_w;
        for (int w2 = 0; w2 < warp; ++w2) p += wcnt[w2][e];
        perm[offs[e] + p] = i;
        const int rr = poffs[e] + p;
        inv[i] = rr;
        row_src[rr] = i;
    } else if (valid) {
        inv[i] = -1;
    }
}

// a4 for small batches (up to kPermSmallSlots slots): histogram, scans and the
// stable scatter in one CTA, in slot order, 1024 slots at a time.
__global__ void __launch_bounds__(1024) perm_small_kernel(const int32_t* __restrict__ ids, int nslots, int E,
                                                         int tile_tokens, int* __restrict__ counts,
                                                         int* __restrict__ offs, int* __restrict__ poffs,
                                                         int* __restrict__ mtstart, int4* __restrict__ mt_tab,
                                                         int* __restrict__ perm, int* __restrict__ inv,
                                                         int* __restrict__ row_src, uint32_t* err) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    extern __shared__ int psm[];
    int* s_off = psm;          // [E] counts, then the exclusive offsets
    int* s_poff = psm + E;     // [E] padded offsets
    int* s_run = psm + 2 * E;  // [E] slots of e placed so far
    int* s_wcnt = psm + 3 * E; // [32][E] slots of e in each warp of the current chunk
    __shared__ int sh[32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < E; e += blockDim.x) {
        s_off[e] = 0;
        s_run[e] = 0;
    }
    __syncthreads();
    for (int i = tid; i < nslots; i += blockDim.x) {
        const int e = ids[i];
        if (e >= 0 && e < E) atomicAdd(&s_off[e], 1);
        else atomicOr(err, kErrBadExpert);
    }
    __syncthreads();
    const int c_e = tid < E ? s_off[tid] : 0;
    int t0, t1, t2;
    const int o0 = block_exclusive_scan(c_e, sh, &t0);
    const int o1 = block_exclusive_scan(round_up(c_e, kRowPad), sh, &t1);
    const int o2 = block_exclusive_scan(ceil_div(c_e, tile_tokens), sh, &t2);
    if (tid < E) {
        counts[tid] = c_e;
        offs[tid] = o0;
        poffs[tid] = o1;
        mtstart[tid] = o2;
        s_off[tid] = o0;
        s_poff[tid] = o1;
        for (int rr = o1 + c_e; rr < o1 + round_up(c_e, kRowPad); ++rr) row_src[rr] = -1;
        for (int t = 0; t < ceil_div(c_e, tile_tokens); ++t)
            mt_tab[o2 + t] = make_int4(tid, o1 + t * tile_tokens, min(tile_tokens, c_e - t * tile_tokens), 0);
    }
    if (tid == 0) {
        offs[E] = t0;
        poffs[E] = t1;
        mtstart[E] = t2;
    }
    for (int c0 = 0; c0 < nslots; c0 += blockDim.x) {
        for (int idx = tid; idx < 32 * E; idx += blockDim.x) s_wcnt[idx] = 0;
        __syncthreads();
        const int i = c0 + tid;
        const bool valid = i < nslots;
        const int e = valid ? ids[i] : -1;
        const bool good = valid && e >= 0 && e < E;
        const uint32_t mask = __match_any_sync(0xffffffffu, good ? e : E + lane);
        const int rank_w = __popc(mask & ((1u << lane) - 1u));
        if (good && lane == __ffs(mask) - 1) s_wcnt[warp * E + e] = __popc(mask);
        __syncthreads();
        if (good) {
            int p = s_run[e] + rank_w;
            for (int w2 = 0; w2 < warp; ++w2) p += s_wcnt[w2 * E + e];
            perm[s_off[e] + p] = i;
            inv[i] = s_poff[e] + p;
            row_src[s_poff[e] + p] = i;
        } else if (valid) {
            inv[i] = -1;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += blockDim.x) {
            int add = 0;
            for (int w2 = 0; w2 < 32; ++w2) add += s_wcnt[w2 * E + ee];
            s_run[ee] += add;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// a2 / a6 in the layer: per-row symmetric INT8 into the tiled token rows.  One CTA
// of 128 threads per grouped row; thread t owns the 16-value chunks t, t+128, ...
// of the row and keeps up to kRowCache of them in registers between the max pass
// and the quantisation pass.  Pad rows (row_src < 0) get zero codes and scale 0.
// ---------------------------------------------------------------------------
constexpr int kRowCache = 4;

struct Chunk16 {
    float v[16];
};

__device__ __forceinline__ void load_chunk(const uint16_t* row, int len, int k0, Chunk16& c) {
    if ((len & 15) == 0 && k0 + 16 <= len) {
        const uint4 p0 = *reinterpret_cast<const uint4*>(row + k0);
        const uint4 p1 = *reinterpret_cast<const uint4*>(row + k0 + 8);
        const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            c.v[2 * h] = bf16_to_f32((uint16_t)(pw[h] & 0xFFFFu));
            c.v[2 * h + 1] = bf16_to_f32((uint16_t)(pw[h] >> 16));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) c.v[i] = (k0 + i < len) ? bf16_to_f32(row[k0 + i]) : 0.f;
    }
}
__device__ __forceinline__ void load_chunk(const float* row, int len, int k0, Chunk16& c) {
    if ((len & 15) == 0 && k0 + 16 <= len) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 p = *reinterpret_cast<const float4*>(row + k0 + 4 * i);
            c.v[4 * i] = p.x; c.v[4 * i + 1] = p.y; c.v[4 * i + 2] = p.z; c.v[4 * i + 3] = p.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) c.v[i] = (k0 + i < len) ? row[k0 + i] : 0.f;
    }
}

template <int kCache, typename TIn>
__device__ __forceinline__ void quant_row_cta(const TIn* row, int len, int Kp, int r, int RB,
                                              int8_t* __restrict__ act, float* __restrict__ s) {
    __shared__ float red[4];
    const int nch = Kp / 16;
    const int G = Kp / kGroup;
    const int t = threadIdx.x;
    Chunk16 cache[kCache];
    float amax = 0.f;
    if (row != nullptr) {
#pragma unroll
        for (int c = 0; c < kCache; ++c) {
            const int ci = t + c * 128;
            if (ci < nch) {
                load_chunk(row, len, ci * 16, cache[c]);
#pragma unroll
                for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(cache[c].v[i]));
            }
        }
        for (int ci = t + kCache * 128; ci < nch; ci += 128) {
            Chunk16 tmp;
            load_chunk(row, len, ci * 16, tmp);
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(tmp.v[i]));
        }
    }
    amax = warp_max(amax);
    if ((t & 31) == 0) red[t >> 5] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float sc = __fdiv_rn(amax, 127.0f);
    const float rinv = __fdiv_rn(1.0f, sc);
    auto emit = [&](int ci, const Chunk16& c) {
        uint32_t out[4] = {0u, 0u, 0u, 0u};
        if (amax > 0.f) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t q = (uint32_t)(quant_i8_fast(c.v[i], sc, rinv) & 0xFF);
                out[i >> 2] |= q << (8 * (i & 3));
            }
        }
        *reinterpret_cast<uint4*>(act + act_offset(r, ci * 16, G, RB)) = make_uint4(out[0], out[1], out[2], out[3]);
    };
#pragma unroll
    for (int c = 0; c < kCache; ++c) {
        const int ci = t + c * 128;
        if (ci < nch) {
            if (row == nullptr) {
#pragma unroll
                for (int i = 0; i < 16; ++i) cache[c].v[i] = 0.f;
            }
            emit(ci, cache[c]);
        }
    }
    for (int ci = t + kCache * 128; ci < nch; ci += 128) {
        Chunk16 tmp;
        if (row != nullptr) load_chunk(row, len, ci * 16, tmp);
        else {
#pragma unroll
            for (int i = 0; i < 16; ++i) tmp.v[i] = 0.f;
        }
        emit(ci, tmp);
    }
    if (t == 0) s[r] = sc;
}

// x rows (bf16) -> INT8 rows in expert-grouped order.  CTA t < T quantises token t
// once (one read of x) and writes the codes to each of its k grouped rows; CTA T + e
// writes zero codes and scale 0 into the pad rows of expert e.
__global__ void __launch_bounds__(128) act_scatter_kernel(const uint16_t* __restrict__ x, int T, int H, int Kp, int k,
                                                          const int* __restrict__ inv,
                                                          const int* __restrict__ offs,
                                                          const int* __restrict__ poffs, int RB,
                                                          int8_t* __restrict__ act, float* __restrict__ s) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    const int nch = Kp / 16;
    const int G = Kp / kGroup;
    const int t = threadIdx.x;
    if ((int)blockIdx.x >= T) {
        const int e = (int)blockIdx.x - T;
        const int r0 = __ldg(poffs + e) + (__ldg(offs + e + 1) - __ldg(offs + e));
        const int r1 = __ldg(poffs + e + 1);
        for (int r = r0; r < r1; ++r) {
            for (int ci = t; ci < nch; ci += 128)
                *reinterpret_cast<uint4*>(act + act_offset(r, ci * 16, G, RB)) = make_uint4(0u, 0u, 0u, 0u);
            if (t == 0) s[r] = 0.f;
        }
        return;
    }
    const int tok = blockIdx.x;
    const uint16_t* row = x + (size_t)tok * H;
    __shared__ int dst[32];
    __shared__ float red[4];
    if (t < k) dst[t] = __ldg(inv + (size_t)tok * k + t);
    Chunk16 cache[kRowCache];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < kRowCache; ++c) {
        const int ci = t + c * 128;
        if (ci < nch) {
            load_chunk(row, H, ci * 16, cache[c]);
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(cache[c].v[i]));
        }
    }
    for (int ci = t + kRowCache * 128; ci < nch; ci += 128) {
        Chunk16 tmp;
        load_chunk(row, H, ci * 16, tmp);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(tmp.v[i]));
    }
    amax = warp_max(amax);
    if ((t & 31) == 0) red[t >> 5] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float sc = __fdiv_rn(amax, 127.0f);
    const float rinv = __fdiv_rn(1.0f, sc);
    auto emit = [&](int ci, const Chunk16& c) {
        uint32_t out[4] = {0u, 0u, 0u, 0u};
        if (amax > 0.f) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t q = (uint32_t)(quant_i8_fast(c.v[i], sc, rinv) & 0xFF);
                out[i >> 2] |= q << (8 * (i & 3));
            }
        }
        const uint4 o = make_uint4(out[0], out[1], out[2], out[3]);
        for (int j = 0; j < k; ++j) {
            const int r = dst[j];
            if (r >= 0) *reinterpret_cast<uint4*>(act + act_offset(r, ci * 16, G, RB)) = o;
        }
    };
#pragma unroll
    for (int c = 0; c < kRowCache; ++c) {
        const int ci = t + c * 128;
        if (ci < nch) emit(ci, cache[c]);
    }
    for (int ci = t + kRowCache * 128; ci < nch; ci += 128) {
        Chunk16 tmp;
        load_chunk(row, H, ci * 16, tmp);
        emit(ci, tmp);
    }
    if (t < k && dst[t] >= 0) s[dst[t]] = sc;
}

// h rows (fp32, SwiGLU output of the up GEMM) -> INT8 rows for the down GEMM
// (kCache chunks of 16 per thread stay in registers: 1 covers F <= 2048)
template <int kCache>
__global__ void __launch_bounds__(128) requant_kernel(const uint16_t* __restrict__ h, int ldh, int F, int Kp,
                                                      const int* __restrict__ row_src, const int* __restrict__ poffs,
                                                      int E, int RB, int8_t* __restrict__ act, float* __restrict__ s) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    const int r = blockIdx.x;
    if (r >= __ldg(poffs + E)) return;
    quant_row_cta<kCache, uint16_t>(row_src[r] < 0 ? nullptr : h + (size_t)r * ldh, F, Kp, r, RB, act, s);
}

// ---------------------------------------------------------------------------
// a8: out[t] = sum_j w[t][j] * y2[inv[t*k+j]]  (fp32, j ascending) -> bf16
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y2, int H, const int* __restrict__ inv,
                                                      const float* __restrict__ w, int T, int k,
                                                      uint16_t* __restrict__ out) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    __shared__ int rows[32];
    __shared__ float wts[32];
    const int t = blockIdx.x;
    if (threadIdx.x < k) {
        rows[threadIdx.x] = inv[(size_t)t * k + threadIdx.x];
        wts[threadIdx.x] = w[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    const bool vec = (H & 7) == 0;
    for (int c0 = threadIdx.x * 8; c0 < H; c0 += blockDim.x * 8) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 4
        for (int j = 0; j < k; ++j) {
            const int rr = rows[j];
            if (rr < 0) continue;
            const float wt = wts[j];
            const float* row = y2 + (size_t)rr * H + c0;
            if (vec) {
                const float4 a = *reinterpret_cast<const float4*>(row);
                const float4 b = *reinterpret_cast<const float4*>(row + 4);
                acc[0] = fmaf(wt, a.x, acc[0]); acc[1] = fmaf(wt, a.y, acc[1]);
                acc[2] = fmaf(wt, a.z, acc[2]); acc[3] = fmaf(wt, a.w, acc[3]);
                acc[4] = fmaf(wt, b.x, acc[4]); acc[5] = fmaf(wt, b.y, acc[5]);
                acc[6] = fmaf(wt, b.z, acc[6]); acc[7] = fmaf(wt, b.w, acc[7]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (c0 + i < H) acc[i] = fmaf(wt, row[i], acc[i]);
            }
        }
        uint16_t* o = out + (size_t)t * H + c0;
        if (vec) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                pk[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i])) |
                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1])) << 16);
            *reinterpret_cast<uint4*>(o) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (c0 + i < H) o[i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[i]));
        }
    }
}

// dense GEMM: copy INT8 rows into the tiled planes (pad rows zero) and describe
// them as one "expert" with M rows.
__global__ void __launch_bounds__(256) dense_prep_kernel(const int8_t* __restrict__ qa, int M, int Kq, int Kp, int tile_tokens,
                                                         int RB, int8_t* __restrict__ act, int4* mt_tab, int* n_mtiles) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    const int Mp = round_up(M, kRowPad);
    const int nch = Kp / 16;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int nmt = ceil_div(M, tile_tokens);
    if (idx == 0) *n_mtiles = nmt;
    if (idx < (size_t)nmt) mt_tab[idx] = make_int4(0, (int)idx * tile_tokens, min(tile_tokens, M - (int)idx * tile_tokens), 0);
    if (idx >= (size_t)Mp * nch) return;
    const int r = (int)(idx / nch);
    const int ci = (int)(idx % nch);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < M && ci * 16 < Kq) v = *reinterpret_cast<const uint4*>(qa + (size_t)r * Kq + ci * 16);
    *reinterpret_cast<uint4*>(act + act_offset(r, ci * 16, Kp / kGroup, RB)) = v;
}

// ---------------------------------------------------------------------------
// W4A16 token rows: bf16 values copied (not quantised) into the tiled bf16 layout
// of act16_offset, 16-row blocks, 8 values (16 bytes) per thread and step.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 load8_bf16(const uint16_t* row, int len, int k0) {
    if ((len & 7) == 0 && k0 + 8 <= len) return *reinterpret_cast<const uint4*>(row + k0);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = k0 + 2 * i < len ? row[k0 + 2 * i] : 0u;
        const uint32_t hi = k0 + 2 * i + 1 < len ? row[k0 + 2 * i + 1] : 0u;
        w[i] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// CTA t copies token t's row to each of its k grouped rows (pad K columns zero) and
// zeroes the pad columns [F, Fp) of the same rows of the h buffer, which the up
// projection's epilogue leaves unwritten (chunks that straddle F are zeroed whole;
// the epilogue writes their valid part afterwards, in stream order)
__global__ void __launch_bounds__(128) act_gather_bf16_kernel(const uint16_t* __restrict__ x, int H, int k,
                                                              const int* __restrict__ inv, uint8_t* __restrict__ x16,
                                                              uint8_t* __restrict__ h16, int F) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    const int Hp = round_up(H, kGroup), G1 = Hp / kGroup;
    const int Fp = round_up(F, kGroup), G2 = Fp / kGroup;
    const int tok = blockIdx.x;
    __shared__ int dst[32];
    if ((int)threadIdx.x < k) dst[threadIdx.x] = __ldg(inv + (size_t)tok * k + threadIdx.x);
    __syncthreads();
    const uint16_t* row = x + (size_t)tok * H;
    for (int ci = threadIdx.x; ci < Hp / 8; ci += blockDim.x) {
        const uint4 v = load8_bf16(row, H, ci * 8);
        for (int j = 0; j < k; ++j) {
            const int r = dst[j];
            if (r >= 0) *reinterpret_cast<uint4*>(x16 + act16_offset(r, ci * 8, G1, 16)) = v;
        }
    }
    for (int ci = F / 8 + threadIdx.x; ci < Fp / 8; ci += blockDim.x) {
        for (int j = 0; j < k; ++j) {
            const int r = dst[j];
            if (r >= 0) *reinterpret_cast<uint4*>(h16 + act16_offset(r, ci * 8, G2, 16)) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

// dense W4A16 GEMM: x rows into the tiled bf16 layout (pad rows and columns zero),
// described as one "expert" of 16-row tiles
__global__ void __launch_bounds__(256) dense_prep_bf16_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                              uint8_t* __restrict__ act16, int4* mt_tab,
                                                              int* n_mtiles) {
    grid_dep_wait();  // the previous kernel of the forward has completed
    const int Kp = round_up(K, kGroup), G = Kp / kGroup;
    const int Mp = round_up(M, kRowPad);
    const int nch = Kp / 8;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int nmt = ceil_div(M, 16);
    if (idx == 0) *n_mtiles = nmt;
    if (idx < (size_t)nmt) mt_tab[idx] = make_int4(0, (int)idx * 16, min(16, M - (int)idx * 16), 0);
    if (idx >= (size_t)Mp * nch) return;
    const int r = (int)(idx / nch);
    const int ci = (int)(idx % nch);
    const uint4 v = r < M ? load8_bf16(x + (size_t)r * K, K, ci * 8) : make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(act16 + act16_offset(r, ci * 8, G, 16)) = v;
}

}  // namespace

// ------------------------------- launchers ---------------------------------
cudaError_t launch_pack(const uint16_t* w, int E, int N, int K, int layout, int scheme, int group, uint8_t* packed,
                        uint8_t* codes, uint16_t* scale, uint16_t* zp, cudaStream_t stream) {
    const int G = k_padded_for(K, group) / kGroup;
    const int NT = layout == 1 ? ceil_div(N / 2, kTileRows / 2) : ceil_div(N, kTileRows);
    dim3 grid(G * kGroup / group, NT, E);
    uint8_t* blocks = packed + kHeaderBytes;
    if (group == 64)
        pack_kernel<64><<<grid, 128, 0, stream>>>(w, N, K, layout, scheme, NT, G, blocks, codes, scale, zp);
    else if (group == 256)
        pack_kernel<256><<<grid, 128, 0, stream>>>(w, N, K, layout, scheme, NT, G, blocks, codes, scale, zp);
    else
        pack_kernel<128><<<grid, 128, 0, stream>>>(w, N, K, layout, scheme, NT, G, blocks, codes, scale, zp);
    return cudaGetLastError();
}

cudaError_t launch_quant_act(const uint16_t* x, int T, int K, int8_t* q, float* s, cudaStream_t stream) {
    return launch_pdl(quant_act_kernel, ceil_div(T, 8), 256, 0, stream, x, T, K, round_up(K, kGroup), q, s);
}

cudaError_t launch_route_topk(const uint16_t* logits, int T, int E, int k, int32_t* ids, float* w,
                              cudaStream_t stream) {
    return launch_pdl(route_topk_kernel, ceil_div(T, 8), 256, 0, stream, logits, T, E, k, ids, w);
}

int perm_launch_count(int nslots) { return nslots <= kPermSmallSlots ? 1 : 3; }

cudaError_t launch_perm(const int32_t* ids, int nslots, int E, int tile_tokens, int* chist, int nchunk, int* counts,
                        int* offs, int* poffs, int* mtstart, int4* mt_tab, int* perm, int* inv, int* row_src,
                        uint32_t* err, cudaStream_t stream) {
    if (nslots <= kPermSmallSlots) {
        const size_t smem = (size_t)35 * E * sizeof(int);
        static int attr_done[64] = {0};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 0 || dev >= 64 || !attr_done[dev]) {
            const cudaError_t e = cudaFuncSetAttribute(perm_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       35 * kMaxExperts * (int)sizeof(int));
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) attr_done[dev] = 1;
        }
        return launch_pdl(perm_small_kernel, 1, 1024, smem, stream, ids, nslots, E, tile_tokens, counts, offs, poffs,
                          mtstart, mt_tab, perm, inv, row_src, err);
    }
    cudaError_t e = launch_pdl(perm_hist_kernel, nchunk, kPermChunk, 0, stream, ids, nslots, E, chist, err);
    if (e != cudaSuccess) return e;
    e = launch_pdl(perm_scan_kernel, 1, 1024, 0, stream, chist, nchunk, E, tile_tokens, counts, offs, poffs, mtstart,
                   mt_tab, row_src);
    if (e != cudaSuccess) return e;
    return launch_pdl(perm_scatter_kernel, nchunk, kPermChunk, 0, stream, ids, nslots, E, chist, offs, poffs, perm, inv,
                      row_src);
}

cudaError_t launch_act_scatter(const uint16_t* x, int T, int H, int Kp, int k, const int* inv, const int* offs,
                               const int* poffs, int E, int rb, int8_t* act, float* s, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    return launch_pdl(act_scatter_kernel, T + E, 128, 0, stream, x, T, H, Kp, k, inv, offs, poffs, rb, act, s);
}

cudaError_t launch_requant(const uint16_t* h, int ldh, int F, int Kp, const int* row_src, const int* poffs, int E,
                           int rows_cap, int rb, int8_t* act, float* s, cudaStream_t stream) {
    if (rows_cap == 0) return cudaSuccess;
    if (F <= 128 * 16)
        return launch_pdl(requant_kernel<1>, rows_cap, 128, 0, stream, h, ldh, F, Kp, row_src, poffs, E, rb, act, s);
    return launch_pdl(requant_kernel<kRowCache>, rows_cap, 128, 0, stream, h, ldh, F, Kp, row_src, poffs, E, rb, act, s);
}

cudaError_t launch_combine(const float* y2, int H, const int* inv, const float* w, int T, int k, uint16_t* out,
                           cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    return launch_pdl(combine_kernel, T, 256, 0, stream, y2, H, inv, w, T, k, out);
}

cudaError_t launch_dense_prep(const int8_t* qa, int M, int Kq, int Kp, int tile_tokens, int rb, int8_t* act, int4* mt_tab,
                              int* n_mtiles, cudaStream_t stream) {
    const size_t n = (size_t)round_up(M, kRowPad) * (Kp / 16);
    return launch_pdl(dense_prep_kernel, (unsigned)((n + 255) / 256 + 1), 256, 0, stream, qa, M, Kq, Kp, tile_tokens, rb,
                      act, mt_tab, n_mtiles);
}

cudaError_t launch_dense_prep_bf16(const uint16_t* x, int M, int K, uint8_t* act16, int4* mt_tab, int* n_mtiles,
                                   cudaStream_t stream) {
    const size_t n = (size_t)round_up(M, kRowPad) * (round_up(K, kGroup) / 8);
    return launch_pdl(dense_prep_bf16_kernel, (unsigned)((n + 255) / 256 + 1), 256, 0, stream, x, M, K, act16, mt_tab,
                      n_mtiles);
}

cudaError_t launch_act_gather_bf16(const uint16_t* x, int T, int H, int k, const int* inv, uint8_t* x16, uint8_t* h16,
                                   int F, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    return launch_pdl(act_gather_bf16_kernel, T, 128, 0, stream, x, H, k, inv, x16, h16, F);
}

}  // namespace w4a8

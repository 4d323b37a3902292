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
// a1: weight quantisation + packing.  One block per (group g, tile t, matrix e);
// thread r quantises tiled row r's 128 weights of group g.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) pack_kernel(const uint16_t* __restrict__ w, int N, int K, int layout, int NT,
                                                   int G, uint8_t* __restrict__ blocks, uint8_t* __restrict__ codes_out,
                                                   uint16_t* __restrict__ scale_out, uint16_t* __restrict__ zp_out) {
    const int g = blockIdx.x, t = blockIdx.y, e = blockIdx.z;
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
    float v[kGroup];
    const int k0 = g * kGroup;
    if (valid) {
        const uint16_t* row = w + ((size_t)e * N + src) * (size_t)K;
        if ((K & 7) == 0 && k0 + kGroup <= K) {
#pragma unroll
            for (int i = 0; i < kGroup / 8; ++i) {
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
            for (int i = 0; i < kGroup; ++i) v[i] = (k0 + i < K) ? bf16_to_f32(row[k0 + i]) : 0.f;
        }
    } else {
#pragma unroll
        for (int i = 0; i < kGroup; ++i) v[i] = 0.f;
    }
    // range widened to contain 0
    float mn = 0.f, mx = 0.f;
#pragma unroll
    for (int i = 0; i < kGroup; ++i) {
        mn = fminf(mn, v[i]);
        mx = fmaxf(mx, v[i]);
    }
    // scale = (max - min) / (2^4 - 1), stored as fp16; the fp16 value is the one used
    const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    __half sh = __float2half_rn(s32);
    if (__half2float(sh) == 0.f) sh = __float2half_rn(1.0f);
    const float shf = __half2float(sh);
    // zero_point = round(-min / scale)
    const int zp = (int)fminf(fmaxf(rintf(__fdiv_rn(-mn, shf)), 0.f), 15.f);
    // index = clamp(round(w / scale) + zero_point, 0, 15)
    uint32_t code[kGroup];
#pragma unroll
    for (int i = 0; i < kGroup; ++i) {
        const int c = (int)rintf(__fdiv_rn(v[i], shf)) + zp;
        code[i] = (uint32_t)min(max(c, 0), 15);
    }
    // tiled block: word i (K = 8i..8i+7): byte b = code[8i+b] | code[8i+4+b] << 4
    uint8_t* blk = blocks + ((size_t)(e * NT + t) * G + g) * kBlockBytes;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t wd[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = 4 * c + q;
            uint32_t x = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) x |= (code[8 * i + b] | (code[8 * i + 4 + b] << 4)) << (8 * b);
            wd[q] = x;
        }
        *reinterpret_cast<uint4*>(blk + code_chunk_offset(r, c)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    }
    reinterpret_cast<__half*>(blk + kScaleOff)[r] = sh;
    reinterpret_cast<__half*>(blk + kZpOff)[r] = __float2half_rn((float)zp);

    if (valid) {
        const int Kp = G * kGroup;
        if (codes_out != nullptr) {
            uint8_t* dst = codes_out + ((size_t)e * N + src) * (size_t)(Kp / 2) + (size_t)g * (kGroup / 2);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t wd[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t x = 0;
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const int j = 16 * c + 4 * q + b;  // canonical byte j: code[2j] | code[2j+1] << 4
                        x |= (code[2 * j] | (code[2 * j + 1] << 4)) << (8 * b);
                    }
                    wd[q] = x;
                }
                *reinterpret_cast<uint4*>(dst + 16 * c) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            }
        }
        if (scale_out != nullptr) scale_out[((size_t)e * N + src) * G + g] = __half_as_ushort(sh);
        if (zp_out != nullptr) zp_out[((size_t)e * N + src) * G + g] = __half_as_ushort(__float2half_rn((float)zp));
    }
    if (e == 0 && t == 0 && g == 0 && r == 0) {
        PackHeader* h = reinterpret_cast<PackHeader*>(blocks - kHeaderBytes);
        h->magic = kPackMagic;
        h->version = 1;
        h->layout = (uint32_t)layout;
        h->E = gridDim.z;
        h->N = (uint32_t)N;
        h->K = (uint32_t)K;
        h->Kp = (uint32_t)(G * kGroup);
        h->G = (uint32_t)G;
        h->NT = (uint32_t)NT;
        h->rows_per_tile = kTileRows;
        h->block_bytes = kBlockBytes;
    }
}

// ---------------------------------------------------------------------------
// a2: per-token INT8, natural layout [T][Kp].  One warp per row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_act_kernel(const uint16_t* __restrict__ x, int T, int K, int Kp,
                                                        int8_t* __restrict__ q, float* __restrict__ s) {
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= T) return;
    const uint16_t* xr = x + (size_t)row * K;
    float amax = 0.f;
    for (int k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(bf16_to_f32(xr[k])));
    amax = warp_max(amax);
    const float sc = __fdiv_rn(amax, 127.0f);
    int8_t* qr = q + (size_t)row * Kp;
    for (int k = lane; k < Kp; k += 32) {
        int c = 0;
        if (k < K && amax > 0.f) c = quant_i8(bf16_to_f32(xr[k]), sc);
        qr[k] = (int8_t)c;
    }
    if (lane == 0) s[row] = sc;
}

// ---------------------------------------------------------------------------
// a3: top-k softmax routing.  One warp per token; lane l owns experts l, l+32, ...
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) route_topk_kernel(const uint16_t* __restrict__ logits, int T, int E, int k,
                                                         int32_t* __restrict__ ids, float* __restrict__ wout) {
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

// ---------------------------------------------------------------------------
// a2 in the layer: per-token INT8 of x, written straight into the tiled planes in
// expert-grouped row order (one warp per grouped row; pad rows get zeros).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) act_scatter_kernel(const uint16_t* __restrict__ x, int H, int k,
                                                          const int* __restrict__ row_src,
                                                          const int* __restrict__ poffs, int E,
                                                          int RB, int8_t* __restrict__ act,
                                                          float* __restrict__ s) {
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= __ldg(poffs + E)) return;
    const int Hp = round_up(H, kGroup);
    const int nchunks = Hp / 16;  // 16-byte chunks of the row
    const int src = row_src[r];
    if (src < 0) {
        for (int ci = lane; ci < nchunks; ci += 32)
            *reinterpret_cast<uint4*>(act + act_offset(r, ci * 16, Hp / kGroup, RB)) = make_uint4(0, 0, 0, 0);
        if (lane == 0) s[r] = 0.f;
        return;
    }
    const uint16_t* xr = x + (size_t)(src / k) * H;
    float amax = 0.f;
    const bool vec = (H & 15) == 0;
    if (vec) {
        for (int ci = lane; ci < H / 8; ci += 32) {
            const uint4 p = *reinterpret_cast<const uint4*>(xr + 8 * ci);
            const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int h = 0; h < 4; ++h)
                amax = fmaxf(amax, fmaxf(fabsf(bf16_to_f32((uint16_t)(pw[h] & 0xFFFFu))),
                                         fabsf(bf16_to_f32((uint16_t)(pw[h] >> 16)))));
        }
    } else {
        for (int kk = lane; kk < H; kk += 32) amax = fmaxf(amax, fabsf(bf16_to_f32(xr[kk])));
    }
    amax = warp_max(amax);
    const float sc = __fdiv_rn(amax, 127.0f);
    for (int base = 0; base < nchunks; base += 32) {
        const int ci = base + lane;
        const int k0 = ci * 16;
        uint32_t out[4] = {0u, 0u, 0u, 0u};
        if (ci < nchunks && amax > 0.f) {
            float vals[16];
            if (vec && k0 < H) {
                const uint4 p0 = *reinterpret_cast<const uint4*>(xr + k0);
                const uint4 p1 = *reinterpret_cast<const uint4*>(xr + k0 + 8);
                const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    vals[2 * h] = bf16_to_f32((uint16_t)(pw[h] & 0xFFFFu));
                    vals[2 * h + 1] = bf16_to_f32((uint16_t)(pw[h] >> 16));
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) vals[i] = (k0 + i < H) ? bf16_to_f32(xr[k0 + i]) : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t c = (uint32_t)(quant_i8(vals[i], sc) & 0xFF);
                out[i >> 2] |= c << (8 * (i & 3));
            }
        }
        if (ci < nchunks)
            *reinterpret_cast<uint4*>(act + act_offset(r, k0, Hp / kGroup, RB)) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (lane == 0) s[r] = sc;
}

// ---------------------------------------------------------------------------
// a6 (second half): requantise h per row (max |h| over the row, then INT8 codes).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) requant_kernel(const float* __restrict__ h, int ldh, int F,
                                                      const int* __restrict__ row_src, const int* __restrict__ poffs,
                                                      int E, int RB, int8_t* __restrict__ act,
                                                      float* __restrict__ s) {
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= __ldg(poffs + E)) return;
    const int Fp = round_up(F, kGroup);
    const int nchunks = Fp / 16;
    const bool live = row_src[r] >= 0;
    const float* hr = h + (size_t)r * ldh;
    const bool vec = (F & 15) == 0;
    float amax = 0.f;
    if (live) {
        if (vec) {
            for (int i = lane; i < F / 4; i += 32) {
                const float4 p = *reinterpret_cast<const float4*>(hr + 4 * i);
                amax = fmaxf(amax, fmaxf(fmaxf(fabsf(p.x), fabsf(p.y)), fmaxf(fabsf(p.z), fabsf(p.w))));
            }
        } else {
            for (int i = lane; i < F; i += 32) amax = fmaxf(amax, fabsf(hr[i]));
        }
        amax = warp_max(amax);
    }
    const float sc = __fdiv_rn(amax, 127.0f);
    for (int base = 0; base < nchunks; base += 32) {
        const int ci = base + lane;
        const int k0 = ci * 16;
        uint32_t out[4] = {0u, 0u, 0u, 0u};
        if (ci < nchunks && amax > 0.f) {
            float vals[16];
            if (vec && k0 < F) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 p = *reinterpret_cast<const float4*>(hr + k0 + 4 * i);
                    vals[4 * i] = p.x; vals[4 * i + 1] = p.y; vals[4 * i + 2] = p.z; vals[4 * i + 3] = p.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) vals[i] = (k0 + i < F) ? hr[k0 + i] : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t c = (uint32_t)(quant_i8(vals[i], sc) & 0xFF);
                out[i >> 2] |= c << (8 * (i & 3));
            }
        }
        if (ci < nchunks)
            *reinterpret_cast<uint4*>(act + act_offset(r, k0, Fp / kGroup, RB)) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (lane == 0) s[r] = sc;
}

// ---------------------------------------------------------------------------
// a8: out[t] = sum_j w[t][j] * y2[inv[t*k+j]]  (fp32, j ascending) -> bf16
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y2, int H, const int* __restrict__ inv,
                                                      const float* __restrict__ w, int T, int k,
                                                      uint16_t* __restrict__ out) {
    const int cols8 = (H + 7) >> 3;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (size_t)T * cols8) return;
    const int t = (int)(idx / cols8);
    const int c0 = (int)(idx % cols8) * 8;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    const bool vec = (H & 7) == 0;
    for (int j = 0; j < k; ++j) {
        const int rr = inv[(size_t)t * k + j];
        if (rr < 0) continue;
        const float wt = w[(size_t)t * k + j];
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

// dense GEMM: copy INT8 rows into the tiled planes (pad rows zero) and describe
// them as one "expert" with M rows.
__global__ void __launch_bounds__(256) dense_prep_kernel(const int8_t* __restrict__ qa, int M, int Kp, int tile_tokens,
                                                         int RB, int8_t* __restrict__ act, int4* mt_tab, int* n_mtiles) {
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
    if (r < M) v = *reinterpret_cast<const uint4*>(qa + (size_t)r * Kp + ci * 16);
    *reinterpret_cast<uint4*>(act + act_offset(r, ci * 16, Kp / kGroup, RB)) = v;
}

}  // namespace

// ------------------------------- launchers ---------------------------------
cudaError_t launch_pack(const uint16_t* w, int E, int N, int K, int layout, uint8_t* packed, uint8_t* codes,
                        uint16_t* scale, uint16_t* zp, cudaStream_t stream) {
    const int G = ceil_div(K, kGroup);
    const int NT = layout == 1 ? ceil_div(N / 2, kTileRows / 2) : ceil_div(N, kTileRows);
    dim3 grid(G, NT, E);
    pack_kernel<<<grid, 128, 0, stream>>>(w, N, K, layout, NT, G, packed + kHeaderBytes, codes, scale, zp);
    return cudaGetLastError();
}

cudaError_t launch_quant_act(const uint16_t* x, int T, int K, int8_t* q, float* s, cudaStream_t stream) {
    quant_act_kernel<<<ceil_div(T, 8), 256, 0, stream>>>(x, T, K, round_up(K, kGroup), q, s);
    return cudaGetLastError();
}

cudaError_t launch_route_topk(const uint16_t* logits, int T, int E, int k, int32_t* ids, float* w,
                              cudaStream_t stream) {
    route_topk_kernel<<<ceil_div(T, 8), 256, 0, stream>>>(logits, T, E, k, ids, w);
    return cudaGetLastError();
}

cudaError_t launch_perm(const int32_t* ids, int nslots, int E, int tile_tokens, int* chist, int nchunk, int* counts,
                        int* offs, int* poffs, int* mtstart, int4* mt_tab, int* perm, int* inv, int* row_src,
                        uint32_t* err, cudaStream_t stream) {
    perm_hist_kernel<<<nchunk, kPermChunk, 0, stream>>>(ids, nslots, E, chist, err);
    perm_scan_kernel<<<1, 1024, 0, stream>>>(chist, nchunk, E, tile_tokens, counts, offs, poffs, mtstart, mt_tab,
                                             row_src);
    perm_scatter_kernel<<<nchunk, kPermChunk, 0, stream>>>(ids, nslots, E, chist, offs, poffs, perm, inv, row_src);
    return cudaGetLastError();
}

cudaError_t launch_act_scatter(const uint16_t* x, int H, int k, const int* row_src, const int* poffs, int E,
                               int rows_cap, int rb, int8_t* act, float* s, cudaStream_t stream) {
    act_scatter_kernel<<<ceil_div(rows_cap, 8), 256, 0, stream>>>(x, H, k, row_src, poffs, E, rb, act, s);
    return cudaGetLastError();
}

cudaError_t launch_requant(const float* h, int ldh, int F, const int* row_src, const int* poffs, int E,
                           int rows_cap, int rb, int8_t* act, float* s, cudaStream_t stream) {
    requant_kernel<<<ceil_div(rows_cap, 8), 256, 0, stream>>>(h, ldh, F, row_src, poffs, E, rb, act, s);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float* y2, int H, const int* inv, const float* w, int T, int k, uint16_t* out,
                           cudaStream_t stream) {
    const size_t n = (size_t)T * ((H + 7) / 8);
    if (n == 0) return cudaSuccess;
    combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(y2, H, inv, w, T, k, out);
    return cudaGetLastError();
}

cudaError_t launch_dense_prep(const int8_t* qa, int M, int Kp, int tile_tokens, int rb, int8_t* act, int4* mt_tab,
                              int* n_mtiles, cudaStream_t stream) {
    const size_t n = (size_t)round_up(M, kRowPad) * (Kp / 16);
    dense_prep_kernel<<<(unsigned)((n + 255) / 256 + 1), 256, 0, stream>>>(qa, M, Kp, tile_tokens, rb, act, mt_tab,
                                                                          n_mtiles);
    return cudaGetLastError();
}

}  // namespace w4a8

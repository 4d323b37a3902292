// Host-side declarations shared by the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace w4a8 {

// Arguments of the grouped W4A8 GEMM (one launch = one projection of every expert).
struct GemmArgs {
    const uint8_t* wblocks;   // packed weight blocks (after the 256-byte header)
    int NT;                   // 128-row tiles per weight matrix
    int G;                    // 128-wide K groups
    const int8_t* act;        // tiled INT8 token rows, layout [rows/RB][G][RB][128] (see act_offset)
    size_t act_plane;         // bytes between consecutive K groups of a row block (RB * 128)
    size_t act_rb_stride;     // bytes between consecutive row blocks (G * RB * 128)
    const float* act_scale;   // token scale per row
    const int4* mt_tab;       // per row tile: (expert, first row, rows, 0)
    const int* n_mtiles;      // number of row tiles (device)
    int mode;                 // 0: y = fp32 [rows][ldo];  1: SwiGLU -> h [rows][ldo];  2: like 0
    float* out;               // mode 1 with out_bf16: bf16 values, `out` cast to uint16_t*
    int ldo;
    int nvalid;               // valid output columns (N, or F for mode 1)
    int32_t* partials;        // mode 0 only, optional: exact INT32 partials [rows][nvalid][G]
    uint32_t* err;            // device error word
    long long wait_limit;     // clock cycles a bounded wait may last (> 0; normally ~2 s)
    uint32_t debug;           // test hook: bit 0 = CTA 0 issues no copy for its first step
    // W4A16 only (bf16 token rows, layout act16_offset): mode 1 writes h as bf16 into
    // the tiled token rows of out16 (16-row blocks, out16_G K groups) instead of `out`
    uint8_t* out16;
    int out16_G;
    // weights per scale along K in the packed blocks: 64, 128 (also 0) or 256; G above
    // counts 128-wide planes, the partials [rows][nvalid][G * 128 / group] groups
    int group;
    int out_bf16;             // mode 1: write h as bf16 (RNE of the fp32 result)
};

// Test hook of the failure-detection path (w4a8_debug_inject): while set on the
// calling host thread, GEMM launches get this wait limit and debug word.
struct DebugInject {
    uint32_t flags = 0;
    long long wait_limit = 0;
};

// launchers (all asynchronous on `stream`); return the cudaGetLastError() of the launch
// Tokens per GEMM tile (16: decode kernel, 128: wide-tile kernel) for a given mean
// number of tokens per expert; the permutation's row-tile table must be built with
// the same value, and the token rows laid out in blocks of act_block_rows() rows.
int gemm_tile_tokens(int avg_tokens_per_expert);
inline int act_block_rows(int tile_tokens, int rows_cap) { return tile_tokens == 16 ? 16 : rows_cap; }
cudaError_t launch_gemm(const GemmArgs& a, int tile_tokens, int num_ctas, cudaStream_t stream);
cudaError_t launch_gemm_decode(const GemmArgs& a, int num_ctas, cudaStream_t stream);
// W4A16: the decode-tile kernel on bf16 token rows (act points at act16_offset rows with
// 16-row blocks, act_rb_stride = G * 16 * 256); no partials; mode 1 needs out16
cudaError_t launch_gemm_w4a16(const GemmArgs& a, int num_ctas, cudaStream_t stream);

// scheme: 0 asymmetric (min/max), 1 symmetric, 2 asymmetric on the 0.1th..99.9th percentiles
// group: weights per scale along K (64, 128 or 256)
cudaError_t launch_pack(const uint16_t* w, int E, int N, int K, int layout, int scheme, int group, uint8_t* packed,
                        uint8_t* codes, uint16_t* scale, uint16_t* zp, cudaStream_t stream);
cudaError_t launch_quant_act(const uint16_t* x, int T, int K, int8_t* q, float* s, cudaStream_t stream);
cudaError_t launch_route_topk(const uint16_t* logits, int T, int E, int k, int32_t* ids, float* w,
                              cudaStream_t stream);

// MoE pipeline pieces
cudaError_t launch_perm(const int32_t* ids, int nslots, int E, int tile_tokens, int* chist, int nchunk, int* counts,
                        int* offs, int* poffs, int* mtstart, int4* mt_tab, int* perm, int* inv, int* row_src,
                        uint32_t* err, cudaStream_t stream);
// capacity of the row-tile table for a layer: sum over experts of ceil(count / tile)
// <= nslots / tile + E, with tiles of at least 16 rows
inline int mt_tab_capacity(int nslots, int E) { return nslots / 16 + E + 1; }
// Kp: the padded row length of the tiled rows (a multiple of 128, >= H)
cudaError_t launch_act_scatter(const uint16_t* x, int T, int H, int Kp, int k, const int* inv, const int* offs,
                               const int* poffs, int E, int rb, int8_t* act, float* s, cudaStream_t stream);
// h: bf16 SwiGLU output rows of ldh values
cudaError_t launch_requant(const uint16_t* h, int ldh, int F, int Kp, const int* row_src, const int* poffs, int E,
                           int rows_cap, int rb, int8_t* act, float* s, cudaStream_t stream);
// y2: fp32 expert outputs [rows][H]
cudaError_t launch_combine(const float* y2, int H, const int* inv, const float* w, int T, int k, uint16_t* out,
                           cudaStream_t stream);
// qa rows of Kq columns into tiled rows of Kp >= Kq columns (the rest zero)
cudaError_t launch_dense_prep(const int8_t* qa, int M, int Kq, int Kp, int tile_tokens, int rb, int8_t* act, int4* mt_tab,
                              int* n_mtiles, cudaStream_t stream);
// W4A16 token rows: x bf16 [M][K] -> tiled bf16 rows (16-row blocks, K padded with
// zeros) described as one "expert" of 16-row tiles
cudaError_t launch_dense_prep_bf16(const uint16_t* x, int M, int K, uint8_t* act16, int4* mt_tab, int* n_mtiles,
                                   cudaStream_t stream);
// W4A16 layer: each token's bf16 row copied to its k grouped rows (tiled, 16-row
// blocks, pad K columns zero); the pad K columns [F, Fp) of the same rows of the h
// buffer are zeroed too
cudaError_t launch_act_gather_bf16(const uint16_t* x, int T, int H, int k, const int* inv, uint8_t* x16, uint8_t* h16,
                                   int F, cudaStream_t stream);

constexpr int kPermChunk = 256;       // slots per permutation chunk (multi-CTA path)
constexpr int kPermSmallSlots = 16384;  // up to this many slots the permutation runs in one CTA
int perm_launch_count(int nslots);

// INT8 KV cache (kv_int8.cu)
int kv_max_heads();
cudaError_t launch_kv_calibrate(const uint16_t* x, int T, int H, int D, float* scale, int sm_count,
                                cudaStream_t stream);
cudaError_t launch_kv_quant(const uint16_t* x, int T, int H, int D, const float* scale, int8_t* q, int sm_count,
                            cudaStream_t stream);
cudaError_t launch_kv_dequant(const int8_t* q, int T, int H, int D, const float* scale, uint16_t* x, int sm_count,
                              cudaStream_t stream);

}  // namespace w4a8

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
    const int8_t* act;        // tiled INT8 activation planes [G][rows][128]
    size_t act_plane;         // bytes per plane
    const float* act_scale;   // token scale per row
    const int* counts;        // [E] rows per expert
    const int* poffs;         // [E+1] first row of each expert (16-row aligned)
    const int* mtstart;       // [E+1] prefix sum of row tiles (kBN rows) per expert
    int E;
    int mode;                 // 0: y = fp32 [rows][ldo];  1: SwiGLU -> h fp32 + row amax;  2: like 0
    float* out;
    int ldo;
    int nvalid;               // valid output columns (N, or F for mode 1)
    uint32_t* amax;           // mode 1: per-row max |h| (float bits), zeroed beforehand
    int32_t* partials;        // mode 0 only, optional: exact INT32 partials [rows][nvalid][G]
    uint32_t* err;            // device error word
};

// launchers (all asynchronous on `stream`); return the cudaGetLastError() of the launch
cudaError_t launch_gemm(const GemmArgs& a, int num_ctas, cudaStream_t stream);
size_t gemm_smem_bytes();

cudaError_t launch_pack(const uint16_t* w, int E, int N, int K, int layout, uint8_t* packed,
                        uint8_t* codes, uint16_t* scale, uint16_t* zp, cudaStream_t stream);
cudaError_t launch_quant_act(const uint16_t* x, int T, int K, int8_t* q, float* s, cudaStream_t stream);
cudaError_t launch_route_topk(const uint16_t* logits, int T, int E, int k, int32_t* ids, float* w,
                              cudaStream_t stream);

// MoE pipeline pieces
struct MoeWs;  // workspace carve-up, defined in api.cu
cudaError_t launch_perm(const int32_t* ids, int nslots, int E, int* chist, int nchunk, int* counts, int* offs,
                        int* poffs, int* mtstart, int* perm, int* inv, int* row_src, uint32_t* err,
                        cudaStream_t stream);
cudaError_t launch_act_scatter(const uint16_t* x, int H, int k, const int* row_src, const int* poffs, int E,
                               int rows_cap, int8_t* act, size_t plane, float* s, uint32_t* amax,
                               cudaStream_t stream);
cudaError_t launch_requant(const float* h, int ldh, int F, const int* row_src, const int* poffs, int E,
                           int rows_cap, const uint32_t* amax, int8_t* act, size_t plane, float* s,
                           cudaStream_t stream);
cudaError_t launch_combine(const float* y2, int H, const int* inv, const float* w, int T, int k, uint16_t* out,
                           cudaStream_t stream);
cudaError_t launch_dense_prep(const int8_t* qa, int M, int Kp, int8_t* act, size_t plane, int* counts,
                              int* poffs, int* mtstart, cudaStream_t stream);

constexpr int kPermChunk = 256;  // slots per permutation chunk

}  // namespace w4a8

/*
 * w4a8.h -- C ABI of libw4a8.so: the W4A8 mixture-of-experts expert FFN on
 * NVIDIA B200 (sm_100a).
 *
 * The method (sources: «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解», pptc.cn, sections
 * 2.1-2.3 and 3.2; the Kimi 2.7T MoE W4A8 article, hotelren.com 5173946, section
 * 4.3; the LLM quantisation primer, hotelren.com 5982361, section 2.1):
 *   - weights are group-wise asymmetric INT4, 128 weights per group along K, one
 *     fp16 scale and one fp16 zero point per group:
 *       scale = (max - min) / 15, zp = round(-min / scale),
 *       index = clamp(round(w / scale) + zp, 0, 15),  w ~= (index - zp) * scale;
 *     two indices per byte, the first in the low nibble;
 *   - activations are quantised per token to symmetric INT8 at run time:
 *       s = max|x| / 127, q = clamp(round(x / s), -127, 127);
 *   - the product is an INT8 x INT8 matrix multiply with INT32 accumulation, one
 *     INT32 partial per 128-wide K group, scaled back to floating point by
 *     (weight scale of the group) x (token scale).
 * "round" is round-half-to-even everywhere; the min/max range of a weight group
 * is widened to contain 0; an fp16 scale that rounds to 0 is stored as 1.
 * The packer also offers a symmetric INT4 scheme and a percentile-clipped range
 * (W4A8_PACK_SYMMETRIC, W4A8_PACK_CLIP999) in the same packed format, and the
 * library carries an INT8 KV cache with static per-head scales (w4a8_kv_*).
 *
 * Conventions for every entry point:
 *   - pointers are DEVICE pointers owned by the caller unless a parameter says
 *     "host"; the library allocates nothing -- scratch memory is the caller's
 *     workspace `ws`, sized by the matching *_workspace_bytes() function;
 *   - device pointers must be 16-byte aligned (W4A8_EALIGN otherwise), workspace
 *     and packed-weight pointers 256-byte aligned;
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); all work is
 *     enqueued asynchronously on it and the call returns after launching;
 *   - the return value reports argument validation and launch errors only
 *     (w4a8_status).  Faults detected on the device (a bounded wait that ran out,
 *     an expert id out of range) set a word in the workspace that
 *     w4a8_last_device_error() reads back;
 *   - no CUDA context is created or changed, no exception crosses the ABI, and
 *     there is no CPU fallback: an unsupported shape returns W4A8_EUNSUPPORTED.
 */
#ifndef W4A8_H
#define W4A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4A8_OK = 0,
    W4A8_EINVAL = -1,       /* bad argument (null pointer, negative size, k > E, ...) */
    W4A8_EALIGN = -2,       /* a pointer is not aligned as required */
    W4A8_ENOSPACE = -3,     /* packed buffer or workspace smaller than required */
    W4A8_ECUDA = -4,        /* a CUDA runtime call or kernel launch failed */
    W4A8_EUNSUPPORTED = -5, /* shape outside what the kernels handle */
    W4A8_ETIMEOUT = -6,     /* (device error word) a bounded wait in a kernel ran out */
    W4A8_EDEVICE = -7       /* (device error word) bad data seen on the device */
} w4a8_status;

/* Packed-weight layouts.
 * W4A8_LAYOUT_PLAIN : rows in order (a plain linear layer, or an expert's down
 *                     projection [H][F]).
 * W4A8_LAYOUT_GATEUP: the expert's up projection [2F][H] whose rows [0,F) are the
 *                     gate projection and rows [F,2F) the up projection; each
 *                     128-row tile holds 64 gate rows interleaved with the 64
 *                     matching up rows, so that SwiGLU can be applied in the
 *                     GEMM's epilogue.                                            */
enum { W4A8_LAYOUT_PLAIN = 0, W4A8_LAYOUT_GATEUP = 1 };

/* Quantisation scheme flag, OR-ed into the `layout` argument of w4a8_packed_bytes
 * and w4a8_pack_weights.
 * Without it (the default): asymmetric INT4 per 128-wide group along K (the
 *   «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» page, section 2.2): scale = (max - min)/15
 *   over the group's range widened to contain 0, stored as fp16 and used for the
 *   codes; zero_point = round(-min/scale); code = clamp(round(w/scale) + zp, 0, 15).
 * W4A8_PACK_SYMMETRIC: symmetric INT4 (the LLM quantisation primer at
 *   hotelren.com/news/5982361, section 2.1, with b = 4): scale = max|w|/7 (fp16),
 *   q = clamp(round(w/scale), -7, 7), stored as code q + 8 with zero point 8.
 * W4A8_PACK_CLIP999: asymmetric as the default, but over the range from the group's
 *   0.1th to its 99.9th percentile (same page, section 2.2: a percentile keeps
 *   outliers from stretching the range), each by linear interpolation between the
 *   two nearest order statistics (positions 0.127 and 126.873 of the 128 sorted
 *   values) evaluated in fp32 as a + f*(b - a), f = 0.127f / 0.873f; values outside
 *   the range land on codes 0 / 15 through the clamp.
 * At most one of these may be set.  All write the same tiled format, so w4a8_gemm and
 * w4a8_moe_forward take any of them.  Rounding is half to even; divisions are
 * correctly rounded fp32; an fp16 scale that rounds to 0 is replaced by 1.
 * Group size flags (the same page, section 4.3: groups of 64, 128 and 256 weights
 * were tried; the Kimi 2.7T MoE W4A8 article, hotelren.com 5173946, section 5: 128 or
 * 256 is usual): W4A8_PACK_GROUP64 / W4A8_PACK_GROUP256 give each 64 / 256 weights
 * along K their own scale and zero point instead of each 128 (with the asymmetric or
 * the symmetric scheme; the percentile range is defined for 128-value groups only).
 * Such weights are multiplied with w4a8_gemm_g / w4a8_moe_forward_g, which take the
 * group size, and K is padded to a whole number of groups (and of 128).           */
enum { W4A8_PACK_SYMMETRIC = 0x100, W4A8_PACK_CLIP999 = 0x200, W4A8_PACK_GROUP64 = 0x400,
       W4A8_PACK_GROUP256 = 0x800 };

/* Bytes of a packed weight buffer for E matrices of shape [N][K] in `layout`:
 * a 256-byte header, then one block per (matrix, 128-row tile, 128-wide K plane):
 * 8192 bytes of 4-bit codes, then 128 fp16 scales and 128 fp16 zero points of the
 * plane's group (8704 bytes).  Group 64: the plane holds two groups, and the scales
 * and zero points of the second follow those of the first (9216 bytes).  Group 256:
 * both planes of a group carry its scales and zero points (8704 bytes).  K is padded
 * to a multiple of 128 and of the group (zero weights).  Returns 0 for invalid shapes
 * (GATEUP needs an even N) or an unknown flag combination. */
size_t w4a8_packed_bytes(int E, int N, int K, int layout);

/* Quantise and pack E weight matrices  (a1: the offline conversion step).
 *   layout      : W4A8_LAYOUT_PLAIN or W4A8_LAYOUT_GATEUP, optionally | one scheme flag.
 *   w_bf16      : device, bf16 [E][N][K], row-major (nn.Linear orientation).
 *   packed      : device, w4a8_packed_bytes(E,N,K,layout) bytes (256-B aligned),
 *                 the tiled layout consumed by w4a8_gemm / w4a8_moe_forward.
 *   codes_opt   : device or NULL; canonical packed codes uint8 [E][N][Kp/2],
 *                 byte j of a row = code[2j] | code[2j+1] << 4.
 *   scale_f16_opt, zp_f16_opt : device or NULL; fp16 bit patterns [E][N][Kp/128].
 * Returns W4A8_ENOSPACE if packed_bytes is too small. */
int w4a8_pack_weights(const void* w_bf16, int E, int N, int K, int layout,
                      void* packed, size_t packed_bytes,
                      uint8_t* codes_opt, uint16_t* scale_f16_opt, uint16_t* zp_f16_opt,
                      void* stream);

/* Per-token symmetric INT8 quantisation of activations  (a2).
 *   x_bf16 : device, bf16 [T][K] row-major.
 *   q      : device, int8 [T][Kp], Kp = K rounded up to 128 (padding written as 0).
 *   s      : device, float [T]; s = max|x|/127 (0 for an all-zero row, with q = 0). */
int w4a8_quant_act(const void* x_bf16, int T, int K, int8_t* q, float* s, void* stream);

/* Top-k softmax routing  (a3).  The Kimi 2.7T MoE W4A8 article (hotelren.com
 * 5173946), section 5.2: the router is not quantised; it reads 16-bit logits and
 * picks each token's experts, whose gate weights scale the expert outputs in the
 * combine (section 4.3, step 4).  The selection and weights follow the plainest
 * softmax gating, which the pages do not spell out.
 *   logits_bf16 : device, bf16 [T][E];  1 <= k <= min(E, 32), E <= 1024.
 *   ids         : device, int32 [T][k]: the k largest logits, largest first, ties
 *                 to the lower expert id.
 *   w           : device, float [T][k]: softmax probability over all E experts
 *                 of each chosen expert (not renormalised over the k). */
int w4a8_route_topk(const void* logits_bf16, int T, int E, int k, int32_t* ids, float* w,
                    void* stream);

/* Workspace bytes needed by w4a8_moe_forward for this layer shape. */
size_t w4a8_moe_workspace_bytes(int T, int E, int k, int H, int F);

/* The W4A8 MoE expert FFN  (a4..a8):
 *   out[t] = sum_j w[t][j] * Down_e( SwiGLU( Up_e( x[t] ) ) ),  e = ids[t][j],
 * with x quantised per token to INT8, Up/Down W4A8 GEMMs (INT32 per-group
 * partials), h = silu(gate) * up rounded to bf16 and requantised per token to INT8
 * before Down (section 4.3, step 4: the GEMM result is handed on in 16-bit
 * floating point), and the fp32 weighted sum of the experts' Down results rounded
 * to bf16.
 * Source: the Kimi 2.7T MoE W4A8 article (hotelren.com 5173946), section 4.3: the
 * activations are quantised per token at run time, the INT4 weights are expanded
 * inside the kernel and multiplied in INT8 with INT32 accumulation, the result is
 * scaled back and the input of the next projection is quantised again; section 5.1:
 * tokens are grouped by expert before the expert GEMMs; «Kimi 2.7 Moe 从 4 bit 存储到
 * INT8 拆解» (pptc.cn), section 3.2: INT8 x INT8 products accumulate in INT32.
 *   packed_up   : from w4a8_pack_weights(E, 2F, H, W4A8_LAYOUT_GATEUP).
 *   packed_down : from w4a8_pack_weights(E, H, F, W4A8_LAYOUT_PLAIN).
 *   x_bf16      : device bf16 [T][H].   ids: device int32 [T][k] (0 <= id < E;
 *                 an id out of range drops that slot and sets W4A8_EDEVICE).
 *   w           : device float [T][k].  out_bf16: device bf16 [T][H].
 *   ws          : device, >= w4a8_moe_workspace_bytes(T,E,k,H,F) bytes.
 * Limits: E <= 1024, k <= 32, T*k < 2^31. */
int w4a8_moe_forward(const void* packed_up, const void* packed_down, int E, int H, int F,
                     const void* x_bf16, int T, const int32_t* ids, const float* w, int k,
                     void* out_bf16, void* ws, size_t ws_bytes, void* stream);

/* w4a8_moe_forward for experts packed with another group size (group = 64, 128 or
 * 256, both projections packed with it); the token rows are padded to whole groups.
 * Workspace from w4a8_moe_workspace_bytes_g; stages readable with w4a8_debug_dump(what
 * | W4A8_DUMP_GROUP64 or W4A8_DUMP_GROUP256).  Returns W4A8_EINVAL for another group. */
size_t w4a8_moe_workspace_bytes_g(int T, int E, int k, int H, int F, int group);
int w4a8_moe_forward_g(const void* packed_up, const void* packed_down, int E, int H, int F, int group,
                       const void* x_bf16, int T, const int32_t* ids, const float* w, int k,
                       void* out_bf16, void* ws, size_t ws_bytes, void* stream);

/* Same as w4a8_moe_forward, but x_bf16, ids, w and out_bf16 are HOST buffers
 * (pinned memory recommended): they are copied to / from the workspace on
 * `stream` with cudaMemcpyAsync before and after the forward.  Needs
 * w4a8_moe_host_workspace_bytes() of workspace.  The call returns once the work
 * is enqueued; out_bf16 is valid after the stream is synchronised. */
size_t w4a8_moe_host_workspace_bytes(int T, int E, int k, int H, int F);
int w4a8_moe_forward_host(const void* packed_up, const void* packed_down, int E, int H, int F,
                          const void* x_bf16_host, int T, const int32_t* ids_host,
                          const float* w_host, int k, void* out_bf16_host,
                          void* ws, size_t ws_bytes, void* stream);

/* The layer routed from router logits, with HOST buffers: x_bf16_host [T][H] and
 * logits_bf16_host [T][E] (bf16) are copied into the workspace, the experts are
 * chosen on the device exactly as w4a8_route_topk does, the layer runs as in
 * w4a8_moe_forward and out_bf16_host [T][H] is copied back, all on `stream`.
 * Same workspace as w4a8_moe_forward_host; asynchronous like it. */
int w4a8_moe_forward_logits_host(const void* packed_up, const void* packed_down, int E, int H, int F,
                                 const void* x_bf16_host, int T, const void* logits_bf16_host, int k,
                                 void* out_bf16_host, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes needed by w4a8_gemm. */
size_t w4a8_gemm_workspace_bytes(int M, int N, int K);

/* One dense W4A8 linear layer  (a5 on a single weight matrix):
 *   y[m][n] = sa[m] * sum_g scale[n][g] * acc[m][n][g],
 *   acc[m][n][g] = sum_{k in group g} qa[m][k] * (code[n][k] - zp[n][g])   (INT32).
 * Source: «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» (pptc.cn), section 3.2: the INT4
 * weights become INT8 values (code - zero point), INT8 x INT8 products accumulate in
 * INT32, and the integer result is scaled back to floating point by the weight scale
 * (one per 128-wide group, section 2.1) and the token scale; the Kimi 2.7T MoE W4A8
 * article (hotelren.com 5173946), section 4.3, steps 2-4.
 *   qa          : device int8 [M][Kp] (as written by w4a8_quant_act), sa: float [M].
 *   packed      : from w4a8_pack_weights(1, N, K, W4A8_LAYOUT_PLAIN).
 *   y           : device float [M][N].
 *   partials_opt: device int32 [M][N][Kp/128] or NULL -- the exact INT32 partials. */
int w4a8_gemm(const int8_t* qa, const float* sa, int M, const void* packed, int N, int K,
              float* y, int32_t* partials_opt, void* ws, size_t ws_bytes, void* stream);

/* w4a8_gemm for weights packed with another group size (group = 64, 128 or 256, as
 * packed): one INT32 partial per group, partials_opt int32 [M][N][Kp/group], where Kp
 * is K padded to a multiple of 128 and of the group; qa as for w4a8_gemm ([M][K
 * rounded up to 128], the row padding to Kp is implicit zeros).  Workspace from
 * w4a8_gemm_workspace_bytes_g.  Returns W4A8_EINVAL for another group. */
size_t w4a8_gemm_workspace_bytes_g(int M, int N, int K, int group);
int w4a8_gemm_g(const int8_t* qa, const float* sa, int M, const void* packed, int N, int K, int group,
                float* y, int32_t* partials_opt, void* ws, size_t ws_bytes, void* stream);

/* w4a8_gemm for callers that cannot allocate device memory.  (The pages describe
 * no such variant: it exists for integration, not for the method.)
 * Some callers cannot hand this library a workspace: a plugin inside a host
 * framework that owns every device allocation and forbids new ones on its
 * execution path, code running where a cudaMalloc would synchronise the device
 * or is not allowed, a binding with no allocator at hand.  This entry point takes
 * the same inputs and outputs as w4a8_gemm and uses instead a fixed 8 MiB device
 * array inside the library (reserved on every GPU that loads the library, until
 * the process exits).  It calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *   - Limit: w4a8_gemm_workspace_bytes(M, N, K) must not exceed 8 MiB (about
 *     8.3 million INT8 values of M x Kp, e.g. M = 1024 at K = 7168); larger
 *     sizes return W4A8_ENOSPACE before anything is launched.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture.
 *   - Every call, on every stream, shares the one array: calls whose work
 *     overlaps on the GPU race with each other and give wrong results.  Each call
 *     rewrites all of the scratch it reads, so nothing carries over between calls.
 *   - The device error word lives in that array and is not readable by the caller. */
int w4a8_gemm_noalloc(const int8_t* qa, const float* sa, int M, const void* packed, int N, int K,
                      float* y, int32_t* partials_opt, void* stream);

/* The device error word of the last w4a8_gemm_noalloc call on the current device
 * (the same bits as w4a8_last_device_error): synchronises `stream`, then reads the
 * word from the library's scratch array.  Read it before the next noalloc call,
 * which clears it. */
int w4a8_gemm_noalloc_last_error(void* stream);

/* ---- W4A16: the comparison point of the pages ----
 * The same packed INT4 weights multiplied with 16-bit (bf16) activations that are
 * never quantised: y[m][n] = sum_k x[m][k] * (code[n][k] - zp[n][g(k)]) * scale[n][g(k)].
 * «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» (pptc.cn), section 1 (W4A16 keeps 16-bit
 * activations; W4A8 decodes 20-40% faster) and section 3.3 (the W4A16 / W4A8 / W8A8
 * table); the Kimi 2.7T MoE W4A8 article (hotelren.com 5173946), section 3.2 (W4A8
 * over W4A16 on H100) and section 4.4.  Computed on the tensor core as bf16
 * (code - zp) x bf16 x with one fp32 partial per 128-wide K group (every product is
 * exact; the partial's sum is fp32), then acc += scale * partial in fp32.  The
 * kernel uses 16-token tiles (the decode-shaped path): it is meant for decode-sized
 * layers, where both schemes stream the same weight bytes.
 *
 * w4a16_gemm: x device bf16 [M][K] row-major (2-byte aligned), packed from
 *   w4a8_pack_weights(1, N, K, W4A8_LAYOUT_PLAIN), y device float [M][N]; scratch
 *   in ws (w4a16_gemm_workspace_bytes).  Error returns as w4a8_gemm. */
size_t w4a16_gemm_workspace_bytes(int M, int N, int K);
int w4a16_gemm(const void* x_bf16, int M, const void* packed, int N, int K, float* y, void* ws,
               size_t ws_bytes, void* stream);

/* w4a16_moe_forward: the MoE expert FFN with W4A16 experts, with the arguments and
 * the routing, permutation and combine of w4a8_moe_forward: each token's bf16 row
 * goes to its k experts, up GEMM (gate|up) -> SwiGLU -> h rounded to bf16 (the
 * activations between the projections stay 16-bit) -> down GEMM -> weighted combine
 * -> bf16.  Workspace from w4a16_moe_workspace_bytes; stages readable with
 * w4a8_debug_dump(what | W4A8_DUMP_W4A16). */
size_t w4a16_moe_workspace_bytes(int T, int E, int k, int H, int F);
int w4a16_moe_forward(const void* packed_up, const void* packed_down, int E, int H, int F,
                      const void* x_bf16, int T, const int32_t* ids, const float* w, int k,
                      void* out_bf16, void* ws, size_t ws_bytes, void* stream);

/* Intermediate results kept in a w4a8_moe_forward workspace, for stage tests. */
enum {
    W4A8_DUMP_COUNTS = 0, /* int32 [E]      tokens routed to each expert             */
    W4A8_DUMP_OFFS = 1,   /* int32 [E+1]    exclusive prefix sum of counts           */
    W4A8_DUMP_PERM = 2,   /* int32 [T*k]    slot (t*k+j) at each grouped position     */
    W4A8_DUMP_INV = 3,    /* int32 [T*k]    padded row of each slot                   */
    W4A8_DUMP_POFFS = 4,  /* int32 [E+1]    row offsets with every expert padded to 16 */
    W4A8_DUMP_ACT1 = 5,   /* int8, R x Hp: INT8 x rows (tiled, see below)             */
    W4A8_DUMP_S1 = 6,     /* float [R]      token scale of each padded row            */
    W4A8_DUMP_H = 7,      /* bf16 [R][Fp]   SwiGLU output h per padded row             */
    W4A8_DUMP_ACT2 = 8,   /* int8, R x Fp: requantised h (tiled, see below)           */
    W4A8_DUMP_S2 = 9,     /* float [R]      scale of the requantised h rows           */
    W4A8_DUMP_Y2 = 10,    /* float [R][H]   down-projection output per padded row     */
    W4A8_DUMP_ERR = 11,   /* uint32 [1]     device error word                         */
    /* OR-ed into `what`: the region of a w4a16_moe_forward workspace.  There ACT1 holds
     * the bf16 x rows and ACT2 the bf16 h rows, both tiled as below with 16-row blocks
     * and 256 bytes per row and K group ([R/16][Kp/128][2][16][128 bytes]: the two
     * 64-column halves of a group one after the other, each swizzled like the INT8
     * rows); S1, H and S2 are empty. */
    W4A8_DUMP_W4A16 = 0x100,
    /* OR-ed into `what`: the region of a w4a8_moe_forward_g workspace of that group size
     * (the tiled rows are then Hp = H and Fp = F padded to 128 and to the group). */
    W4A8_DUMP_GROUP64 = 0x400,
    W4A8_DUMP_GROUP256 = 0x800
};
/* R = w4a8_moe_rows_capacity(T,E,k).  Tiled INT8 rows: rows are grouped in blocks of
 * RB = w4a8_moe_act_block_rows(T,E,k) rows (16 for decode-shaped layers, whose mean
 * tokens per expert is at most 16; otherwise RB = R); the buffer is
 * [R/RB][Kp/128][RB][128 bytes]: block b, K group g, row i (= r % RB) starts at byte
 * ((b * Kp/128 + g) * RB + i) * 128, and the row's 16-byte chunk c (K columns
 * 128g + 16c .. +15) sits at chunk position c ^ (i & 7). */
int w4a8_moe_rows_capacity(int T, int E, int k);
int w4a8_moe_act_block_rows(int T, int E, int k);

/* Byte offset and size of dump region `what` inside the workspace. */
int w4a8_debug_region(int T, int E, int k, int H, int F, int what, size_t* offset, size_t* bytes);

/* Copy dump region `what` of workspace `ws` to `dst` (device or host memory,
 * cudaMemcpyDefault), at most `bytes` bytes, on `stream`. */
int w4a8_debug_dump(const void* ws, int T, int E, int k, int H, int F, int what, void* dst,
                    size_t bytes, void* stream);

/* Synchronise `stream`, then return the device error word kept in workspace `ws`
 * (0 = none; bit 0 = a bounded wait timed out, bit 1 = expert id out of range).
 * Any workspace from w4a8_moe_forward / w4a8_gemm may be passed. */
int w4a8_last_device_error(const void* ws, void* stream);

/* Per-kernel device timing, for benchmarks.  After w4a8_profile_start(), every
 * w4a8_quant_act / w4a8_route_topk / w4a8_moe_forward / w4a8_moe_forward_host /
 * w4a8_moe_forward_logits_host / w4a8_gemm call made from the same
 * host thread records a pair of CUDA events around each kernel kind it launches
 * (on the call's stream).  w4a8_profile_stop() waits for those events, writes
 * per kind the number of kernel launches and their summed device milliseconds
 * (arrays of n entries, indexed by the W4A8_KERNEL_* values; a "perm" entry covers
 * the permutation kernels), stops recording and returns W4A8_OK.  Timing
 * adds one event record per kernel; it changes no result. */
enum {
    W4A8_KERNEL_PERM = 0,      /* histogram, scan, scatter (1 or 3 launches)  */
    W4A8_KERNEL_ACT_QUANT = 1, /* per-token INT8 into the grouped tiled rows    */
    W4A8_KERNEL_GEMM_UP = 2,   /* grouped W4A8 GEMM, gate|up, SwiGLU epilogue   */
    W4A8_KERNEL_REQUANT = 3,   /* per-row INT8 of h                             */
    W4A8_KERNEL_GEMM_DOWN = 4, /* grouped W4A8 GEMM, down projection            */
    W4A8_KERNEL_COMBINE = 5,   /* weighted sum of the k expert outputs          */
    W4A8_KERNEL_GEMM_DENSE = 6,/* w4a8_gemm (re-layout + GEMM, 2 launches)      */
    W4A8_KERNEL_ROUTE = 7,     /* top-k softmax routing                         */
    W4A8_KERNEL_KINDS = 8
};
int w4a8_profile_start(void);
int w4a8_profile_stop(int* launches, float* total_ms, int n);

/* Test hook of the failure detection (no counterpart in the pages).  Every bounded
 * wait inside the GEMM kernels gives up after a number of clock cycles (about 2 s by
 * default), sets bit 0 of the device error word, drains what it issued, frees its
 * tensor memory and returns.  While set on the calling host thread, this makes the
 * GEMM launches of w4a8_moe_forward* and w4a8_gemm* use `wait_limit_cycles` (0 = the
 * default) and, with flags = W4A8_DEBUG_SKIP_FIRST_COPY, has the first CTA issue no
 * copy for its first pipeline step, so that the waits for it run out: the result of
 * that call is undefined and its device error word has bit 0 set.  flags = 0 and
 * wait_limit_cycles = 0 restore normal operation.  Returns W4A8_EINVAL for unknown
 * flags or a negative limit. */
enum { W4A8_DEBUG_SKIP_FIRST_COPY = 1 };
int w4a8_debug_inject(unsigned int flags, long long wait_limit_cycles);

/* INT8 KV cache with static per-head scales (the Kimi 2.7T MoE W4A8 article,
 * hotelren.com/news/5173946, section 5: the attention KV cache is quantised to INT8
 * statically, one scale per head fixed from a little calibration data; the scale is
 * the symmetric form of the LLM quantisation primer, section 2.1).
 * Layout: x [T][H][D] bf16 row-major (token, head, channel); q [T][H][D] int8;
 * scale [H] fp32.  D must be a multiple of 16 (16 <= D), 1 <= H <= 1024; x, q 16-byte
 * aligned, scale 4-byte aligned (W4A8_EUNSUPPORTED / W4A8_EALIGN otherwise).
 * Device pointers owned by the caller; asynchronous on `stream`.
 *
 * w4a8_kv_calibrate: scale[h] = max|x[:, h, :]| / 127 over the calibration tokens
 *   (correctly rounded fp32 division); 0 for a head whose values are all zero (and
 *   for T = 0).
 * w4a8_kv_quant:     q = clamp(round(x / scale[h]), -127, 127), fp32 division, round
 *   half to even; values beyond the calibrated range saturate; scale 0 -> q = 0.
 * w4a8_kv_dequant:   x = bf16(q * scale[h]), the fp32 product rounded once (RNE). */
int w4a8_kv_calibrate(const void* x_bf16, int T, int H, int D, float* scale, void* stream);
int w4a8_kv_quant(const void* x_bf16, int T, int H, int D, const float* scale, int8_t* q, void* stream);
int w4a8_kv_dequant(const int8_t* q, int T, int H, int D, const float* scale, void* x_bf16, void* stream);

/* Human-readable name of a w4a8_status value. */
const char* w4a8_status_string(int status);

/* ABI version (major * 100 + minor). */
int w4a8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A8_H */

// Internal declarations shared by the kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/matmamba.h"

namespace mm {

// ------------------------------------------------------------------ element access

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// SiLU(a) = a * sigmoid(a) ("MatMamba: A Matryoshka State Space Model": sigma = SiLU).
__device__ __forceinline__ float silu_f(float a) { return a / (1.0f + expf(-a)); }

// softplus(v) = log(1 + e^v).  Above 20 the identity is within 2.1e-9 relative.
__device__ __forceinline__ float softplus_f(float v) { return v > 20.0f ? v : log1pf(expf(v)); }

// ------------------------------------------------------------------ segmented GEMM
//
// out_s[m, j] (+)= sum_k A[m, k] * Bs[j, k] for j in [0, n_s) of each segment s.
// A and every Bs are K-major (rows of K contiguous elements).  The segments
// concatenate along N; they let one launch read a width view of W_in whose
// rows sit in four separate blocks, and route each block of output columns to
// its own buffer (and dtype).
enum GemmEpi { kEpiStore = 0, kEpiConv = 1, kEpiSoftplus = 2 };

struct GemmSeg {
    const void* B;   // first row of this segment's weights, row stride ldb
    void* out;       // output of this segment's first column, row stride ldo
    int64_t ldo;
    int n;           // number of columns (rows of B) in this segment
    int out_f32;     // output stored as fp32 (else in the input dtype)
    int accumulate;  // fp32 output only: out += result
    int kind;        // GemmEpi (tensor-core kernel only)
    int conv_row0;   // kEpiConv: conv row of column 0; kEpiSoftplus: unused
};

constexpr int kMaxSeg = 4;

// Epilogue extras of the tensor-core kernel.
//  - kEpiConv segments apply the block's causal depthwise conv (K taps) and
//    SiLU down the token axis: tiles then overlap by K-1 rows so every output
//    row sees its K-1 predecessors, taps never cross a sequence start (L
//    tokens per sequence) and read the given history there instead.
//  - kEpiSoftplus segments store softplus(acc + dt_bias[col]) in fp32.
//  - row_parts != null scales every output row m by
//    rsqrt(sum_j row_parts[m * nparts + j] * rs_inv_n + rs_eps), the parts
//    added in index order (RMSNorm applied after the GEMM, deterministic).
struct GemmExtra {
    const void* conv_w;
    const void* conv_b;
    const float* dt_bias;
    int L, K, conv_rows;
    const void* conv_state_in;
    void* conv_state_out;
    const float* row_parts;
    int nparts;
    float rs_inv_n, rs_eps;
};

struct GemmDesc {
    const void* A;
    int64_t lda;
    int64_t ldb;
    int M, K;
    int nseg;
    GemmSeg seg[kMaxSeg];
    GemmExtra ex;
    // launch as a programmatic dependent of the stream's previous kernel: the CTAs may become resident
    // while it finishes, and wait for its completion before reading anything
    int pdl = 0;
};

// ------------------------------------------------------------------ scan arguments

struct ScanArgs {
    const void* x; int64_t sx;
    const float* dt; int64_t sdt;
    const float* A;
    const void* B; int64_t sB;
    const void* C; int64_t sC;
    const float* D;
    int batch, L, h, P, N, G, hpg, chunk;
    const float* init_state; int64_t state_stride;
    void* y; int64_t sy;
    float* final_state;
};

// ------------------------------------------------------------------ launchers (return cudaError_t)

cudaError_t launch_gemm_simt(int dtype, const GemmDesc& g, cudaStream_t s);
cudaError_t launch_conv_silu_dt(int dtype, const void* zxbc, int64_t ld_in, int col0, const float* dt_raw,
                                const void* conv_w, const void* conv_b, const float* dt_bias, int E, int d, int nconv,
                                int h, int K, int batch, int L, const void* conv_state_in, int conv_rows, void* xbc_out,
                                float* dt_out, cudaStream_t s);
cudaError_t launch_conv_state_out(int dtype, const void* zxbc, int64_t ld_in, int col0, int E, int d, int nconv, int K,
                                  int batch, int L, const void* conv_state_in, int conv_rows, void* conv_state_out,
                                  cudaStream_t s);
cudaError_t launch_scan_seq(int dtype, const ScanArgs& a, cudaStream_t s);
cudaError_t launch_gate_rmsnorm(int dtype, const void* y, int64_t ldy, const void* z, int64_t ldz, const void* w,
                                float eps, int d, int rows, void* out, int64_t ldo, cudaStream_t s);
cudaError_t launch_rmsnorm_rows_f32in(int dtype, const float* x, const void* w, float eps, int cols, int rows, void* out,
                                      cudaStream_t s);
cudaError_t launch_to_f32(int dtype, const void* in, float* out, int64_t n, cudaStream_t s);
cudaError_t launch_from_f32(int dtype, const float* in, void* out, int64_t n, cudaStream_t s);
cudaError_t launch_step_conv_dt(int dtype, const void* zxbc, int64_t ld_in, int col0, const float* dt_raw,
                                const void* conv_w, const void* conv_b, const float* dt_bias, int E, int d, int nconv,
                                int h, int K, int batch, void* conv_state, int conv_rows, void* xbc_out, float* dt_out,
                                cudaStream_t s);
cudaError_t launch_step_scan(int dtype, const void* xbc, int nconv, int d, const float* dt, const float* A,
                             const float* D, float* ssm_state, int H, int h, int P, int N, int GN, int hpg, int batch,
                             void* y, cudaStream_t s);

cudaError_t launch_step_scan_gated(const void* xbc, int nconv, int d, const float* dt, const float* A, const float* D,
                                   float* ssm_state, int H, int h, int GN, int hpg, int batch, const void* z,
                                   int64_t ldz, const void* norm_w, void* nrm, float* row_parts, cudaStream_t s);

// Device status word of the current device (MM_OK or a code a kernel recorded).
int* device_status_ptr();
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch,
                    uint32_t box_inner, uint32_t box_rows);
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t planes,
                       uint64_t pitch, uint64_t plane_pitch, uint32_t box_inner, uint32_t box_rows);

// Tensor-core paths (bf16 only).
bool gemm_tc_supported(const GemmDesc& g);
cudaError_t launch_gemm_tc(const GemmDesc& g, cudaStream_t s);
bool scan_tc_supported(const ScanArgs& a);
size_t scan_tc_workspace(const ScanArgs& a);
int scan_tc_kernel_count(const ScanArgs& a);
cudaError_t launch_scan_tc(const ScanArgs& a, void* ws, size_t ws_bytes, cudaStream_t s);

// Gate + RMSNorm fused into the tensor-core scan's output: instead of y the scan
// stores (y * SiLU(z)) * norm_w in bf16, and the sum of squares of y * SiLU(z)
// over each (token, head, 32-channel half) into row_parts[tok * 2h + 2 head + half].
struct ScanGate {
    const void* z;
    int64_t sz;
    const void* norm_w;
    float* row_parts;
};
cudaError_t launch_scan_tc_gated(const ScanArgs& a, const ScanGate& g, void* ws, size_t ws_bytes, cudaStream_t s);

}  // namespace mm

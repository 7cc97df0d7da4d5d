// CUDA-core kernels: the fp32 path of every step, the elementwise steps of the
// bf16 path (conv + SiLU + dt, gate + RMSNorm, residual pre-norm), the decode
// step, and the CUDA-core GEMM / sequential scan used for shapes the
// tensor-core kernels do not cover.
//
// Steps follow "MatMamba: A Matryoshka State Space Model", block-definition
// paragraph (in_proj, causal conv of kernel 4 per channel, SiLU, selective
// scan with A and D, Norm = RMSNorm, out_proj) at the width view of the nested
// sub-block paragraph.
#include "mm_internal.cuh"

namespace mm {

// ====================================================================== GEMM (CUDA cores)

__device__ __forceinline__ int gemm_find_seg(const GemmDesc& g, int n, int& local)
{
    int base = 0;
    for (int s = 0; s < g.nseg; ++s) {
        if (n < base + g.seg[s].n) { local = n - base; return s; }
        base += g.seg[s].n;
    }
    local = 0;
    return -1;
}

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmDesc g, int n_total)
{
    constexpr int BM = 64, BN = 64, BK = 32;
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;  // row blocks on x: up to 2^31 - 1 of them
    const T* A = static_cast<const T*>(g.A);

    // loader role: one A row and one B row, 8 consecutive k each
    const int lr = tid >> 2, lk = (tid & 3) * 8;
    const int am = m0 + lr;
    const T* arow = am < g.M ? A + (int64_t)am * g.lda : nullptr;
    const T* brow = nullptr;
    {
        int loc, s = (n0 + lr < n_total) ? gemm_find_seg(g, n0 + lr, loc) : -1;
        if (s >= 0) brow = static_cast<const T*>(g.seg[s].B) + (int64_t)loc * g.ldb;
    }

    const int ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < g.K; k0 += BK) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            int k = k0 + lk + j;
            As[lk + j][lr] = (arow && k < g.K) ? to_f32(arow[k]) : 0.0f;
            Bs[lk + j][lr] = (brow && k < g.K) ? to_f32(brow[k]) : 0.0f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < BK; ++k) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[k][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        int n = n0 + tx + 16 * j;
        if (n >= n_total) continue;
        int loc, s = gemm_find_seg(g, n, loc);
        const GemmSeg& sg = g.seg[s];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int m = m0 + ty + 16 * i;
            if (m >= g.M) continue;
            if (sg.out_f32) {
                float* o = static_cast<float*>(sg.out) + (int64_t)m * sg.ldo + loc;
                *o = sg.accumulate ? *o + acc[i][j] : acc[i][j];
            } else {
                static_cast<T*>(sg.out)[(int64_t)m * sg.ldo + loc] = from_f32<T>(acc[i][j]);
            }
        }
    }
}

cudaError_t launch_gemm_simt(int dtype, const GemmDesc& g, cudaStream_t s)
{
    int n_total = 0;
    for (int i = 0; i < g.nseg; ++i) n_total += g.seg[i].n;
    if (g.M == 0 || n_total == 0) return cudaSuccess;
    if ((n_total + 63) / 64 > 65535) return cudaErrorInvalidValue;
    dim3 grid((g.M + 63) / 64, (n_total + 63) / 64);
    if (dtype == MM_BF16) gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(g, n_total);
    else gemm_simt_kernel<float><<<grid, 256, 0, s>>>(g, n_total);
    return cudaGetLastError();
}

// ====================================================================== conv + SiLU + dt

// One thread per (token, channel).  Channels [0, nconv) are x | B | C of the
// width view (conv rows [0,d) u [E, E+2GN)); channels [nconv, nconv+h) compute
// dt = softplus(raw + dt_bias) for head c - nconv.
template <typename T>
__global__ void conv_silu_dt_kernel(const T* __restrict__ zxbc, int64_t ld_in, int col0,
                                    const float* __restrict__ dt_raw, const T* __restrict__ conv_w,
                                    const T* __restrict__ conv_b, const float* __restrict__ dt_bias, int E, int d,
                                    int nconv, int h, int K, int L, const T* __restrict__ conv_state_in, int conv_rows,
                                    T* __restrict__ xbc_out, float* __restrict__ dt_out)
{
    const int c = blockIdx.y * blockDim.x + threadIdx.x;
    const int64_t tok = blockIdx.x;
    if (c >= nconv + h) return;
    if (c >= nconv) {
        const int i = c - nconv;
        dt_out[tok * h + i] = softplus_f(dt_raw[tok * h + i] + dt_bias[i]);
        return;
    }
    const int b = (int)(tok / L), t = (int)(tok % L);
    const int row = c < d ? c : E + (c - d);
    float acc = to_f32(conv_b[row]);
    for (int j = 0; j < K; ++j) {
        const int tau = t - (K - 1) + j;
        float v;
        if (tau >= 0) v = to_f32(zxbc[((int64_t)b * L + tau) * ld_in + col0 + c]);
        else if (conv_state_in) v = to_f32(conv_state_in[((int64_t)b * conv_rows + row) * (K - 1) + (K - 1 + tau)]);
        else v = 0.0f;
        acc = fmaf(to_f32(conv_w[(int64_t)row * K + j]), v, acc);
    }
    xbc_out[tok * nconv + c] = from_f32<T>(silu_f(acc));
}

cudaError_t launch_conv_silu_dt(int dtype, const void* zxbc, int64_t ld_in, int col0, const float* dt_raw,
                                const void* conv_w, const void* conv_b, const float* dt_bias, int E, int d, int nconv,
                                int h, int K, int batch, int L, const void* conv_state_in, int conv_rows, void* xbc_out,
                                float* dt_out, cudaStream_t s)
{
    dim3 grid((unsigned)((int64_t)batch * L), (nconv + h + 127) / 128);
    if (dtype == MM_BF16)
        conv_silu_dt_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(
            (const __nv_bfloat16*)zxbc, ld_in, col0, dt_raw, (const __nv_bfloat16*)conv_w,
            (const __nv_bfloat16*)conv_b, dt_bias, E, d, nconv, h, K, L, (const __nv_bfloat16*)conv_state_in,
            conv_rows, (__nv_bfloat16*)xbc_out, dt_out);
    else
        conv_silu_dt_kernel<float><<<grid, 128, 0, s>>>((const float*)zxbc, ld_in, col0, dt_raw,
                                                         (const float*)conv_w, (const float*)conv_b, dt_bias, E, d,
                                                         nconv, h, K, L, (const float*)conv_state_in, conv_rows,
                                                         (float*)xbc_out, dt_out);
    return cudaGetLastError();
}

// Conv state after a prefill: the last K-1 pre-conv inputs of each active
// channel, oldest first.  One thread per (batch, channel) walks k upward, so
// an in-place update (state_out == state_in) would also be safe.
template <typename T>
__global__ void conv_state_out_kernel(const T* __restrict__ zxbc, int64_t ld_in, int col0, int E, int d, int nconv,
                                      int K, int batch, int L, const T* conv_state_in, int conv_rows, T* conv_state_out)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    if (c >= nconv) return;
    const int row = c < d ? c : E + (c - d);
    for (int k = 0; k < K - 1; ++k) {
        const int tau = L - (K - 1) + k;
        T v;
        if (tau >= 0) v = zxbc[((int64_t)b * L + tau) * ld_in + col0 + c];
        else if (conv_state_in) v = conv_state_in[((int64_t)b * conv_rows + row) * (K - 1) + (K - 1 + tau)];
        else v = from_f32<T>(0.0f);
        conv_state_out[((int64_t)b * conv_rows + row) * (K - 1) + k] = v;
    }
}

cudaError_t launch_conv_state_out(int dtype, const void* zxbc, int64_t ld_in, int col0, int E, int d, int nconv, int K,
                                  int batch, int L, const void* conv_state_in, int conv_rows, void* conv_state_out,
                                  cudaStream_t s)
{
    dim3 grid((nconv + 127) / 128, batch);
    if (dtype == MM_BF16)
        conv_state_out_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(
            (const __nv_bfloat16*)zxbc, ld_in, col0, E, d, nconv, K, batch, L, (const __nv_bfloat16*)conv_state_in,
            conv_rows, (__nv_bfloat16*)conv_state_out);
    else
        conv_state_out_kernel<float><<<grid, 128, 0, s>>>((const float*)zxbc, ld_in, col0, E, d, nconv, K, batch, L,
                                                           (const float*)conv_state_in, conv_rows,
                                                           (float*)conv_state_out);
    return cudaGetLastError();
}

// ====================================================================== sequential scan

// The scan in its recurrent form on CUDA cores: one CTA per (batch, head,
// 8 state rows p); 16 threads share one p and hold NPT state entries n each.
// Tokens are staged through shared memory 16 at a time.
template <typename T, int NPT>
__global__ void __launch_bounds__(128) scan_seq_kernel(ScanArgs a)
{
    constexpr int PR = 8, TC = 16;
    extern __shared__ float sm[];
    const int N = a.N, P = a.P;
    float* Bs = sm;                  // [TC][N]
    float* Cs = Bs + TC * N;         // [TC][N]
    float* xs = Cs + TC * N;         // [TC][PR]
    float* dts = xs + TC * PR;       // [TC]
    const int b = blockIdx.z, i = blockIdx.y, p0 = blockIdx.x * PR;
    const int tid = threadIdx.x, pr = tid >> 4, nq = tid & 15;
    const int p = p0 + pr;
    const int g = i / a.hpg;
    const float Ai = a.A[i];
    const float Di = a.D ? a.D[i] : 0.0f;
    const T* X = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.B);
    const T* Cm = static_cast<const T*>(a.C);
    T* Y = static_cast<T*>(a.y);

    float hs[NPT];
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
        const int n = nq + 16 * j;
        hs[j] = (a.init_state && p < P && n < N) ? a.init_state[(int64_t)b * a.state_stride + ((int64_t)i * P + p) * N + n]
                                                 : 0.0f;
    }
    for (int t0 = 0; t0 < a.L; t0 += TC) {
        const int tc = min(TC, a.L - t0);
        __syncthreads();
        for (int e = tid; e < TC * N; e += 128) {
            const int tt = e / N, n = e % N;
            const int64_t tok = (int64_t)b * a.L + t0 + tt;
            Bs[e] = tt < tc ? to_f32(Bm[tok * a.sB + (int64_t)g * N + n]) : 0.0f;
            Cs[e] = tt < tc ? to_f32(Cm[tok * a.sC + (int64_t)g * N + n]) : 0.0f;
        }
        for (int e = tid; e < TC * PR; e += 128) {
            const int tt = e / PR, q = p0 + e % PR;
            const int64_t tok = (int64_t)b * a.L + t0 + tt;
            xs[e] = (tt < tc && q < P) ? to_f32(X[tok * a.sx + (int64_t)i * P + q]) : 0.0f;
        }
        if (tid < TC) dts[tid] = tid < tc ? a.dt[((int64_t)b * a.L + t0 + tid) * a.sdt + i] : 0.0f;
        __syncthreads();
        for (int tt = 0; tt < tc; ++tt) {
            const float dtv = dts[tt];
            const float av = expf(dtv * Ai);
            const float xv = xs[tt * PR + pr];
            const float dx = dtv * xv;
            float acc = 0.0f;
#pragma unroll
            for (int j = 0; j < NPT; ++j) {
                const int n = nq + 16 * j;
                if (n < N) {
                    hs[j] = fmaf(av, hs[j], dx * Bs[tt * N + n]);
                    acc = fmaf(Cs[tt * N + n], hs[j], acc);
                }
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 8);
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            if (nq == 0 && p < P) {
                const int64_t tok = (int64_t)b * a.L + t0 + tt;
                Y[tok * a.sy + (int64_t)i * P + p] = from_f32<T>(fmaf(Di, xv, acc));
            }
        }
    }
    if (a.final_state && p < P) {
#pragma unroll
        for (int j = 0; j < NPT; ++j) {
            const int n = nq + 16 * j;
            if (n < N) a.final_state[(int64_t)b * a.state_stride + ((int64_t)i * P + p) * N + n] = hs[j];
        }
    }
}

template <typename T>
static cudaError_t scan_seq_dispatch(const ScanArgs& a, cudaStream_t s)
{
    dim3 grid((a.P + 7) / 8, a.h, a.batch);
    const size_t smem = sizeof(float) * (16 * a.N * 2 + 16 * 8 + 16);
    if (a.N <= 16) scan_seq_kernel<T, 1><<<grid, 128, smem, s>>>(a);
    else if (a.N <= 32) scan_seq_kernel<T, 2><<<grid, 128, smem, s>>>(a);
    else if (a.N <= 64) scan_seq_kernel<T, 4><<<grid, 128, smem, s>>>(a);
    else if (a.N <= 128) scan_seq_kernel<T, 8><<<grid, 128, smem, s>>>(a);
    else scan_seq_kernel<T, 16><<<grid, 128, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_scan_seq(int dtype, const ScanArgs& a, cudaStream_t s)
{
    if (a.batch == 0 || a.L == 0) return cudaSuccess;
    return dtype == MM_BF16 ? scan_seq_dispatch<__nv_bfloat16>(a, s) : scan_seq_dispatch<float>(a, s);
}

// ====================================================================== gate + RMSNorm

// One warp per token: q = y * SiLU(z); out = q / sqrt(mean(q^2) + eps) * w.
// n = RMSNorm_d(y (x) SiLU(z)) (x) w, one CTA of 256 threads per row: each thread
// keeps q = y * SiLU(z) for up to kGateCols / 256 channels in registers between
// the sum of squares (a block reduction) and the scaled store.
constexpr int kGateThreads = 256, kGatePer = 16;  // rows up to 4096 channels stay in registers

template <typename T>
__global__ void __launch_bounds__(kGateThreads) gate_rmsnorm_kernel(const T* __restrict__ y, int64_t ldy,
                                                                    const T* __restrict__ z, int64_t ldz,
                                                                    const T* __restrict__ w, float eps, int d,
                                                                    T* __restrict__ out, int64_t ldo)
{
    __shared__ float wsum[kGateThreads / 32];
    const int row = blockIdx.x;
    const T* yr = y + (int64_t)row * ldy;
    const T* zr = z + (int64_t)row * ldz;
    T* orow = out + (int64_t)row * ldo;
    float q[kGatePer];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < kGatePer; ++i) {
        const int c = threadIdx.x + i * kGateThreads;
        q[i] = 0.0f;
        if (c < d) {
            q[i] = to_f32(yr[c]) * silu_f(to_f32(zr[c]));
            ss = fmaf(q[i], q[i], ss);
        }
    }
    for (int c = threadIdx.x + kGatePer * kGateThreads; c < d; c += kGateThreads) {  // wider rows
        const float v = to_f32(yr[c]) * silu_f(to_f32(zr[c]));
        ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int j = 0; j < kGateThreads / 32; ++j) tot += wsum[j];
    const float rstd = rsqrtf(tot / d + eps);
#pragma unroll
    for (int i = 0; i < kGatePer; ++i) {
        const int c = threadIdx.x + i * kGateThreads;
        if (c < d) orow[c] = from_f32<T>(q[i] * rstd * to_f32(w[c]));
    }
    for (int c = threadIdx.x + kGatePer * kGateThreads; c < d; c += kGateThreads) {
        const float v = to_f32(yr[c]) * silu_f(to_f32(zr[c]));
        orow[c] = from_f32<T>(v * rstd * to_f32(w[c]));
    }
}

cudaError_t launch_gate_rmsnorm(int dtype, const void* y, int64_t ldy, const void* z, int64_t ldz, const void* w,
                                float eps, int d, int rows, void* out, int64_t ldo, cudaStream_t s)
{
    if (rows == 0) return cudaSuccess;
    if (dtype == MM_BF16)
        gate_rmsnorm_kernel<__nv_bfloat16><<<rows, kGateThreads, 0, s>>>(
            (const __nv_bfloat16*)y, ldy, (const __nv_bfloat16*)z, ldz, (const __nv_bfloat16*)w, eps, d,
            (__nv_bfloat16*)out, ldo);
    else
        gate_rmsnorm_kernel<float><<<rows, kGateThreads, 0, s>>>((const float*)y, ldy, (const float*)z, ldz,
                                                                  (const float*)w, eps, d, (float*)out, ldo);
    return cudaGetLastError();
}

// ====================================================================== residual pre-norm

// One warp per row of the fp32 residual stream: out = x / sqrt(mean(x^2)+eps) * w.
template <typename T>
__global__ void rmsnorm_rows_kernel(const float* __restrict__ x, const T* __restrict__ w, float eps, int cols, int rows,
                                    T* __restrict__ out)
{
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* xr = x + (int64_t)row * cols;
    float ss = 0.0f;
    for (int c = lane; c < cols; c += 32) ss = fmaf(xr[c], xr[c], ss);
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rstd = rsqrtf(ss / cols + eps);
    for (int c = lane; c < cols; c += 32) out[(int64_t)row * cols + c] = from_f32<T>(xr[c] * rstd * to_f32(w[c]));
}

// The same for bf16 weights and output with cols = 128 NV: a lane keeps its NV float4 of the row in
// registers, so the row is read once with 16-byte loads and written with 8-byte stores.
template <int NV>
__global__ void rmsnorm_rows_vec_kernel(const float* __restrict__ x, const __nv_bfloat16* __restrict__ w, float eps,
                                        int rows, __nv_bfloat16* __restrict__ out)
{
    constexpr int cols = 128 * NV;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float4* xr = reinterpret_cast<const float4*>(x + (int64_t)row * cols);
    float4 v[NV];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        v[i] = xr[lane + 32 * i];
        ss = fmaf(v[i].x, v[i].x, ss);
        ss = fmaf(v[i].y, v[i].y, ss);
        ss = fmaf(v[i].z, v[i].z, ss);
        ss = fmaf(v[i].w, v[i].w, ss);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rstd = rsqrtf(ss / cols + eps);
    const uint2* wr = reinterpret_cast<const uint2*>(w);
    uint2* orow = reinterpret_cast<uint2*>(out + (int64_t)row * cols);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const uint2 wv = wr[lane + 32 * i];
        const float w0 = __uint_as_float(wv.x << 16), w1 = __uint_as_float(wv.x & 0xFFFF0000u);
        const float w2 = __uint_as_float(wv.y << 16), w3 = __uint_as_float(wv.y & 0xFFFF0000u);
        uint2 o;
        o.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[i].x * rstd * w0)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[i].y * rstd * w1)) << 16);
        o.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[i].z * rstd * w2)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[i].w * rstd * w3)) << 16);
        orow[lane + 32 * i] = o;
    }
}

cudaError_t launch_rmsnorm_rows_f32in(int dtype, const float* x, const void* w, float eps, int cols, int rows, void* out,
                                      cudaStream_t s)
{
    if (rows == 0) return cudaSuccess;
    dim3 grid((rows + 7) / 8);
    const bool vec = dtype == MM_BF16 && cols % 128 == 0 && cols <= 2048 &&
                     (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (reinterpret_cast<uintptr_t>(w) & 7u) == 0 &&
                     (reinterpret_cast<uintptr_t>(out) & 7u) == 0;
    if (vec) {
        const __nv_bfloat16* wb = (const __nv_bfloat16*)w;
        __nv_bfloat16* ob = (__nv_bfloat16*)out;
        switch (cols / 128) {
            case 1: rmsnorm_rows_vec_kernel<1><<<grid, 256, 0, s>>>(x, wb, eps, rows, ob); return cudaGetLastError();
            case 2: rmsnorm_rows_vec_kernel<2><<<grid, 256, 0, s>>>(x, wb, eps, rows, ob); return cudaGetLastError();
            case 4: rmsnorm_rows_vec_kernel<4><<<grid, 256, 0, s>>>(x, wb, eps, rows, ob); return cudaGetLastError();
            case 6: rmsnorm_rows_vec_kernel<6><<<grid, 256, 0, s>>>(x, wb, eps, rows, ob); return cudaGetLastError();
            case 8: rmsnorm_rows_vec_kernel<8><<<grid, 256, 0, s>>>(x, wb, eps, rows, ob); return cudaGetLastError();
            case 12: rmsnorm_rows_vec_kernel<12><<<grid, 256, 0, s>>>(x, wb, eps, rows, ob); return cudaGetLastError();
            case 16: rmsnorm_rows_vec_kernel<16><<<grid, 256, 0, s>>>(x, wb, eps, rows, ob); return cudaGetLastError();
            default: break;
        }
    }
    if (dtype == MM_BF16)
        rmsnorm_rows_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(x, (const __nv_bfloat16*)w, eps, cols, rows,
                                                                  (__nv_bfloat16*)out);
    else
        rmsnorm_rows_kernel<float><<<grid, 256, 0, s>>>(x, (const float*)w, eps, cols, rows, (float*)out);
    return cudaGetLastError();
}

template <typename T>
__global__ void to_f32_kernel(const T* __restrict__ in, float* __restrict__ out, int64_t n)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
        out[e] = to_f32(in[e]);
}

template <typename T>
__global__ void from_f32_kernel(const float* __restrict__ in, T* __restrict__ out, int64_t n)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
        out[e] = from_f32<T>(in[e]);
}

// bf16 -> fp32, four elements per thread (8-byte loads, 16-byte stores)
__global__ void to_f32_bf16x4_kernel(const uint2* __restrict__ in, float4* __restrict__ out, int64_t n4)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
        const uint2 v = in[e];
        out[e] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                             __uint_as_float(v.y & 0xFFFF0000u));
    }
}

cudaError_t launch_to_f32(int dtype, const void* in, float* out, int64_t n, cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    if (dtype == MM_BF16 && n % 4 == 0 && (reinterpret_cast<uintptr_t>(in) & 7u) == 0 &&
        (reinterpret_cast<uintptr_t>(out) & 15u) == 0) {
        const int64_t blocks = (n / 4 + 255) / 256;
        const int grid = (int)(blocks < 148 * 8 ? blocks : 148 * 8);
        to_f32_bf16x4_kernel<<<grid, 256, 0, s>>>(static_cast<const uint2*>(in), reinterpret_cast<float4*>(out), n / 4);
        return cudaGetLastError();
    }
    const int64_t blocks = (n + 255) / 256;
    const int grid = (int)(blocks < 148 * 16 ? blocks : 148 * 16);
    if (dtype == MM_BF16) to_f32_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)in, out, n);
    else to_f32_kernel<float><<<grid, 256, 0, s>>>((const float*)in, out, n);
    return cudaGetLastError();
}

// fp32 -> bf16, four elements per thread (16-byte loads, 8-byte stores)
__global__ void from_f32_bf16x4_kernel(const float4* __restrict__ in, uint2* __restrict__ out, int64_t n4)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
        const float4 v = in[e];
        uint2 o;
        o.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.x)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.y)) << 16);
        o.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.z)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.w)) << 16);
        out[e] = o;
    }
}

cudaError_t launch_from_f32(int dtype, const float* in, void* out, int64_t n, cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    if (dtype == MM_BF16 && n % 4 == 0 && (reinterpret_cast<uintptr_t>(in) & 15u) == 0 &&
        (reinterpret_cast<uintptr_t>(out) & 7u) == 0) {
        const int64_t blocks = (n / 4 + 255) / 256;
        const int grid = (int)(blocks < 148 * 8 ? blocks : 148 * 8);
        from_f32_bf16x4_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(in), static_cast<uint2*>(out), n / 4);
        return cudaGetLastError();
    }
    const int64_t blocks = (n + 255) / 256;
    const int grid = (int)(blocks < 148 * 16 ? blocks : 148 * 16);
    if (dtype == MM_BF16) from_f32_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(in, (__nv_bfloat16*)out, n);
    else from_f32_kernel<float><<<grid, 256, 0, s>>>(in, (float*)out, n);
    return cudaGetLastError();
}

// ====================================================================== decode step

// Conv window roll for one token: each thread owns one (sequence, channel),
// reads its K-1 stored inputs, appends the new one, writes the shifted window
// back and emits SiLU(conv).  Threads past nconv compute dt for one head.
template <typename T>
__global__ void step_conv_dt_kernel(const T* __restrict__ zxbc, int64_t ld_in, int col0, const float* __restrict__ dt_raw,
                                    const T* __restrict__ conv_w, const T* __restrict__ conv_b,
                                    const float* __restrict__ dt_bias, int E, int d, int nconv, int h, int K,
                                    T* __restrict__ conv_state, int conv_rows, T* __restrict__ xbc_out,
                                    float* __restrict__ dt_out)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    if (c >= nconv + h) return;
    if (c >= nconv) {
        const int i = c - nconv;
        dt_out[(int64_t)b * h + i] = softplus_f(dt_raw[(int64_t)b * h + i] + dt_bias[i]);
        return;
    }
    const int row = c < d ? c : E + (c - d);
    T* st = conv_state + ((int64_t)b * conv_rows + row) * (K - 1);
    const T vnew = zxbc[(int64_t)b * ld_in + col0 + c];
    float acc = to_f32(conv_b[row]);
    for (int j = 0; j < K; ++j) {
        const float v = j < K - 1 ? to_f32(st[j]) : to_f32(vnew);
        acc = fmaf(to_f32(conv_w[(int64_t)row * K + j]), v, acc);
    }
    for (int k = 0; k < K - 2; ++k) st[k] = st[k + 1];
    if (K > 1) st[K - 2] = vnew;
    xbc_out[(int64_t)b * nconv + c] = from_f32<T>(silu_f(acc));
}

// The same for bf16 and a window of 4 taps, four channels per thread: the three stored inputs of
// four channels are 24 contiguous bytes, their taps 32, so every access is an 8- or 16-byte vector.
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t v, int hi) { return __uint_as_float(hi ? (v & 0xFFFF0000u) : (v << 16)); }

__global__ void step_conv_dt4_kernel(const __nv_bfloat16* __restrict__ zxbc, int64_t ld_in, int col0,
                                     const float* __restrict__ dt_raw, const __nv_bfloat16* __restrict__ conv_w,
                                     const __nv_bfloat16* __restrict__ conv_b, const float* __restrict__ dt_bias, int E,
                                     int d, int nconv, int h, __nv_bfloat16* __restrict__ conv_state, int conv_rows,
                                     __nv_bfloat16* __restrict__ xbc_out, float* __restrict__ dt_out)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    const int ngrp = nconv / 4;
    if (t >= ngrp + h) return;
    if (t >= ngrp) {
        const int i = t - ngrp;
        dt_out[(int64_t)b * h + i] = softplus_f(dt_raw[(int64_t)b * h + i] + dt_bias[i]);
        return;
    }
    const int c0 = 4 * t;
    const int row0 = c0 < d ? c0 : E + (c0 - d);  // groups of four never straddle d (a multiple of 4)
    uint2* st = reinterpret_cast<uint2*>(conv_state + ((int64_t)b * conv_rows + row0) * 3);
    const uint2 s01 = st[0], s12 = st[1], s23 = st[2];  // channel j's inputs are bf16 [3 j, 3 j + 3) of these 12
    const uint32_t sw[6] = {s01.x, s01.y, s12.x, s12.y, s23.x, s23.y};
    const uint2 xn = *reinterpret_cast<const uint2*>(zxbc + (int64_t)b * ld_in + col0 + c0);
    const uint32_t xw[2] = {xn.x, xn.y};
    const uint4 w01 = *reinterpret_cast<const uint4*>(conv_w + (int64_t)row0 * 4);
    const uint4 w23 = *reinterpret_cast<const uint4*>(conv_w + (int64_t)row0 * 4 + 8);
    const uint32_t ww[8] = {w01.x, w01.y, w01.z, w01.w, w23.x, w23.y, w23.z, w23.w};
    const uint2 bb = *reinterpret_cast<const uint2*>(conv_b + row0);
    const uint32_t bw[2] = {bb.x, bb.y};
    float in[4][4];  // [channel][tap]: three stored inputs, then the new one
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int e = 3 * j + k;  // bf16 element of the 12 stored ones
            in[j][k] = bf16_bits_to_f32(sw[e >> 1], e & 1);
        }
        in[j][3] = bf16_bits_to_f32(xw[j >> 1], j & 1);
    }
    float out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float acc = bf16_bits_to_f32(bw[j >> 1], j & 1);
#pragma unroll
        for (int k = 0; k < 4; ++k) acc = fmaf(bf16_bits_to_f32(ww[(4 * j + k) >> 1], k & 1), in[j][k], acc);
        out[j] = silu_f(acc);
    }
    // the shifted window: channel j keeps inputs 1, 2 and the new one
    uint32_t nw[6];
#pragma unroll
    for (int e2 = 0; e2 < 6; ++e2) {
        uint32_t v = 0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int e = 2 * e2 + half, j = e / 3, k = e % 3;
            const __nv_bfloat16 q = __float2bfloat16_rn(in[j][k + 1]);  // exact: a bf16 value moves
            v |= (uint32_t)__bfloat16_as_ushort(q) << (16 * half);
        }
        nw[e2] = v;
    }
    st[0] = make_uint2(nw[0], nw[1]);
    st[1] = make_uint2(nw[2], nw[3]);
    st[2] = make_uint2(nw[4], nw[5]);
    uint2 o;
    o.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(out[0])) |
          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(out[1])) << 16);
    o.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(out[2])) |
          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(out[3])) << 16);
    *reinterpret_cast<uint2*>(xbc_out + (int64_t)b * nconv + c0) = o;
}

cudaError_t launch_step_conv_dt(int dtype, const void* zxbc, int64_t ld_in, int col0, const float* dt_raw,
                                const void* conv_w, const void* conv_b, const float* dt_bias, int E, int d, int nconv,
                                int h, int K, int batch, void* conv_state, int conv_rows, void* xbc_out, float* dt_out,
                                cudaStream_t s)
{
    auto al = [](const void* q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; };
    if (dtype == MM_BF16 && K == 4 && nconv % 4 == 0 && d % 4 == 0 && E % 4 == 0 && conv_rows % 4 == 0 &&
        ld_in % 4 == 0 && col0 % 4 == 0 && al(zxbc, 8) && al(conv_w, 16) && al(conv_b, 8) && al(conv_state, 8) &&
        al(xbc_out, 8)) {
        dim3 grid((nconv / 4 + h + 127) / 128, batch);
        step_conv_dt4_kernel<<<grid, 128, 0, s>>>(
            (const __nv_bfloat16*)zxbc, ld_in, col0, dt_raw, (const __nv_bfloat16*)conv_w, (const __nv_bfloat16*)conv_b,
            dt_bias, E, d, nconv, h, (__nv_bfloat16*)conv_state, conv_rows, (__nv_bfloat16*)xbc_out, dt_out);
        return cudaGetLastError();
    }
    dim3 grid((nconv + h + 127) / 128, batch);
    if (dtype == MM_BF16)
        step_conv_dt_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(
            (const __nv_bfloat16*)zxbc, ld_in, col0, dt_raw, (const __nv_bfloat16*)conv_w,
            (const __nv_bfloat16*)conv_b, dt_bias, E, d, nconv, h, K, (__nv_bfloat16*)conv_state, conv_rows,
            (__nv_bfloat16*)xbc_out, dt_out);
    else
        step_conv_dt_kernel<float><<<grid, 128, 0, s>>>((const float*)zxbc, ld_in, col0, dt_raw, (const float*)conv_w,
                                                         (const float*)conv_b, dt_bias, E, d, nconv, h, K,
                                                         (float*)conv_state, conv_rows, (float*)xbc_out, dt_out);
    return cudaGetLastError();
}

// State update for one token, H <- exp(dt A) H + dt x_p B; y_p = C . H + D x_p.
// One CTA per (sequence, head): B and C of the head's group are read once into
// registers and every warp walks state rows p = warp, warp + 8, ...  With
// N == 128 a lane owns state entries [4 lane, 4 lane + 4) of a row, so a warp
// moves a whole 512-byte row with one 16-byte load and one 16-byte store per lane.
template <typename T>
__global__ void __launch_bounds__(256) step_scan_kernel(const T* __restrict__ xbc, int nconv, int d,
                                                        const float* __restrict__ dt, const float* __restrict__ A,
                                                        const float* __restrict__ D, float* __restrict__ ssm_state,
                                                        int H, int h, int P, int N, int GN, int hpg, int vec,
                                                        T* __restrict__ y)
{
    const int b = blockIdx.x / h, i = blockIdx.x % h;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = i / hpg;
    const T* xr = xbc + (int64_t)b * nconv;
    const float dtv = dt[(int64_t)b * h + i];
    const float av = expf(dtv * A[i]);
    const float Di = D[i];
    const T* Bv = xr + d + g * N;
    const T* Cv = xr + d + GN + g * N;
    float* st = ssm_state + ((int64_t)b * H + i) * P * N;
    if (vec) {  // N == 128, 16-byte aligned state rows
        float bq[4], cq[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            bq[e] = to_f32(Bv[4 * lane + e]);
            cq[e] = to_f32(Cv[4 * lane + e]);
        }
        for (int p0 = warp; p0 < P; p0 += 16) {  // two rows in flight per warp
            const int p1 = p0 + 8;
            const bool two = p1 < P;
            float4* r0 = reinterpret_cast<float4*>(st + (int64_t)p0 * N) + lane;
            float4* r1 = reinterpret_cast<float4*>(st + (int64_t)p1 * N) + lane;
            float4 s0 = *r0, s1 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (two) s1 = *r1;
            const float x0 = to_f32(xr[i * P + p0]), x1 = two ? to_f32(xr[i * P + p1]) : 0.0f;
            const float d0 = dtv * x0, d1 = dtv * x1;
            s0.x = fmaf(av, s0.x, d0 * bq[0]); s0.y = fmaf(av, s0.y, d0 * bq[1]);
            s0.z = fmaf(av, s0.z, d0 * bq[2]); s0.w = fmaf(av, s0.w, d0 * bq[3]);
            s1.x = fmaf(av, s1.x, d1 * bq[0]); s1.y = fmaf(av, s1.y, d1 * bq[1]);
            s1.z = fmaf(av, s1.z, d1 * bq[2]); s1.w = fmaf(av, s1.w, d1 * bq[3]);
            *r0 = s0;
            if (two) *r1 = s1;
            float a0 = fmaf(cq[3], s0.w, fmaf(cq[2], s0.z, fmaf(cq[1], s0.y, cq[0] * s0.x)));
            float a1 = fmaf(cq[3], s1.w, fmaf(cq[2], s1.z, fmaf(cq[1], s1.y, cq[0] * s1.x)));
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                a0 += __shfl_xor_sync(0xffffffffu, a0, o);
                a1 += __shfl_xor_sync(0xffffffffu, a1, o);
            }
            if (lane == 0) {
                y[(int64_t)b * d + i * P + p0] = from_f32<T>(fmaf(Di, x0, a0));
                if (two) y[(int64_t)b * d + i * P + p1] = from_f32<T>(fmaf(Di, x1, a1));
            }
        }
        return;
    }
    for (int p = warp; p < P; p += 8) {  // any N: lanes stride the row
        const float xv = to_f32(xr[i * P + p]);
        const float dx = dtv * xv;
        float* row = st + (int64_t)p * N;
        float acc = 0.0f;
        for (int n = lane; n < N; n += 32) {
            const float hv = fmaf(av, row[n], dx * to_f32(Bv[n]));
            row[n] = hv;
            acc = fmaf(to_f32(Cv[n]), hv, acc);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) y[(int64_t)b * d + i * P + p] = from_f32<T>(fmaf(Di, xv, acc));
    }
}

// The same update with the gate folded into its output (bf16, N == 128, P == 64, 16-byte aligned
// state rows): instead of y it stores n = (y * SiLU(z)) * norm_w and, per (sequence, head, 32-channel
// half), the sum of squares of y * SiLU(z) into row_parts[b * 2h + 2 i + half]; the output projection
// then scales each row by 1/RMS.  The per-warp partial sums are added in warp order (deterministic).
__global__ void __launch_bounds__(256) step_scan_gated_kernel(const __nv_bfloat16* __restrict__ xbc, int nconv, int d,
                                                              const float* __restrict__ dt, const float* __restrict__ A,
                                                              const float* __restrict__ D, float* __restrict__ ssm_state,
                                                              int H, int h, int GN, int hpg,
                                                              const __nv_bfloat16* __restrict__ z, int64_t ldz,
                                                              const __nv_bfloat16* __restrict__ norm_w,
                                                              __nv_bfloat16* __restrict__ nrm, float* __restrict__ row_parts)
{
    constexpr int P = 64, N = 128;
    __shared__ float part[8][2];
    const int b = blockIdx.x / h, i = blockIdx.x % h;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = i / hpg;
    const __nv_bfloat16* xr = xbc + (int64_t)b * nconv;
    const __nv_bfloat16* zr = z + (int64_t)b * ldz;
    const float dtv = dt[(int64_t)b * h + i];
    const float av = expf(dtv * A[i]);
    const float Di = D[i];
    const __nv_bfloat16* Bv = xr + d + g * N;
    const __nv_bfloat16* Cv = xr + d + GN + g * N;
    float* st = ssm_state + ((int64_t)b * H + i) * P * N;
    float bq[4], cq[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        bq[e] = to_f32(Bv[4 * lane + e]);
        cq[e] = to_f32(Cv[4 * lane + e]);
    }
    // this warp's rows are p = warp + 8 j (j < 8); lane j < 8 fetches z and norm_w of row j up front and
    // later gates that row, so no dependent global load sits in the state loop
    float zr_l = 0.0f, nw_l = 0.0f;
    if (lane < 8) {
        const int c = i * P + warp + 8 * lane;
        zr_l = silu_f(to_f32(zr[c]));
        nw_l = to_f32(norm_w[c]);
    }
    float ssq = 0.0f;  // lane j's row (lanes < 8)
#pragma unroll 1
    for (int p0 = warp; p0 < P; p0 += 16) {  // rows p0 and p0 + 8: both in the same half
        const int p1 = p0 + 8;
        float4* r0 = reinterpret_cast<float4*>(st + (int64_t)p0 * N) + lane;
        float4* r1 = reinterpret_cast<float4*>(st + (int64_t)p1 * N) + lane;
        float4 s0 = *r0, s1 = *r1;
        const float x0 = to_f32(xr[i * P + p0]), x1 = to_f32(xr[i * P + p1]);
        const float d0 = dtv * x0, d1 = dtv * x1;
        s0.x = fmaf(av, s0.x, d0 * bq[0]); s0.y = fmaf(av, s0.y, d0 * bq[1]);
        s0.z = fmaf(av, s0.z, d0 * bq[2]); s0.w = fmaf(av, s0.w, d0 * bq[3]);
        s1.x = fmaf(av, s1.x, d1 * bq[0]); s1.y = fmaf(av, s1.y, d1 * bq[1]);
        s1.z = fmaf(av, s1.z, d1 * bq[2]); s1.w = fmaf(av, s1.w, d1 * bq[3]);
        *r0 = s0;
        *r1 = s1;
        float a0 = fmaf(cq[3], s0.w, fmaf(cq[2], s0.z, fmaf(cq[1], s0.y, cq[0] * s0.x)));
        float a1 = fmaf(cq[3], s1.w, fmaf(cq[2], s1.z, fmaf(cq[1], s1.y, cq[0] * s1.x)));
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            a0 += __shfl_xor_sync(0xffffffffu, a0, o);
            a1 += __shfl_xor_sync(0xffffffffu, a1, o);
        }
        // row p0 is lane j0 = (p0 - warp) / 8's, row p1 lane j0 + 1's
        const int j0 = (p0 - warp) >> 3;
        if (lane == j0 || lane == j0 + 1) {
            const bool second = lane == j0 + 1;
            const float q = fmaf(Di, second ? x1 : x0, second ? a1 : a0) * zr_l;
            ssq = q * q;
            nrm[(int64_t)b * d + i * P + (second ? p1 : p0)] = from_f32<__nv_bfloat16>(q * nw_l);
        }
    }
    // half 0 holds rows p < 32 (lanes 0-3), half 1 rows p >= 32 (lanes 4-7); summed in lane order
    float h0 = 0.0f, h1 = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float v = __shfl_sync(0xffffffffu, ssq, j);
        if (j < 4) h0 += v;
        else h1 += v;
    }
    const float ssq2[2] = {h0, h1};
    if (lane == 0) {
        part[warp][0] = ssq2[0];
        part[warp][1] = ssq2[1];
    }
    __syncthreads();
    if (threadIdx.x < 2) {
        float tot = 0.0f;
        for (int w = 0; w < 8; ++w) tot += part[w][threadIdx.x];
        row_parts[(int64_t)b * 2 * h + 2 * i + threadIdx.x] = tot;
    }
}

cudaError_t launch_step_scan_gated(const void* xbc, int nconv, int d, const float* dt, const float* A, const float* D,
                                   float* ssm_state, int H, int h, int GN, int hpg, int batch, const void* z,
                                   int64_t ldz, const void* norm_w, void* nrm, float* row_parts, cudaStream_t s)
{
    const int64_t heads = (int64_t)batch * h;
    if (heads == 0) return cudaSuccess;
    if (heads > 0x7fffffff) return cudaErrorInvalidValue;
    step_scan_gated_kernel<<<(unsigned)heads, 256, 0, s>>>(
        (const __nv_bfloat16*)xbc, nconv, d, dt, A, D, ssm_state, H, h, GN, hpg, (const __nv_bfloat16*)z, ldz,
        (const __nv_bfloat16*)norm_w, (__nv_bfloat16*)nrm, row_parts);
    return cudaGetLastError();
}

cudaError_t launch_step_scan(int dtype, const void* xbc, int nconv, int d, const float* dt, const float* A,
                             const float* D, float* ssm_state, int H, int h, int P, int N, int GN, int hpg, int batch,
                             void* y, cudaStream_t s)
{
    const int64_t heads = (int64_t)batch * h;
    if (heads == 0) return cudaSuccess;
    if (heads > 0x7fffffff) return cudaErrorInvalidValue;
    const int vec = N == 128 && (reinterpret_cast<uintptr_t>(ssm_state) & 15u) == 0;
    if (dtype == MM_BF16)
        step_scan_kernel<__nv_bfloat16><<<(unsigned)heads, 256, 0, s>>>((const __nv_bfloat16*)xbc, nconv, d, dt, A, D,
                                                                         ssm_state, H, h, P, N, GN, hpg, vec,
                                                                         (__nv_bfloat16*)y);
    else
        step_scan_kernel<float><<<(unsigned)heads, 256, 0, s>>>((const float*)xbc, nconv, d, dt, A, D, ssm_state, H, h,
                                                                 P, N, GN, hpg, vec, (float*)y);
    return cudaGetLastError();
}

}  // namespace mm

// Chunked selective scan on sm_100a tensor cores (bf16 x, B, C; fp32 dt, A, D
// and fp32 state), for d_head = 64 and d_state = 128.
//
// The scan H_t = exp(dt_t A) H_{t-1} + dt_t B_t x_t^T, y_t = C_t^T H_t + D x_t
// ("MatMamba: A Matryoshka State Space Model", block-definition paragraph:
// "chunk + selective scan", A and D learnable) is evaluated on blocks of
// Q = 128 tokens.  With cs_t the running sum of dt*A inside a block:
//   Y_diag = (Lmask o C B^T) (dt o X),  Lmask[t,s] = exp(cs_t - cs_s), s <= t
//   Y_off  = exp(cs_t) C_t^T H_prev
//   H_next = exp(cs_end) H_prev + B^T (w o X),  w_s = exp(cs_end - cs_s) dt_s
// which unrolls the recurrence exactly.  The sequence is cut into segments of
// whole blocks so that (batch, head, segment) CTAs fill the GPU:
//   1. seg_state  : each segment's end state from a zero start (tcgen05)
//   2. chunk_scan : every segment from its true start state (the initial state
//                   carried over the earlier segments' end states at the CTA's
//                   start), carrying the state across blocks in TMEM (tcgen05).
//                   It is a programmatic dependent of seg_state: segment 0 needs
//                   no carried state and may run beside it.
// Only segment end states touch HBM.
//
// A CTA takes two heads of one (batch, segment) so that the B and C blocks and
// G = C B^T are loaded and computed once per pair; the thread roles of the
// chunk scan are described above ssd_chunk_kernel.
#include <cuda.h>

#include <cmath>
#include <cstring>
#include <utility>

#include "mm_internal.cuh"
#include "sm100.cuh"

namespace mm {

using namespace sm100;

namespace {

constexpr int kQ = 128;                       // tokens per block
constexpr int kP = 64;                        // head dim
constexpr int kN = 128;                       // state dim
constexpr int kTileQN = kQ * kN * 2;              // C or B block: two 64-column panels
constexpr int kTileQP = kQ * kP * 2;              // x, X' or H block of one head: one panel
constexpr int kOffC = 0, kOffB = kTileQN, kOffX = 2 * kTileQN;
constexpr int kStage = 2 * kTileQN + 2 * kTileQP; // C | B | x of two heads
constexpr int kNStage = 2;
constexpr int kOffHX = kNStage * kStage;          // H (then X') of two heads

// TMEM columns: G = C B^T, overwritten in place by the masked M_0 | M_1 (A operands);
// Y_0 | Y_1; Y_off of both heads; S of both heads.
constexpr uint32_t kTG = 0, kTY = 128, kTYO = 256, kTS = 384, kTCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

struct ScanTcParams {
    int L, h, nseg, cps, nchunks, hpg;
    int c0;         // blocks in segment 0; segments 1.. take cps blocks each (the last may be shorter)
    int wait_all;   // 1: every chunk-scan CTA waits for the segment-state grid (y overlaps an input)
    const float* dt;
    int64_t sdt;
    const float* A;
    const float* D;
    void* y;
    int64_t sy;
    float* states;     // [b*h][nseg][P*N]: slot k = start state of segment k
    float* seg_decay;  // [b*h][nseg]: log2 of the decay over segment k (k < nseg - 1)
    const float* init_state;
    float* final_state;
    int64_t state_stride;
    int* status;
    // gated output (optional): y -> (y * SiLU(z)) * norm_w, sum of squares of y * SiLU(z) into row_sumsq
    const __nv_bfloat16* z;
    int64_t sz;
    const __nv_bfloat16* norm_w;
    float* row_parts;
    int y_tma;  // 1: y tiles leave through bulk tensor stores (mapY), 0: per-thread stores
};

__device__ __forceinline__ void named_sync_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128-byte-swizzled panel.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// 2^x on the MUFU unit (PTX ex2.approx.ftz: relative error ~2^-22, results below 2^-126 flush to 0,
// far below what the bf16 products built from it can hold).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// x / (1 + 2^(-x log2 e)) from the MUFU approximations of 2^x and 1/x (relative error of each
// about 2^-22); -0 for very negative x, where 2^(-x log2 e) overflows to +inf.
__device__ __forceinline__ float silu_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + ex2(-x * kLog2e)));
    return x * r;
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Chunk scan.  A CTA takes two heads of one (batch, segment); 512 threads in roles:
//   warps 0-7   M builders, except warp 4: thread (quarter q = warp % 4, lane) owns TMEM lane and
//               token row r = 32 q + lane and builds, for both heads, the masked decay matrix M
//               over some of its row's 32-token column blocks, in place over G = C B^T.  The two
//               warps of a quarter split the causal blocks (at most two blocks of both heads per
//               warp) and one of them writes the zero blocks above the diagonal.
//   warp 4      control: one lane issues the TMA loads and the tcgen05.mma; the warp owns TMEM
//   warps 8-15  state warps: thread (q, lane, head hf) owns row r of head hf: decay scan, state
//               read-back (bf16 copy for Y_off, decayed fp32 state for the S MMA), X', epilogue
// The M builders work on block k while the state warps finish block k-1's epilogue.  Per block
// k the tensor core runs G = C B^T (once Y of block k-1 has consumed M), Y_off = C [H_0 | H_1]
// (after the read-back), then Y_j = M_j X_j and S += B^T [X'_0 | X'_1] (after M and X').
// M factors the decay through the anchor of each 32-token column block cb (a_cb = cs at row
// 32 cb): 2^(cs_t - cs_s) dt_s = 2^(cs_t - a_cb) * (2^(a_cb - cs_s) dt_s) for s in block cb,
// s <= t.  The first factor is <= 1; the second, g_s, is a per-token table bounded by the decay
// across one 32-token block.  A block whose decay exceeds 2^-kDropMax would overflow g and
// takes direct exponentials instead (g_s = dt_s, M = G 2^min(cs_t - cs_s, 0) g_s).
// Element-wise products use the paired fp32 instructions (mul/fma .f32x2, rounded per lane
// exactly like their scalar forms).
// Blocks [c_begin, c_end) of segment `seg`.
__device__ __forceinline__ void seg_range(const ScanTcParams& p, int seg, int* c_begin, int* c_end)
{
    *c_begin = seg == 0 ? 0 : p.c0 + (seg - 1) * p.cps;
    *c_end = min(p.nchunks, seg == 0 ? p.c0 : *c_begin + p.cps);
}

// Programmatic dependent launch: let the dependent grid start, and wait for the
// prerequisite grid's completion (and its memory) before reading what it wrote.
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

constexpr int kChunkThreads = 512;
constexpr int kCtlWarp = 4;
constexpr float kDropMax = 100.0f;  // log2 units
// small tables after the H/X' buffers (floats): state-warp scan totals [2 parity][2 heads][4],
// M-builder scan totals [2][2][4], g [2 heads][128], cs [2][128], anchors [2][4], fallback flags [2][4]
constexpr int kTabWtotS = 0, kTabWtotM = 16, kTabG = 32, kTabC = 288, kTabAnch = 544, kTabFlag = 552, kTabFloats = 560;
constexpr int kOffTab = kOffHX + 2 * kTileQP;
constexpr int kOffBar = kOffTab + kTabFloats * 4;
constexpr int kChunkSmem = kOffBar + 11 * 8 + 16;
static_assert(kChunkSmem <= 232448, "chunk scan exceeds the 227 KB of shared memory a CTA can have");

__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 bf2(uint32_t v) { return make_float2(bf_lo(v), bf_hi(v)); }
__device__ __forceinline__ uint32_t pack2(float2 v) { return pack_bf16(v.x, v.y); }

__global__ void __launch_bounds__(kChunkThreads, 1)
    ssd_chunk_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapB,
                     const __grid_constant__ CUtensorMap mapC, const __grid_constant__ CUtensorMap mapY,
                     const ScanTcParams p)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    float* tab = reinterpret_cast<float*>(sm + kOffTab);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kOffBar);
    uint64_t* empty = full + kNStage;
    uint64_t* g_done = empty + kNStage;
    uint64_t* h_ready = g_done + 1;
    uint64_t* yo_done = h_ready + 1;
    uint64_t* mx_ready = yo_done + 1;
    uint64_t* ys_full = mx_ready + 1;  // all MMAs of the block done (Y, then S)
    uint64_t* y_done = ys_full + 1;    // Y of the block done (S may still run)
    uint64_t* done = y_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    // segment is the slowest grid dimension: segment 0's CTAs are scheduled first, on the SMs the
    // segment-state grid leaves free, since they need no carried state
    const int pair = blockIdx.x, b = blockIdx.y, seg = blockIdx.z;
    const int head0 = 2 * pair;
    int c_begin, c_end;
    seg_range(p, seg, &c_begin, &c_end);
    const int nch = max(c_end - c_begin, 0);
    const int grp = head0 / p.hpg;  // both heads of a pair share a group (hpg is even or G == 1)
    const int64_t tok0 = (int64_t)b * p.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNStage; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 8);
        }
        mbar_init(g_done, 1);
        mbar_init(h_ready, 8);
        mbar_init(yo_done, 1);
        mbar_init(mx_ready, 15);  // 7 M-builder warps and 8 state warps
        mbar_init(ys_full, 1);
        mbar_init(y_done, 1);
        mbar_init(done, 1);
        *abort = (smem_u32(sm) & 1023u) ? 1 : 0;  // tiles need 1024-byte alignment; never fault on it
        if (*abort) raise_timeout(abort, p.status);
        fence_mbar_init();
        prefetch_tmap(&mapX);
        prefetch_tmap(&mapB);
        prefetch_tmap(&mapC);
        if (p.y_tma) prefetch_tmap(&mapY);
    }
    if (warp == kCtlWarp) {
        tmem_alloc(tmem_slot, kTCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint8_t* sHX = sm + kOffHX;  // [2 heads] x 16 KB: bf16 state copy H, then X' of the current block

    if (warp == kCtlWarp) {
        if (lane == 0 && !*abort) {  // ------------------------------------ TMA loads and tcgen05.mma
            const uint32_t id_g = idesc_bf16(128, 128, 0, 0);   // C (K-major) x B (K-major)
            const uint32_t id_o = idesc_bf16(128, 128, 0, 1);   // C (K-major) x [H_0 | H_1] (MN-major)
            const uint32_t id_y = idesc_bf16(128, 64, 0, 1);    // M_j (TMEM) x X_j (MN-major)
            const uint32_t id_s = idesc_bf16(128, 128, 1, 1);   // B^T (MN-major) x [X'_0 | X'_1] (MN-major)
            const uint32_t aHX = smem_u32(sHX);
            auto load = [&](int c) {  // block c of the segment into stage c % 2
                const int s = c % kNStage;
                const int row = (int)(tok0 + (int64_t)(c_begin + c) * kQ);
                uint8_t* base = sm + s * kStage;
                mbar_arrive_expect_tx(&full[s], kStage);
                tma_load_2d(base + kOffC, &mapC, &full[s], grp * kN, row);
                tma_load_2d(base + kOffC + kTileQN / 2, &mapC, &full[s], grp * kN + 64, row);
                tma_load_2d(base + kOffB, &mapB, &full[s], grp * kN, row);
                tma_load_2d(base + kOffB + kTileQN / 2, &mapB, &full[s], grp * kN + 64, row);
                tma_load_2d(base + kOffX, &mapX, &full[s], head0 * kP, row);
                // a pair's second head past the last head reloads the last head (its dt is zero)
                tma_load_2d(base + kOffX + kTileQP, &mapX, &full[s], min(head0 + 1, p.h - 1) * kP, row);
            };
            int loaded = 0;  // blocks whose loads were issued
            for (; loaded < nch && loaded < kNStage; ++loaded) load(loaded);
            for (int k = 0; k < nch; ++k) {
                const int s = k % kNStage;
                // stage k is loaded, and block k-1's Y MMAs (which read M from the G columns) are done;
                // its S MMAs may still run, ahead of G in the tensor pipe
                if (!mbar_wait(&full[s], (k / kNStage) & 1, abort) ||
                    (k > 0 && !mbar_wait(y_done, (k - 1) & 1, abort))) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t aS = smem_u32(sm + s * kStage);
                const uint32_t aC = aS + kOffC, aB = aS + kOffB, aX = aS + kOffX;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // G = C . B^T
                    const uint32_t off = (kk & 3) * 32 + (kk >> 2) * (kTileQN / 2);
                    mma_ss(tmem + kTG, desc_sw128(aC + off, 16, 1024), desc_sw128(aB + off, 16, 1024), id_g, kk > 0);
                }
                mma_commit(g_done);
                if (!mbar_wait(h_ready, k & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // Y_off = C . [H_0 | H_1] over the state dim
                    const uint32_t off = (kk & 3) * 32 + (kk >> 2) * (kTileQN / 2);
                    mma_ss(tmem + kTYO, desc_sw128(aC + off, 16, 1024), desc_sw128(aHX + kk * 2048, kTileQP, 1024),
                           id_o, kk > 0);
                }
                mma_commit(yo_done);
                // block k+1 goes into the stage block k-1 used, free once its epilogue has read x and
                // its y tile has left (released after the read-back that h_ready waited for)
                if (loaded == k + 1 && loaded < nch) {
                    if (!mbar_wait(&empty[loaded % kNStage], ((loaded / kNStage) & 1) ^ 1, abort)) {
                        raise_timeout(abort, p.status);
                        break;
                    }
                    load(loaded++);
                }
                if (!mbar_wait(mx_ready, k & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                // Y first, so the epilogue can start while S still runs
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // Y_j = M_j . X_j over the block's tokens
                        mma_ts(tmem + kTY + 64 * j, tmem + kTG + 32 * (kk >> 1) + 16 * j + 8 * (kk & 1),
                               desc_sw128(aX + j * kTileQP + kk * 2048, kTileQP, 1024), id_y, kk > 0);
                mma_commit(y_done);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // S += B^T . [X'_0 | X'_1] over the block's tokens
                    mma_ss(tmem + kTS, desc_sw128(aB + kk * 2048, kTileQN / 2, 1024),
                           desc_sw128(aHX + kk * 2048, kTileQP, 1024), id_s, 1u);
                mma_commit(ys_full);
            }
            // every issued load lands before the CTA exits (bounded; only the last two can be pending)
            for (int j = max(0, loaded - kNStage); j < loaded; ++j) mbar_wait(&full[j % kNStage], (j / kNStage) & 1, abort);
            mma_commit(done);
            mbar_wait(done, 0, nullptr);
        }
    } else if (warp < 8) {  // ------------------------------------------------------ M builders
        const int q = warp & 3, hb = warp >> 2, r = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        // causal column blocks of this warp, and the zero blocks it writes
        // quarter 0: {0} (its second warp is the control warp); 1: {0} {1}; 2: {0,1} {2}; 3: {0,1} {2,3}
        const int cb_lo = hb == 0 ? 0 : (q >= 2 ? 2 : 1);
        const int cb_hi = hb == 0 ? (q >= 2 ? 1 : 0) : q;  // inclusive
        const bool zero_writer = (q <= 1) ? hb == 0 : hb == 1;
        float A2[2], dn[2] = {0.0f, 0.0f};
#pragma unroll
        for (int j = 0; j < 2; ++j) A2[j] = head0 + j < p.h ? p.A[head0 + j] * kLog2e : 0.0f;
        if (nch > 0 && c_begin * kQ + r < p.L) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
                if (head0 + j < p.h) dn[j] = p.dt[(tok0 + c_begin * kQ + r) * p.sdt + head0 + j];
        }
        for (int k = 0; k < nch; ++k) {  // every warp runs every iteration (named barrier 1)
            const float dv[2] = {dn[0], dn[1]};
            const int t1 = (c_begin + k + 1) * kQ + r;
            dn[0] = dn[1] = 0.0f;
            if (k + 1 < nch && t1 < p.L) {  // prefetch the next block's dt
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    if (head0 + j < p.h) dn[j] = p.dt[(tok0 + t1) * p.sdt + head0 + j];
            }
            float* wt = tab + kTabWtotM + 8 * (k & 1);
            float c2[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {  // inclusive scan of dt A (log2 units) within the warp
                float sc = dv[j] * A2[j];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, sc, o);
                    if (lane >= o) sc += v;
                }
                if (lane == 31 && hb == 0) wt[4 * j + q] = sc;
                c2[j] = sc;
            }
            asm volatile("bar.sync 1, 224;" ::: "memory");
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float pre = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) pre += i < q ? wt[4 * j + i] : 0.0f;
                c2[j] += pre;
                if (hb == 0) {  // this row block's anchor (cs at its first row) and the decay across it
                    const float a = __shfl_sync(0xffffffffu, c2[j], 0);
                    const float last = __shfl_sync(0xffffffffu, c2[j], 31);
                    const bool fb = a - last > kDropMax;
                    tab[kTabG + 128 * j + r] = fb ? dv[j] : ex2(a - c2[j]) * dv[j];
                    tab[kTabC + 128 * j + r] = c2[j];
                    if (lane == 0) {
                        tab[kTabAnch + 4 * j + q] = a;
                        tab[kTabFlag + 4 * j + q] = fb ? 1.0f : 0.0f;
                    }
                }
            }
            asm volatile("bar.sync 1, 224;" ::: "memory");  // tables of block k complete

            const bool ok = __all_sync(0xffffffffu, mbar_wait(g_done, k & 1, abort));
            if (ok) {
                tc_fence_after();
                if (zero_writer) {  // above the diagonal: zeros for both heads
                    uint32_t z[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) z[e] = 0u;
#pragma unroll
                    for (int cb = 1; cb < 4; ++cb)
                        if (cb > q) tmem_st32(tmem + lane_base + kTG + 32 * cb, z);
                }
#pragma unroll 1
                for (int cb = cb_lo; cb <= cb_hi; ++cb) {  // column block s in [32 cb, 32 cb + 32)
                    uint32_t gv[32];
                    tmem_ld32(tmem + lane_base + kTG + 32 * cb, gv);
                    tmem_ld_wait();
                    const bool diag = cb == q;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        uint32_t pk[16];
                        const float* gt = tab + kTabG + 128 * j + 32 * cb;
                        if (tab[kTabFlag + 4 * j + cb] == 0.0f) {
                            const float er = ex2(c2[j] - tab[kTabAnch + 4 * j + cb]);
                            const float2 er2 = make_float2(er, er);
#pragma unroll
                            for (int e = 0; e < 32; e += 4) {
                                const float4 g4 = *reinterpret_cast<const float4*>(gt + e);
                                float2 m01 = mul2(mul2(make_float2(__uint_as_float(gv[e]), __uint_as_float(gv[e + 1])), er2),
                                                  make_float2(g4.x, g4.y));
                                float2 m23 = mul2(mul2(make_float2(__uint_as_float(gv[e + 2]), __uint_as_float(gv[e + 3])), er2),
                                                  make_float2(g4.z, g4.w));
                                if (diag) {  // causal mask inside the diagonal block: s <= t
                                    m01.x = e <= lane ? m01.x : 0.0f;
                                    m01.y = e + 1 <= lane ? m01.y : 0.0f;
                                    m23.x = e + 2 <= lane ? m23.x : 0.0f;
                                    m23.y = e + 3 <= lane ? m23.y : 0.0f;
                                }
                                pk[e >> 1] = pack2(m01);
                                pk[(e >> 1) + 1] = pack2(m23);
                            }
                        } else {  // steep block: direct exponentials, g holds dt
                            const float* ct = tab + kTabC + 128 * j + 32 * cb;
#pragma unroll
                            for (int e = 0; e < 32; e += 2) {
                                float m0 = __uint_as_float(gv[e]) * ex2(fminf(c2[j] - ct[e], 0.0f)) * gt[e];
                                float m1 = __uint_as_float(gv[e + 1]) * ex2(fminf(c2[j] - ct[e + 1], 0.0f)) * gt[e + 1];
                                if (diag) {
                                    m0 = e <= lane ? m0 : 0.0f;
                                    m1 = e + 1 <= lane ? m1 : 0.0f;
                                }
                                pk[e >> 1] = pack_bf16(m0, m1);
                            }
                        }
                        // head j's 16 packed columns of this block (the A operand of Y_j)
                        tmem_st16(tmem + lane_base + kTG + 32 * cb + 16 * j, pk);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(mx_ready);
            } else {
                raise_timeout(abort, p.status);
            }
        }
    } else {  // ------------------------------------------------------------------- state warps
        const int cw = warp - 8, q = warp & 3, hf = cw >> 2;
        const int r = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int head = head0 + hf;
        const bool head_ok = head < p.h;
        const float A2 = head_ok ? p.A[head] * kLog2e : 0.0f;
        const float Dh = (p.D && head_ok) ? p.D[head] : 0.0f;
        const int64_t bh = (int64_t)b * p.h + head;
        const int PN = kP * kN;
        uint8_t* myHX = sHX + hf * kTileQP;
        const uint32_t bar_id = 2 + hf;

        // The fp32 state of this head lives in TMEM columns kTS + 64 hf (row n = lane r): each
        // block, it is read for its bf16 copy (Y_off's operand), 2^tot H_k is written back, and
        // the S MMA accumulates B^T X' on top, leaving H_{k+1}.  A segment's start state is the
        // initial state (or zero) carried over the earlier segments:
        // H <- 2^decay_j H + S_j, S_j being segment j's end state from a zero start.
        {
            if (p.nseg > 1 && (seg > 0 || p.wait_all)) grid_dependency_wait();  // segment end states written
            const float* init = (head_ok && p.init_state)
                                    ? p.init_state + (int64_t)b * p.state_stride + (int64_t)head * PN
                                    : nullptr;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = init ? init[(32 * h2 + j) * kN + r] : 0.0f;
                for (int sj = 0; head_ok && sj < seg; ++sj) {
                    const float dec = exp2f(p.seg_decay[bh * p.nseg + sj]);
                    const float* sp = p.states + (bh * p.nseg + sj + 1) * PN;
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = fmaf(dec, v[j], sp[(32 * h2 + j) * kN + r]);
                }
                uint32_t u[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(v[j]);
                tmem_st32(tmem + lane_base + kTS + 64 * hf + 32 * h2, u);
            }
            tmem_st_wait();
        }
        float dt_next = 0.0f;
        if (head_ok && nch > 0 && c_begin * kQ + r < p.L) dt_next = p.dt[(tok0 + c_begin * kQ + r) * p.sdt + head];
        float c2_prev = 0.0f;
        bool ok = __all_sync(0xffffffffu, !*abort);
        bool pending_release = false;  // the storing warp still owes the previous stage's release

        // Iteration k: decay scan of block k, epilogue of block k-1, read-back and X' of block k.
        // Every warp runs every iteration (named barrier 2 + hf); a failed wait skips work only.
        for (int k = 0; k <= nch; ++k) {
            float dtv = 0.0f, c2 = 0.0f, tot = 0.0f;
            if (k < nch) {
                dtv = dt_next;
                const int t1 = (c_begin + k + 1) * kQ + r;
                dt_next = (head_ok && k + 1 < nch && t1 < p.L) ? p.dt[(tok0 + t1) * p.sdt + head] : 0.0f;
                float sc = dtv * A2;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, sc, o);
                    if (lane >= o) sc += v;
                }
                float* wt = tab + kTabWtotS + 8 * (k & 1) + 4 * hf;
                if (lane == 31) wt[q] = sc;
                asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
                float pre = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float w = wt[i];
                    pre += i < q ? w : 0.0f;
                    tot += w;
                }
                c2 = sc + pre;
            }

            if (k > 0) {  // ---- epilogue of block k-1 (TMEM loads are warp-collective)
                if (ok) ok = __all_sync(0xffffffffu, mbar_wait(y_done, (k - 1) & 1, abort));
                const int sp = (k - 1) % kNStage;
                const int tp0 = (c_begin + k - 1) * kQ;
                // x of block k-1 (this head); with bulk stores each thread overwrites its own row of
                // it with its y row, in the same swizzled layout, once that row's x has been read
                uint8_t* sX = sm + sp * kStage + kOffX + hf * kTileQP;
                if (ok) {
                    tc_fence_after();
                    const bool valid = head_ok && tp0 + r < p.L;
                    const float ey = ex2(c2_prev);
                    const float2 ey2 = make_float2(ey, ey), dh2 = make_float2(Dh, Dh);
                    const int64_t tok = tok0 + tp0 + r;
                    const int col = head * kP;
                    __nv_bfloat16* yo = static_cast<__nv_bfloat16*>(p.y) + tok * p.sy + col;
                    float ssq[2] = {0.0f, 0.0f};
                    // z rows of this warp's 32 tokens, loaded four rows per instruction (coalesced) into
                    // this warp's 4 KB of block k-1's C tile, which no MMA reads any more
                    uint8_t* zs = sm + sp * kStage + kOffC + hf * (kTileQN / 2) + 32 * q * 128;
                    if (p.z) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int rr = (lane >> 3) + 4 * i, ch = lane & 7;
                            uint4 zv = make_uint4(0, 0, 0, 0);
                            if (head_ok && tp0 + 32 * q + rr < p.L)
                                zv = *reinterpret_cast<const uint4*>(p.z + (tok0 + tp0 + 32 * q + rr) * p.sz + col + 8 * ch);
                            *reinterpret_cast<uint4*>(zs + rr * 128 + ((ch ^ (rr & 7)) << 4)) = zv;
                        }
                        __syncwarp();
                    }
#pragma unroll
                    for (int h2 = 0; h2 < 4; ++h2) {  // 16 output columns at a time
                        uint32_t yv[16], ov[16];
                        tmem_ld16(tmem + lane_base + kTY + 64 * hf + 16 * h2, yv);
                        tmem_ld16(tmem + lane_base + kTYO + 64 * hf + 16 * h2, ov);
                        tmem_ld_wait();
                        if (!valid && !p.y_tma) continue;
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const int cc = 2 * h2 + c;
                            const uint4 xv = *reinterpret_cast<const uint4*>(sX + sw128(r, cc));
                            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                            uint4 zw4 = make_uint4(0, 0, 0, 0), nw4 = make_uint4(0, 0, 0, 0);
                            if (p.z && valid) {
                                zw4 = *reinterpret_cast<const uint4*>(zs + lane * 128 + ((cc ^ (lane & 7)) << 4));
                                nw4 = *reinterpret_cast<const uint4*>(p.norm_w + col + 8 * cc);
                            }
                            const uint32_t zw[4] = {zw4.x, zw4.y, zw4.z, zw4.w};
                            const uint32_t nw[4] = {nw4.x, nw4.y, nw4.z, nw4.w};
                            uint32_t o[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = 8 * c + 2 * e;
                                // y = Y + 2^cs Y_off + D x, two columns at a time
                                float2 a = fma2(ey2, make_float2(__uint_as_float(ov[j]), __uint_as_float(ov[j + 1])),
                                                make_float2(__uint_as_float(yv[j]), __uint_as_float(yv[j + 1])));
                                a = fma2(dh2, bf2(xw[e]), a);
                                if (p.z) {
                                    const float z0 = bf_lo(zw[e]), z1 = bf_hi(zw[e]);
                                    a = mul2(a, make_float2(silu_approx(z0), silu_approx(z1)));
                                    ssq[h2 >> 1] = fmaf(a.x, a.x, fmaf(a.y, a.y, ssq[h2 >> 1]));
                                    a = mul2(a, bf2(nw[e]));
                                }
                                o[e] = pack2(a);
                            }
                            if (p.y_tma) *reinterpret_cast<uint4*>(sX + sw128(r, cc)) = make_uint4(o[0], o[1], o[2], o[3]);
                            else reinterpret_cast<uint4*>(yo)[cc] = make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    }
                    if (p.z && valid) {
                        p.row_parts[tok * 2 * p.h + 2 * head] = ssq[0];
                        p.row_parts[tok * 2 * p.h + 2 * head + 1] = ssq[1];
                    }
                    tc_fence_before();
                }
                if (p.y_tma) {  // the head's 128 x 64 tile leaves in one bulk store (rows past L clipped)
                    fence_async_smem();
                    asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
                    if (q == 0) {
                        ok = __all_sync(0xffffffffu, ok && !*abort);
                        if (ok && head_ok && lane == 0) {
                            tma_store_3d(&mapY, sX, head * kP, tp0, b);
                            bulk_commit();
                        }
                        __syncwarp();
                    }
                }
                // Block k-1's stage is released after the read-back below, which waits for its S MMA
                // (S reads B there); the storing warp also waits for its store to read the y tile.
                pending_release = ok;
            }
            if (k == nch) break;

            const int s = k % kNStage;
            if (ok && k > 0) ok = __all_sync(0xffffffffu, mbar_wait(ys_full, (k - 1) & 1, abort));  // S done
            if (ok) {  // ---- read-back: H_k as bf16 for Y_off, 2^tot H_k back into TMEM
                const float dec = ex2(tot);
                const float2 dec2 = make_float2(dec, dec);
#pragma unroll
                for (int h4 = 0; h4 < 4; ++h4) {  // 16 state columns at a time
                    uint32_t v[16];
                    tmem_ld16(tmem + lane_base + kTS + 64 * hf + 16 * h4, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1]));
                        w.y = pack_bf16(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3]));
                        w.z = pack_bf16(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5]));
                        w.w = pack_bf16(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]));
                        *reinterpret_cast<uint4*>(myHX + sw128(r, 2 * h4 + c)) = w;
                    }
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        const float2 d = mul2(dec2, make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])));
                        v[j] = __float_as_uint(d.x);
                        v[j + 1] = __float_as_uint(d.y);
                    }
                    tmem_st16(tmem + lane_base + kTS + 64 * hf + 16 * h4, v);
                }
                tmem_st_wait();
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(h_ready);
            }
            if (pending_release) {  // block k-1 is done with its stage: release it
                if (lane == 0) {
                    if (p.y_tma && q == 0) bulk_wait_read0();  // the y tile has been read
                    mbar_arrive(&empty[(k - 1) % kNStage]);
                }
                __syncwarp();
                pending_release = false;
            }
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (k / kNStage) & 1, abort));
            if (ok) {  // ---- X'_j[s=r, :] = 2^(tot - cs_r) dt_r x_j[r, :], formed while Y_off runs
                const uint8_t* sX = sm + s * kStage + kOffX + hf * kTileQP;
                const float wgt = ex2(tot - c2) * dtv;
                const float2 w2 = make_float2(wgt, wgt);
                uint4 xq[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 xv = *reinterpret_cast<const uint4*>(sX + sw128(r, c));
                    xq[c].x = pack2(mul2(bf2(xv.x), w2));
                    xq[c].y = pack2(mul2(bf2(xv.y), w2));
                    xq[c].z = pack2(mul2(bf2(xv.z), w2));
                    xq[c].w = pack2(mul2(bf2(xv.w), w2));
                }
                ok = __all_sync(0xffffffffu, mbar_wait(yo_done, k & 1, abort));  // H read: X' may go there
                if (ok) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(myHX + sw128(r, c)) = xq[c];
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(mx_ready);
                }
            }
            if (!ok) raise_timeout(abort, p.status);
            c2_prev = c2;
        }

        if (p.y_tma && q == 0 && lane == 0) bulk_wait0();  // this head's y tiles are in global memory
        if (seg == p.nseg - 1 && p.final_state) {  // state after the last block: its S MMA is done
            if (ok && nch > 0) ok = __all_sync(0xffffffffu, mbar_wait(ys_full, (nch - 1) & 1, abort));
            ok = __all_sync(0xffffffffu, ok && !*abort);
            if (ok) {
                float* dst = p.final_state + (int64_t)b * p.state_stride + (int64_t)head * PN;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_base + kTS + 64 * hf + 32 * h2, v);
                    tmem_ld_wait();
                    if (head_ok) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) dst[(32 * h2 + j) * kN + r] = __uint_as_float(v[j]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kCtlWarp) tmem_dealloc(tmem, kTCols);
}

// Segment end states from a zero start, for every segment but the last:
//   S_seg = sum_s 2^(cs_end - cs_s) dt_s B_s x_s^T        (cs in log2 units, over the segment)
// The segment's blocks are visited last to first.  With D the decay of the
// blocks already visited (those after the current one), token s of the block
// gets the weight 2^(D + tot - cs_s) <= 1, and every block's B^T X'' is
// accumulated into one TMEM accumulator: no per-block state update, and the
// compute warps wait for the tensor core only to reuse one of two X'' buffers.
// Two heads per CTA as in the chunk scan; S of head j sits in TMEM columns
// [64 j, 64 j + 64), row n = state dim.
constexpr int kSegStage = kTileQN + 2 * kTileQP;          // B | x of two heads
constexpr int kSegOffXP = kNStage * kSegStage;            // two X'' buffers of two heads
constexpr int kSegOffSmall = kSegOffXP + 2 * 2 * kTileQP;
constexpr int kSegSmemBytes = kSegOffSmall + 2 * kQ * 4 + 32 + 256;

__global__ void __launch_bounds__(320, 1)
    ssd_seg_state_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapB,
                         const ScanTcParams p)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    float* wtot = reinterpret_cast<float*>(sm + kSegOffSmall);  // [2 heads][4]
    uint64_t* full = reinterpret_cast<uint64_t*>(wtot + 8 + 2 * kQ);
    uint64_t* empty = full + kNStage;
    uint64_t* xr = empty + kNStage;   // X'' buffer written (compute -> MMA)
    uint64_t* xf = xr + 2;            // X'' buffer consumed (MMA -> compute)
    uint64_t* done = xf + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int pair = blockIdx.x, seg = blockIdx.y, b = blockIdx.z;
    const int head0 = 2 * pair;
    int c_begin, c_end;
    seg_range(p, seg, &c_begin, &c_end);
    const int nch = max(c_end - c_begin, 0);
    const int grp = head0 / p.hpg;
    const int64_t tok0 = (int64_t)b * p.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_launch_dependents();  // the chunk scan may start its first segment beside this grid

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNStage; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
            mbar_init(&xr[i], 8);
            mbar_init(&xf[i], 1);
        }
        mbar_init(done, 1);
        *abort = (smem_u32(sm) & 1023u) ? 1 : 0;
        if (*abort) raise_timeout(abort, p.status);
        fence_mbar_init();
        prefetch_tmap(&mapX);
        prefetch_tmap(&mapB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && !*abort) {  // TMA producer, blocks last to first
            int k = 0;
            for (; k < nch; ++k) {
                const int s = k % kNStage;
                if (!mbar_wait(&empty[s], ((k / kNStage) & 1) ^ 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                const int row = (int)(tok0 + (int64_t)(c_end - 1 - k) * kQ);
                uint8_t* base = sm + s * kSegStage;
                mbar_arrive_expect_tx(&full[s], kSegStage);
                tma_load_2d(base, &mapB, &full[s], grp * kN, row);
                tma_load_2d(base + kTileQN / 2, &mapB, &full[s], grp * kN + 64, row);
                tma_load_2d(base + kTileQN, &mapX, &full[s], head0 * kP, row);
                tma_load_2d(base + kTileQN + kTileQP, &mapX, &full[s], min(head0 + 1, p.h - 1) * kP, row);
            }
            for (int j = max(0, k - kNStage); j < k; ++j) mbar_wait(&full[j % kNStage], (j / kNStage) & 1, abort);
        }
    } else if (warp == 1) {
        if (lane == 0 && !*abort) {  // MMA issuer: S += B^T [X''_0 | X''_1]
            const uint32_t id_s = idesc_bf16(128, 128, 1, 1);
            for (int k = 0; k < nch; ++k) {
                const int s = k % kNStage, xb = k & 1;
                if (!mbar_wait(&full[s], (k / kNStage) & 1, abort) || !mbar_wait(&xr[xb], (k >> 1) & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t aB = smem_u32(sm + s * kSegStage);
                const uint32_t aXP = smem_u32(sm + kSegOffXP + xb * 2 * kTileQP);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmem, desc_sw128(aB + kk * 2048, kTileQN / 2, 1024), desc_sw128(aXP + kk * 2048, kTileQP, 1024),
                           id_s, (k | kk) != 0);
                mma_commit(&xf[xb]);
                mma_commit(&empty[s]);
            }
            mma_commit(done);
            mbar_wait(done, 0, nullptr);  // every issued MMA is done before TMEM can be released (bounded)
        }
    } else {  // compute warps: thread (quarter q, lane) = token / state row r, head hf of the pair
        const int cw = warp - 2, q = warp & 3, hf = cw >> 2;
        const int r = q * 32 + lane;
        const int head = head0 + hf;
        const bool head_ok = head < p.h;
        const float A2 = head_ok ? p.A[head] * kLog2e : 0.0f;
        float D2 = 0.0f;
        float dt_next = 0.0f;
        if (head_ok && nch > 0) {
            const int t0 = (c_end - 1) * kQ;
            if (t0 + r < p.L) dt_next = p.dt[(tok0 + t0 + r) * p.sdt + head];
        }
        for (int k = 0; k < nch; ++k) {  // every warp runs every iteration (named barriers)
            const int s = k % kNStage, xb = k & 1;
            const int t0 = (c_end - 1 - k) * kQ;
            const float dtv = dt_next;
            if (k + 1 < nch) {
                const int t1 = t0 - kQ;
                dt_next = (head_ok && t1 + r < p.L) ? p.dt[(tok0 + t1 + r) * p.sdt + head] : 0.0f;
            }
            float sc = dtv * A2;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, sc, o);
                if (lane >= o) sc += v;
            }
            if (lane == 31) wtot[hf * 4 + q] = sc;
            named_sync_compute();
            float pre = 0.0f, tot = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float w = wtot[hf * 4 + j];
                pre += j < q ? w : 0.0f;
                tot += w;
            }
            named_sync_compute();
            const float c2 = sc + pre;
            bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (k / kNStage) & 1, abort));
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&xf[xb], ((k >> 1) & 1) ^ 1, abort));
            if (ok) {  // X''[r, :] = 2^(D + tot - cs_r) dt_r x[r, :]
                const float wgt = ex2(D2 + tot - c2) * dtv;
                const uint8_t* sX = sm + s * kSegStage + kTileQN + hf * kTileQP;
                uint8_t* dX = sm + kSegOffXP + xb * 2 * kTileQP + hf * kTileQP;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 xv = *reinterpret_cast<const uint4*>(sX + sw128(r, c));
                    uint4 o;
                    o.x = pack_bf16(bf_lo(xv.x) * wgt, bf_hi(xv.x) * wgt);
                    o.y = pack_bf16(bf_lo(xv.y) * wgt, bf_hi(xv.y) * wgt);
                    o.z = pack_bf16(bf_lo(xv.z) * wgt, bf_hi(xv.z) * wgt);
                    o.w = pack_bf16(bf_lo(xv.w) * wgt, bf_hi(xv.w) * wgt);
                    *reinterpret_cast<uint4*>(dX + sw128(r, c)) = o;
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xr[xb]);
            } else {
                raise_timeout(abort, p.status);
            }
            D2 += tot;
        }
        const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0, abort));
        if (ok) {
            tc_fence_after();
            float* dst = p.states + (((int64_t)b * p.h + head) * p.nseg + seg + 1) * (kP * kN);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t sv[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + 64 * hf + 32 * h2, sv);
                tmem_ld_wait();
                if (head_ok && !*abort) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) dst[(32 * h2 + j) * kN + r] = __uint_as_float(sv[j]);
                }
            }
            if (head_ok && r == 0 && !*abort) p.seg_decay[((int64_t)b * p.h + head) * p.nseg + seg] = D2;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem, 128);
    }
}

struct Plan {
    int nchunks, nseg, cps;
    int c0;       // blocks of segment 0 (>= cps when it runs beside the segment-state grid)
    bool overlap;  // segment 0's CTAs fit beside the segment-state grid
};

Plan plan_for(const ScanArgs& a, int sms)
{
    // Costs in units of one 128-token block of chunk-scan work per CTA.  A CTA also pays a
    // fixed start (TMEM, barriers, state fold and pipeline fill: about 1.5 blocks).  A block of
    // the segment-state pass costs about 0.3 of a chunk-scan block.  Segment 0 needs no carried
    // state: when its CTAs fit on the SMs the segment-state grid leaves free, it starts at once
    // and may take more blocks than the others, which start after the segment-state grid.
    Plan pl;
    pl.nchunks = (a.L + kQ - 1) / kQ;
    const int64_t ctas = (int64_t)a.batch * ((a.h + 1) / 2);  // CTAs per segment: head pairs
    double best = 1e30;
    pl.nseg = 1;
    pl.cps = pl.nchunks;
    pl.c0 = pl.nchunks;
    pl.overlap = false;
    for (int ns = 1; ns <= pl.nchunks && ns <= 64; ++ns) {
        const bool overlap = ns > 1 && ctas * ns <= sms;
        const int even = (pl.nchunks + ns - 1) / ns;
        // segment 0 of c0 blocks, the others of c1 blocks each (the last one shorter, never empty);
        // only an overlapped segment 0 may be longer than the even split
        for (int c0 = even; c0 <= (overlap ? pl.nchunks - (ns - 1) : even); ++c0) {
            const int rest = pl.nchunks - c0;
            int c1 = 0;
            double cost;
            if (ns == 1) {
                cost = std::ceil((double)ctas / sms) * (c0 + 1.5);
            } else {
                if (rest < ns - 1) continue;
                c1 = (rest + ns - 2) / (ns - 1);
                if (rest - (ns - 2) * c1 <= 0) continue;
                const double seg_pass = 0.3 * std::ceil((double)(ctas * (ns - 1)) / sms) * (std::max(c0, c1) + 1.5) + 0.4;
                cost = overlap ? std::max(c0 + 1.5, seg_pass + (c1 + 1.5))
                               : seg_pass + std::ceil((double)(ctas * ns) / sms) * (std::max(c0, c1) + 1.5);
            }
            if (cost < best - 1e-9) {
                best = cost;
                pl.nseg = ns;
                pl.c0 = c0;
                pl.cps = ns > 1 ? c1 : c0;
                pl.overlap = overlap;
            }
        }
    }
    return pl;
}

int num_sms()
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

bool scan_tc_supported(const ScanArgs& a)
{
    // a CTA takes two consecutive heads, which must read the same B and C group
    return a.P == kP && a.N == kN && a.chunk % kQ == 0 && a.batch > 0 && a.L > 0 && a.h > 0 && a.G > 0 &&
           (a.G == 1 || a.hpg % 2 == 0) && (int64_t)a.batch * a.L < (1ll << 31);
}

size_t scan_tc_workspace(const ScanArgs& a)
{
    const Plan pl = plan_for(a, num_sms());
    if (pl.nseg == 1) return 256;
    const size_t bh = (size_t)a.batch * a.h;
    return align256(bh * pl.nseg * kP * kN * 4) + align256(bh * pl.nseg * 4);
}

int scan_tc_kernel_count(const ScanArgs& a) { return plan_for(a, num_sms()).nseg > 1 ? 2 : 1; }

static cudaError_t launch_scan_tc_impl(const ScanArgs& a, const ScanGate* gate, void* ws, size_t ws_bytes,
                                       cudaStream_t s);

cudaError_t launch_scan_tc(const ScanArgs& a, void* ws, size_t ws_bytes, cudaStream_t s)
{
    return launch_scan_tc_impl(a, nullptr, ws, ws_bytes, s);
}

cudaError_t launch_scan_tc_gated(const ScanArgs& a, const ScanGate& g, void* ws, size_t ws_bytes, cudaStream_t s)
{
    return launch_scan_tc_impl(a, &g, ws, ws_bytes, s);
}

static cudaError_t launch_scan_tc_impl(const ScanArgs& a, const ScanGate* gate, void* ws, size_t ws_bytes,
                                       cudaStream_t s)
{
    const Plan pl = plan_for(a, num_sms());
    const int64_t rows = (int64_t)a.batch * a.L;
    CUtensorMap mapX, mapB, mapC;
    if (!make_tmap_bf16(&mapX, a.x, (uint64_t)a.h * kP, rows, a.sx * 2, 64, kQ)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&mapB, a.B, (uint64_t)a.G * kN, rows, a.sB * 2, 64, kQ)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&mapC, a.C, (uint64_t)a.G * kN, rows, a.sC * 2, 64, kQ)) return cudaErrorInvalidValue;

    // y leaves through bulk tensor stores when it is 16-byte aligned with 16-byte row pitches
    CUtensorMap mapY;
    std::memset(&mapY, 0, sizeof(mapY));
    const bool y_tma = (reinterpret_cast<uintptr_t>(a.y) & 15u) == 0 && (a.sy * 2) % 16 == 0 &&
                       make_tmap_bf16_3d(&mapY, a.y, (uint64_t)a.h * kP, (uint64_t)a.L, (uint64_t)a.batch,
                                         (uint64_t)a.sy * 2, (uint64_t)a.sy * 2 * a.L, 64, kQ);

    ScanTcParams p{};
    p.L = a.L; p.h = a.h; p.nseg = pl.nseg; p.cps = pl.cps; p.nchunks = pl.nchunks; p.hpg = a.hpg;
    p.c0 = pl.c0;
    p.y_tma = y_tma ? 1 : 0;
    p.dt = a.dt; p.sdt = a.sdt; p.A = a.A; p.D = a.D; p.y = a.y; p.sy = a.sy;
    p.init_state = a.init_state; p.final_state = a.final_state; p.state_stride = a.state_stride;
    p.status = device_status_ptr();
    if (gate) {
        p.z = static_cast<const __nv_bfloat16*>(gate->z);
        p.sz = gate->sz;
        p.norm_w = static_cast<const __nv_bfloat16*>(gate->norm_w);
        p.row_parts = gate->row_parts;
    }
    const size_t bh = (size_t)a.batch * a.h;
    if (pl.nseg > 1) {
        if (!ws || ws_bytes < scan_tc_workspace(a)) return cudaErrorInvalidValue;
        p.states = static_cast<float*>(ws);
        p.seg_decay = reinterpret_cast<float*>(static_cast<char*>(ws) + align256(bh * pl.nseg * kP * kN * 4));
    }
    int dev = 0;
    cudaGetDevice(&dev);
    static unsigned long long attr_set = 0;
    if (dev < 64 && !(attr_set >> dev & 1ull)) {
        cudaError_t e = cudaFuncSetAttribute(ssd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kChunkSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ssd_seg_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSegSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set |= 1ull << dev;
    }
    const dim3 cgrid((a.h + 1) / 2, a.batch, pl.nseg);
    if (pl.nseg == 1) {
        ssd_chunk_kernel<<<cgrid, kChunkThreads, kChunkSmem, s>>>(mapX, mapB, mapC, mapY, p);
        return cudaGetLastError();
    }
    // The chunk scan is launched as a programmatic dependent of the segment-state grid: segment
    // 0's CTAs may run beside it, the others wait for its completion before reading the
    // segment end states.  If y overlaps an input the segment-state grid still reads, every
    // CTA waits.
    {
        auto span = [](const void* q, int64_t bytes) { return std::make_pair((uintptr_t)q, (uintptr_t)q + bytes); };
        const int64_t T = (int64_t)a.batch * a.L;
        const int esz = 2;
        const auto ys = span(a.y, ((T - 1) * a.sy + (int64_t)a.h * kP) * esz);
        const std::pair<uintptr_t, uintptr_t> ins[3] = {span(a.x, ((T - 1) * a.sx + (int64_t)a.h * kP) * esz),
                                                        span(a.B, ((T - 1) * a.sB + (int64_t)a.G * kN) * esz),
                                                        span(a.dt, ((T - 1) * a.sdt + a.h) * 4)};
        p.wait_all = (pl.overlap ? 0 : 1);
        for (const auto& in : ins)
            if (ys.first < in.second && in.first < ys.second) p.wait_all = 1;
    }
    ssd_seg_state_kernel<<<dim3((a.h + 1) / 2, pl.nseg - 1, a.batch), 320, kSegSmemBytes, s>>>(mapX, mapB, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = cgrid;
    cfg.blockDim = dim3(kChunkThreads);
    cfg.dynamicSmemBytes = kChunkSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ssd_chunk_kernel, mapX, mapB, mapC, mapY, p);
}

}  // namespace mm

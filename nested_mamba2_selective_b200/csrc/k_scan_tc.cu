// Chunked selective scan on sm_100a tensor cores (bf16 x, B, C; fp32 dt, A, D
// and fp32 state), for d_head = 64 and d_state = 128.
//
// The scan H_t = exp(dt_t A) H_{t-1} + dt_t B_t x_t^T, y_t = C_t^T H_t + D x_t
// ("MatMamba: A Matryoshka State Space Model", block-definition paragraph:
// "chunk + selective scan", A and D learnable) is evaluated on blocks of
// Q = 128 tokens.  With cs_t the running sum of dt*A inside a block and a the
// value of cs at the block's middle row, the chunk scan's fast blocks use
//   y_t    = 2^(cs_t - a) [ (Gc X~)_t + C_t (2^a H_prev) ] + D x_t
//   H_next = 2^(tot - a) [ 2^a H_prev + B^T X~ ],   X~_s = 2^(a - cs_s) dt_s x_s
// with Gc the causally masked C B^T (log2 units): the decay becomes per-token
// scales of x and per-row scales of y, and one contraction serves both heads of
// a CTA.  Blocks whose decay across half a block exceeds 2^64 use per-head
// masked decay matrices instead (see ssd_chunk_kernel).  Both unroll the
// recurrence exactly.  The sequence is cut into segments of whole blocks so
// that (batch, head pair, segment) CTAs fill the GPU:
//   1. seg_state  : the end state of each sub-segment of every segment but the
//                   last, from a zero start (tcgen05, four heads per CTA)
//   2. chunk_scan : every segment from its true start state (the initial state
//                   carried over the earlier sub-segments' end states at the
//                   CTA's start), carrying the state across blocks in TMEM
//                   (tcgen05).
//                   It is a programmatic dependent of seg_state: segment 0 needs
//                   no carried state and may run beside it.
// Only segment end states touch HBM.
//
// A CTA takes two heads of one (batch, segment) so that the B and C blocks and
// G = C B^T are loaded and computed once per pair; the thread roles of the
// chunk scan are described above ssd_chunk_kernel.
#include <cuda.h>

#include <cmath>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
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

// TMEM columns: G = C B^T, overwritten in place by Gc or M_0 | M_1 (A operands); two output
// accumulators of both heads (Y buffer i at kTY0 + 128 i); the state S of both heads.
constexpr uint32_t kTG = 0, kTY0 = 128, kTS = 384, kTCols = 512;
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
    float* states;     // [b*h][nslot][P*N]: slot j + 1 = end state of sub-segment j from a zero start
    float* seg_decay;  // [b*h][nslot - 1]: log2 of the decay over sub-segment j
    int nsub;          // segment-state sub-segments per segment but the last
    int nslot;         // (nseg - 1) * nsub + 1
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

// Chunk scan.  A CTA takes two heads of one (batch, segment) and walks the segment's 128-token
// blocks in order, carrying the fp32 state of both heads in TMEM.
//
// Fast blocks.  With cs_t the running sum of dt A (log2 units) from the block's start and a the
// anchor cs at the block's middle row (63),
//   y_t    = 2^(cs_t - a) [ sum_{s<=t} G[t,s] X~_s + C_t (2^a H) ] + D x_t,
//   X~_s   = 2^(a - cs_s) dt_s x_s,    G = C B^T,
//   H_next = 2^(tot - a) [ 2^a H + B^T X~ ],
// which unrolls the recurrence exactly.  The causally masked G (Gc) does not depend on the head,
// so one tensor-core contraction [Gc | C] . [X~ ; 2^a H] of K = 256 and N = 128 gives both heads'
// outputs, and the per-head decay reduces to per-token scales of x (X~) and per-row scales of the
// output.  Every exponent stays within the decay across half a block, which fast blocks bound by
// 2^kFastMax (64 in log2 units) for both heads.
// Steep blocks (either half of a head decays faster than that) take the direct form instead:
// per-head masked decay matrices M_j[t,s] = G[t,s] 2^(cs_t - cs_s) dt_s,
//   y_t = M_j x + 2^(cs_t) C_t H + D x_t,   H_next = 2^tot H + B^T X',  X'_s = 2^(tot - cs_s) dt_s x_s,
// with the state term in a second output accumulator.  The builders factor each entry's decay at
// the last row m of its 32-token column block, 2^(cs_t - m) 2^(m - cs_s), so a tile needs one power
// of two per row and per column; only a diagonal tile whose quarter decays by more than 2^64 takes
// one exponential per entry.
//
// 512 threads in roles:
//   warp 0      TMA producer (one lane)
//   warp 1      tcgen05.mma issuer (one lane); the warp owns the TMEM allocation
//   warps 2-7   builders: thread (quarter q = warp % 4, lane) owns TMEM lane and token row
//               r = 32 q + lane, and turns G into Gc (fast) or M_0 | M_1 (steep) in place over
//               some of its row's 32-token column blocks; warps 2 and 3 take the upper column
//               blocks of quarters 2 and 3, and the lower quarters also write the zero blocks
//   warps 8-15  state warps: thread (q, lane, head hf) owns row r of head hf: decay scan and the
//               block's mode, state read-back (bf16 copy of the state for the C.H term, scaled
//               fp32 state back for the state MMA), X~ (in place over x) or X', epilogue
// Per block k the tensor core runs G = C B^T (once block k-1's G columns are consumed), then for
// fast blocks S += B^T X~, Y = C . [2^a H_0 | 2^a H_1] and Y += Gc . [X~_0 | X~_1]; for steep
// blocks Yoff = C . [H_0 | H_1], S += B^T X', Y_j = M_j x_j.  The two output accumulators
// alternate between blocks, so block k-1's epilogue runs under block k's tensor work.
// A stage's B and x regions are free once the block's MMAs are done (a commit), so the next
// block but one starts loading them at once; its C region (where the gated form's z tile then
// lands) holds the block's y tile until the bulk store has read it, and only C waits for that.
// Element-wise products use the paired fp32 instructions (mul/fma .f32x2, rounded per lane
// exactly like their scalar forms).

// Blocks [c_begin, c_end) of segment `seg`.
__device__ __forceinline__ void seg_range(const ScanTcParams& p, int seg, int* c_begin, int* c_end)
{
    *c_begin = seg == 0 ? 0 : p.c0 + (seg - 1) * p.cps;
    *c_end = min(p.nchunks, seg == 0 ? p.c0 : *c_begin + p.cps);
}

// Blocks [c_begin, c_end) of segment-state sub-segment j: part j % nsub of segment j / nsub.
__device__ __forceinline__ void sub_range(const ScanTcParams& p, int j, int* c_begin, int* c_end)
{
    int b0, b1;
    seg_range(p, j / p.nsub, &b0, &b1);
    const int u = j % p.nsub, len = max(b1 - b0, 0);
    *c_begin = b0 + (len * u) / p.nsub;
    *c_end = b0 + (len * (u + 1)) / p.nsub;
}

// Programmatic dependent launch: let the dependent grid start, and wait for the
// prerequisite grid's completion (and its memory) before reading what it wrote.
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

constexpr int kChunkThreads = 512;
constexpr float kFastMax = 64.0f;  // log2 units
// small tables after the H buffer (floats): state-warp scan totals [2 parity][2 heads][4], block
// mode [2 parity], builder tables for steep blocks: cs [2 heads][128], column factors
// 2^(m - cs_s) dt_s [2 heads][128] (m: cs at the last row of the 32-row quarter of s), builder
// scan totals [2 heads][4]
constexpr int kTabPart = 0, kTabMode = 16, kTabCs = 20, kTabV = 276, kTabBPart = 532, kTabFloats = 540;
constexpr int kOffH = kNStage * kStage;  // bf16 state copy of two heads (steep blocks: then X')
constexpr int kOffTab = kOffH + 2 * kTileQP;
constexpr int kOffBar = kOffTab + kTabFloats * 4;
constexpr int kNumBars = 24;
constexpr int kChunkSmem = kOffBar + kNumBars * 8 + 16;
static_assert(kChunkSmem <= 232448, "chunk scan exceeds the 227 KB of shared memory a CTA can have");
static_assert(kOffBar % 8 == 0, "mbarriers need 8-byte alignment");

__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 bf2(uint32_t v) { return make_float2(bf_lo(v), bf_hi(v)); }
__device__ __forceinline__ uint32_t pack2(float2 v) { return pack_bf16(v.x, v.y); }

// Inclusive prefix sum over the 32 lanes of a warp.
__device__ __forceinline__ float warp_incl_scan(float v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Fast-block test of one head from its four 32-row partial sums (log2 units, each <= 0): the
// anchor a (cs at row 63) and the total; exponents of the fast form stay within [-64, 64].
__device__ __forceinline__ bool fast_head(const float* part, float* a_out, float* tot_out)
{
    const float a = part[0] + part[1];
    const float tot = a + part[2] + part[3];
    *a_out = a;
    *tot_out = tot;
    return a - tot <= kFastMax && -a <= kFastMax;
}

template <bool GATED>
__global__ void __launch_bounds__(kChunkThreads, 1)
    ssd_chunk_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapB,
                     const __grid_constant__ CUtensorMap mapC, const __grid_constant__ CUtensorMap mapY,
                     const __grid_constant__ CUtensorMap mapZ, const ScanTcParams p)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    float* tab = reinterpret_cast<float*>(sm + kOffTab);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kOffBar);  // [2] B and x of the stage loaded (TMA)
    uint64_t* full_c = full + 2;                                  // [2] C of the stage loaded (TMA)
    uint64_t* empty = full_c + 2;                                 // [2] B and x free: the block's MMAs done (commit)
    uint64_t* empty_c = empty + 2;                                // [2] C region free: its y tile stored (8 warps)
    uint64_t* g_done = empty_c + 2;                               // G of the block done (commit)
    uint64_t* m_ready = g_done + 1;                               // Gc or M built (6 builder warps)
    uint64_t* mode_rdy = m_ready + 1;                             // [2] block mode written (1 state thread)
    uint64_t* h_ready = mode_rdy + 2;                             // read-back done (8 state warps)
    uint64_t* h_free = h_ready + 1;                               // state MMA and H copy consumed (commit)
    uint64_t* yo_done = h_free + 1;                               // steep blocks: C.H done (commit)
    uint64_t* x_ready = yo_done + 1;                              // [2] X~ or X' written (8 state warps);
                                                                  // a fast block's X~ may come one block early
    uint64_t* y_done = x_ready + 2;                               // [2] every MMA of a block using output
                                                                  // accumulator i done (commit)
    uint64_t* yfree = y_done + 2;                                 // [2] output accumulator read (8 warps)
    uint64_t* zfull = yfree + 2;                                  // [2] gated: z tile in the C region (TMA)
    uint64_t* done = zfull + 2;                                   // drain (commit)
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
            mbar_init(&full_c[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&empty_c[s], 8);
            mbar_init(&yfree[s], 8);
            mbar_init(&y_done[s], 1);
            mbar_init(&zfull[s], 1);
        }
        mbar_init(g_done, 1);
        mbar_init(m_ready, 6);
        mbar_init(&mode_rdy[0], 1);
        mbar_init(&mode_rdy[1], 1);
        mbar_init(h_ready, 8);
        mbar_init(h_free, 1);
        mbar_init(yo_done, 1);
        mbar_init(&x_ready[0], 8);
        mbar_init(&x_ready[1], 8);
        mbar_init(done, 1);
        *abort = (smem_u32(sm) & 1023u) ? 1 : 0;  // tiles need 1024-byte alignment; never fault on it
        if (*abort) raise_timeout(abort, p.status);
        fence_mbar_init();
        prefetch_tmap(&mapX);
        prefetch_tmap(&mapB);
        prefetch_tmap(&mapC);
        if (p.y_tma) prefetch_tmap(&mapY);
        if (GATED) prefetch_tmap(&mapZ);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint8_t* sH = sm + kOffH;
    // a following programmatic dependent (the output projection) may start its set-up once every CTA
    // of this grid has started; it reads nothing of ours before this grid has completed
    grid_launch_dependents();

    if (warp == 0) {
        if (lane == 0 && !*abort) {  // ------------------------------------------------ TMA producer
            // gated: block j's z tile goes into its stage's C region once the C.H MMA has read C
            int zk = 0;  // z tiles issued
            auto load_z = [&](int j) -> bool {
                if (!mbar_wait(h_free, j & 1, abort)) return false;
                const int sj = j % kNStage;
                const int zrow = (int)(tok0 + (int64_t)(c_begin + j) * kQ);
                uint8_t* zb = sm + sj * kStage + kOffC;
                mbar_arrive_expect_tx(&zfull[sj], 2 * kTileQP);
                tma_load_2d(zb, &mapZ, &zfull[sj], head0 * kP, zrow);
                tma_load_2d(zb + kTileQP, &mapZ, &zfull[sj], min(head0 + 1, p.h - 1) * kP, zrow);
                ++zk;
                return true;
            };
            int k = 0, kbx = 0, kc = 0;  // blocks whose B and x / C loads are issued
            for (; k < nch; ++k) {
                const int s = k % kNStage;
                // block k goes into the stage block k-2 used: B and x once that block's MMAs are
                // done, C once its y tile (staged in the C region) has been stored
                if (k >= kNStage && !mbar_wait(&empty[s], ((k / kNStage) - 1) & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                const int row = (int)(tok0 + (int64_t)(c_begin + k) * kQ);
                uint8_t* base = sm + s * kStage;
                mbar_arrive_expect_tx(&full[s], kStage - kOffB);
                tma_load_2d(base + kOffB, &mapB, &full[s], grp * kN, row);
                tma_load_2d(base + kOffB + kTileQN / 2, &mapB, &full[s], grp * kN + 64, row);
                tma_load_2d(base + kOffX, &mapX, &full[s], head0 * kP, row);
                // a pair's second head past the last head reloads the last head (its dt is zero)
                tma_load_2d(base + kOffX + kTileQP, &mapX, &full[s], min(head0 + 1, p.h - 1) * kP, row);
                kbx = k + 1;
                if (k >= kNStage && !mbar_wait(&empty_c[s], ((k / kNStage) - 1) & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                mbar_arrive_expect_tx(&full_c[s], kTileQN);
                tma_load_2d(base + kOffC, &mapC, &full_c[s], grp * kN, row);
                tma_load_2d(base + kOffC + kTileQN / 2, &mapC, &full_c[s], grp * kN + 64, row);
                kc = k + 1;
                if (GATED && k > 0 && !load_z(k - 1)) {  // block k-1's z, once its C.H MMA is done
                    raise_timeout(abort, p.status);
                    break;
                }
            }
            if (GATED && k == nch && nch > 0 && !load_z(nch - 1)) raise_timeout(abort, p.status);
            // every issued load lands before the CTA can exit (bounded; only the last two can be pending)
            for (int j = max(0, kbx - kNStage); j < kbx; ++j) mbar_wait(&full[j % kNStage], (j / kNStage) & 1, nullptr);
            for (int j = max(0, kc - kNStage); j < kc; ++j) mbar_wait(&full_c[j % kNStage], (j / kNStage) & 1, nullptr);
            for (int j = max(0, zk - kNStage); j < zk; ++j) mbar_wait(&zfull[j % kNStage], (j / kNStage) & 1, nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0 && !*abort) {  // -------------------------------------------------- tcgen05.mma
            const uint32_t id_g = idesc_bf16(128, 128, 0, 0);   // C (K-major) x B (K-major)
            const uint32_t id_o = idesc_bf16(128, 128, 0, 1);   // C (K-major) x [H_0 | H_1] (MN-major)
            const uint32_t id_s = idesc_bf16(128, 128, 1, 1);   // B^T (MN-major) x [X_0 | X_1] (MN-major)
            const uint32_t id_y = idesc_bf16(128, 64, 0, 1);    // M_j (TMEM) x x_j (MN-major)
            const uint32_t aH = smem_u32(sH);
            uint32_t nuse[2] = {0u, 0u};  // uses of each output accumulator so far
            auto acc_free = [&](int i) -> bool {  // earlier use of accumulator i read by its epilogue
                if (nuse[i] > 0 && !mbar_wait(&yfree[i], (nuse[i] - 1) & 1, abort)) return false;
                ++nuse[i];
                return true;
            };
            bool ok = true;
            for (int k = 0; ok && k < nch; ++k) {
                const int s = k % kNStage, yi = k & 1;
                // stage k is loaded, and block k-1's output MMAs (the last readers of the G columns) are done
                if (!mbar_wait(&full[s], (k / kNStage) & 1, abort) || !mbar_wait(&full_c[s], (k / kNStage) & 1, abort) ||
                    (k > 0 && !mbar_wait(&y_done[(k - 1) & 1], ((k - 1) >> 1) & 1, abort))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t aS = smem_u32(sm + s * kStage);
                const uint32_t aC = aS + kOffC, aB = aS + kOffB, aX = aS + kOffX;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // G = C . B^T over the state dim
                    const uint32_t off = (kk & 3) * 32 + (kk >> 2) * (kTileQN / 2);
                    mma_ss(tmem + kTG, desc_sw128(aC + off, 16, 1024), desc_sw128(aB + off, 16, 1024), id_g, kk > 0);
                }
                mma_commit(g_done);
                if (!mbar_wait(h_ready, k & 1, abort)) {  // read-back done; the block's mode is written
                    ok = false;
                    break;
                }
                tc_fence_after();
                const bool fast = tab[kTabMode + (k & 1)] != 0.0f;
                const uint32_t yacc = tmem + kTY0 + 128 * yi;
                if (fast) {
                    if (!mbar_wait(&x_ready[k & 1], (k >> 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // S += B^T . [X~_0 | X~_1] over the block's tokens
                        mma_ss(tmem + kTS, desc_sw128(aB + kk * 2048, kTileQN / 2, 1024),
                               desc_sw128(aX + kk * 2048, kTileQP, 1024), id_s, 1u);
                    if (!acc_free(yi)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {  // Y (+)= C . [2^a H_0 | 2^a H_1] over the state dim
                        const uint32_t off = (kk & 3) * 32 + (kk >> 2) * (kTileQN / 2);
                        mma_ss(yacc, desc_sw128(aC + off, 16, 1024), desc_sw128(aH + kk * 2048, kTileQP, 1024), id_o,
                               1u);
                    }
                    mma_commit(h_free);
                    if (!mbar_wait(m_ready, k & 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // Y += Gc . [X~_0 | X~_1] over the block's tokens
                        mma_ts(yacc, tmem + kTG + 32 * (kk >> 1) + 8 * (kk & 1),
                               desc_sw128(aX + kk * 2048, kTileQP, 1024), id_o, 1u);
                    mma_commit(&y_done[yi]);
                    mma_commit(&empty[s]);  // B and x of the stage are read
                } else {
                    const uint32_t oacc = tmem + kTY0 + 128 * (yi ^ 1);
                    if (!acc_free(yi ^ 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {  // Yoff = C . [H_0 | H_1] over the state dim
                        const uint32_t off = (kk & 3) * 32 + (kk >> 2) * (kTileQN / 2);
                        mma_ss(oacc, desc_sw128(aC + off, 16, 1024), desc_sw128(aH + kk * 2048, kTileQP, 1024), id_o,
                               kk > 0);
                    }
                    mma_commit(yo_done);
                    if (!mbar_wait(&x_ready[k & 1], (k >> 1) & 1, abort)) {  // X' written over the state copy
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // S += B^T . [X'_0 | X'_1] over the block's tokens
                        mma_ss(tmem + kTS, desc_sw128(aB + kk * 2048, kTileQN / 2, 1024),
                               desc_sw128(aH + kk * 2048, kTileQP, 1024), id_s, 1u);
                    mma_commit(h_free);
                    if (!mbar_wait(m_ready, k & 1, abort) || !acc_free(yi)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)  // Y_j (+)= M_j . x_j over the block's tokens
                            mma_ts(yacc + 64 * j, tmem + kTG + 32 * (kk >> 1) + 16 * j + 8 * (kk & 1),
                                   desc_sw128(aX + j * kTileQP + kk * 2048, kTileQP, 1024), id_y, 1u);
                    mma_commit(&y_done[yi]);
                    mma_commit(&empty[s]);  // B and x of the stage are read
                }
            }
            if (!ok) raise_timeout(abort, p.status);
            mma_commit(done);
            mbar_wait(done, 0, nullptr);  // every issued MMA is done before TMEM can be released (bounded)
        }
    } else if (warp < 8) {  // ------------------------------------------------------------- builders
        const int q = warp & 3, r = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const bool upper = warp < 4;  // warps 2, 3: the upper column blocks of quarters 2 and 3
        const int cb_lo = upper ? 2 : 0;
        const int cb_hi = upper ? q : min(q, 1);  // inclusive
        const bool zero_writer = upper ? q == 2 : q <= 1;
        float A2[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) A2[j] = head0 + j < p.h ? p.A[head0 + j] * kLog2e : 0.0f;
        for (int k = 0; k < nch; ++k) {  // every warp runs every iteration (named barrier 4)
            const bool okm = __all_sync(0xffffffffu, mbar_wait(&mode_rdy[k & 1], (k >> 1) & 1, abort));
            const bool fast = !okm || tab[kTabMode + (k & 1)] != 0.0f;
            // steep blocks: every builder thread loads dt of its row for both heads; warps 4-7 (one
            // row each) scan dt A into cs through the per-quarter totals and publish cs and the
            // column factors V_s = 2^(m - cs_s) dt_s, m = cs at the last row of the quarter of s
            float c2[2] = {0.0f, 0.0f}, dv[2] = {0.0f, 0.0f};
            if (!fast) {
                const int t = (c_begin + k) * kQ + r;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    dv[j] = (t < p.L && head0 + j < p.h) ? p.dt[(tok0 + t) * p.sdt + head0 + j] : 0.0f;
                    if (!upper) {
                        c2[j] = warp_incl_scan(dv[j] * A2[j], lane);
                        if (lane == 31) tab[kTabBPart + 4 * j + q] = c2[j];
                    }
                }
            }
            asm volatile("bar.sync 4, 192;" ::: "memory");
            // the diagonal tile may use the factored form when its quarter spans at most 2^64 (read
            // here: the next block's totals overwrite the table before its first barrier)
            bool diag_split[2] = {true, true};
#pragma unroll
            for (int j = 0; j < 2; ++j) diag_split[j] = fast || -tab[kTabBPart + 4 * j + q] <= kFastMax;
            if (!fast && !upper) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float pre = 0.0f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) pre += i < q ? tab[kTabBPart + 4 * j + i] : 0.0f;
                    const float cs = c2[j] + pre;
                    const float m = __shfl_sync(0xffffffffu, cs, 31);
                    tab[kTabCs + 128 * j + r] = cs;
                    tab[kTabV + 128 * j + r] = ex2(m - cs) * dv[j];
                }
            }
            asm volatile("bar.sync 4, 192;" ::: "memory");

            const bool ok = okm && __all_sync(0xffffffffu, mbar_wait(g_done, k & 1, abort));
            if (ok) {
                tc_fence_after();
                if (zero_writer) {  // above the diagonal: zeros (both heads' columns in steep blocks)
                    uint32_t z[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) z[e] = 0u;
#pragma unroll
                    for (int cb = 1; cb < 4; ++cb)
                        if (cb > q) tmem_st32(tmem + lane_base + kTG + 32 * cb, z);
                }
                float ct[2] = {0.0f, 0.0f};
                if (!fast) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) ct[j] = tab[kTabCs + 128 * j + r];
                }
#pragma unroll 1
                for (int cb = cb_lo; cb <= cb_hi; ++cb) {  // column block s in [32 cb, 32 cb + 32)
                    uint32_t gv[32];
                    tmem_ld32(tmem + lane_base + kTG + 32 * cb, gv);
                    tmem_ld_wait();
                    const bool diag = cb == q;
                    if (fast) {  // Gc: G with the causal mask s <= t, as bf16 pairs
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float g0 = __uint_as_float(gv[e]), g1 = __uint_as_float(gv[e + 1]);
                            if (diag) {
                                g0 = e <= lane ? g0 : 0.0f;
                                g1 = e + 1 <= lane ? g1 : 0.0f;
                            }
                            pk[e >> 1] = pack_bf16(g0, g1);
                        }
                        tmem_st16(tmem + lane_base + kTG + 32 * cb, pk);
                    } else {  // M_j = G 2^(cs_t - cs_s) dt_s for s <= t, one head after the other
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            uint32_t pk[16];
                            if (!diag || diag_split[j]) {
                                // 2^(cs_t - cs_s) = 2^(cs_t - m) 2^(m - cs_s), m = cs at the last row of
                                // the column block: below the diagonal both factors are <= 1 (a factor
                                // that underflows belongs to an entry below 2^-126); on it the quarter
                                // spans at most 2^64, so neither overflows
                                const float u = ex2(ct[j] - tab[kTabCs + 128 * j + 32 * cb + 31]);
                                const float2 u2 = make_float2(u, u);
                                const float2* v2 = reinterpret_cast<const float2*>(tab + kTabV + 128 * j + 32 * cb);
#pragma unroll
                                for (int e = 0; e < 32; e += 2) {
                                    float2 mv = mul2(mul2(make_float2(__uint_as_float(gv[e]), __uint_as_float(gv[e + 1])),
                                                          v2[e >> 1]), u2);
                                    if (diag) {
                                        mv.x = e <= lane ? mv.x : 0.0f;
                                        mv.y = e + 1 <= lane ? mv.y : 0.0f;
                                    }
                                    pk[e >> 1] = pack2(mv);
                                }
                            } else {  // a diagonal quarter spanning more than 2^64: one exponent per entry,
                                      // cs_s and dt_s from the lane that owns row s
                                const float cs_own = ct[j];
#pragma unroll
                                for (int e = 0; e < 32; e += 2) {
                                    const float cs0 = __shfl_sync(0xffffffffu, cs_own, e);
                                    const float cs1 = __shfl_sync(0xffffffffu, cs_own, e + 1);
                                    const float d0 = __shfl_sync(0xffffffffu, dv[j], e);
                                    const float d1 = __shfl_sync(0xffffffffu, dv[j], e + 1);
                                    float m0 = __uint_as_float(gv[e]) * ex2(fminf(cs_own - cs0, 0.0f)) * d0;
                                    float m1 = __uint_as_float(gv[e + 1]) * ex2(fminf(cs_own - cs1, 0.0f)) * d1;
                                    m0 = e <= lane ? m0 : 0.0f;
                                    m1 = e + 1 <= lane ? m1 : 0.0f;
                                    pk[e >> 1] = pack_bf16(m0, m1);
                                }
                            }
                            tmem_st16(tmem + lane_base + kTG + 32 * cb + 16 * j, pk);
                        }
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(m_ready);
            } else {
                raise_timeout(abort, p.status);
            }
        }
    } else {  // --------------------------------------------------------------------- state warps
        const int cw = warp - 8, q = warp & 3, hf = cw >> 2;
        const int r = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int head = head0 + hf;
        const bool head_ok = head < p.h;
        const float A2 = head_ok ? p.A[head] * kLog2e : 0.0f;
        const float Dh = (p.D && head_ok) ? p.D[head] : 0.0f;
        const int64_t bh = (int64_t)b * p.h + head;
        const int PN = kP * kN;
        uint8_t* myH = sH + hf * kTileQP;
        const uint32_t sacc = tmem + lane_base + kTS + 64 * hf;  // this head's state, row n = r

        // A segment's start state is the initial state (or zero) carried over the earlier
        // segments: H <- 2^decay_j H + S_j, S_j being segment j's end state from a zero start.
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
                for (int sj = 0; head_ok && sj < seg * p.nsub; ++sj) {
                    const float dec = exp2f(p.seg_decay[bh * (p.nslot - 1) + sj]);
                    const float* sp = p.states + (bh * p.nslot + sj + 1) * PN;
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = fmaf(dec, v[j], sp[(32 * h2 + j) * kN + r]);
                }
                uint32_t u[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(v[j]);
                tmem_st32(sacc + 32 * h2, u);
            }
            tmem_st_wait();
        }
        float dt_next = 0.0f;
        if (head_ok && nch > 0 && c_begin * kQ + r < p.L) dt_next = p.dt[(tok0 + c_begin * kQ + r) * p.sdt + head];
        // the previous block: cs and anchor of this row (log2 units), and its mode
        float c2_prev = 0.0f, a_prev = 0.0f;
        bool fast_prev = true;
        float s_in = 1.0f;  // TMEM state x s_in = the state at the current block's start
        int nsteep = 0;     // steep blocks so far (phases of yo_done)
        bool ok = __all_sync(0xffffffffu, !*abort);

        // Epilogue of block kp: y from the output accumulator(s), which already hold the D x term, and
        // the optional gate (z from the tile the producer loaded into the stage's C region).  y rows go
        // into the stage's C region (over z: each thread reads its row's z chunk before writing the
        // y chunk there) in the 128-byte swizzle and leave as one bulk tensor store per head (rows
        // past L clipped); the C region is released once the store has read them.  Every warp of the
        // head calls it once per block (named barrier 2 + hf).
        auto epilogue = [&](int kp) {
            const int sp = kp & 1;
            const int tp0 = (c_begin + kp) * kQ;
            const bool valid = head_ok && tp0 + r < p.L;
            const int64_t tok = tok0 + tp0 + r;
            const int col = head * kP;
            const uint32_t yacc = tmem + lane_base + kTY0 + 128 * sp + 64 * hf;
            const uint32_t oacc = tmem + lane_base + kTY0 + 128 * (sp ^ 1) + 64 * hf;
            uint8_t* sX = sm + sp * kStage + kOffC + hf * kTileQP;        // y rows (over C, or z)
            const uint8_t* sZ = sm + sp * kStage + kOffC + hf * kTileQP;  // z rows (gated)
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&y_done[sp], (kp >> 1) & 1, abort));
            if (GATED && ok) ok = __all_sync(0xffffffffu, mbar_wait(&zfull[sp], (kp >> 1) & 1, abort));
            if (ok) {
                tc_fence_after();
                // fast: y = 2^(cs - a) Y;  steep: y = Y + 2^cs Yoff
                const float sy = fast_prev ? ex2(c2_prev - a_prev) : 1.0f;
                const float so = fast_prev ? 0.0f : ex2(c2_prev);
                const float2 sy2 = make_float2(sy, sy), so2 = make_float2(so, so);
                uint4* yrow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.y) + tok * p.sy + col);
                float ssq[2] = {0.0f, 0.0f};
                // 16 output columns from yv (and ov): 16-byte chunks cc and cc + 1 of the row
                auto out16 = [&](int cc, const uint32_t* yv, const uint32_t* ov) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint4 zq = make_uint4(0, 0, 0, 0), nw4 = make_uint4(0, 0, 0, 0);
                        if (GATED) {
                            zq = *reinterpret_cast<const uint4*>(sZ + sw128(r, cc + c));
                            nw4 = *reinterpret_cast<const uint4*>(p.norm_w + col + 8 * (cc + c));
                        }
                        const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
                        const uint32_t nw[4] = {nw4.x, nw4.y, nw4.z, nw4.w};
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = 8 * c + 2 * e;
                            float2 v = mul2(sy2, make_float2(__uint_as_float(yv[j]), __uint_as_float(yv[j + 1])));
                            if (ov) v = fma2(so2, make_float2(__uint_as_float(ov[j]), __uint_as_float(ov[j + 1])), v);
                            if (GATED) {
                                v = mul2(v, make_float2(silu_approx(bf_lo(zw[e])), silu_approx(bf_hi(zw[e]))));
                                ssq[cc >> 2] = fmaf(v.x, v.x, fmaf(v.y, v.y, ssq[cc >> 2]));
                                v = mul2(v, bf2(nw[e]));
                            }
                            o[e] = pack2(v);
                        }
                        const uint4 ow = make_uint4(o[0], o[1], o[2], o[3]);
                        if (p.y_tma) *reinterpret_cast<uint4*>(sX + sw128(r, cc + c)) = ow;
                        else if (valid) yrow[cc + c] = ow;
                    }
                };
                auto release = [&]() {  // the accumulators of block kp are read: the MMA lane may reuse them
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&yfree[sp]);
                        if (!fast_prev) mbar_arrive(&yfree[sp ^ 1]);
                    }
                };
                if (fast_prev) {  // 32 columns per TMEM round trip
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t yv[32];
                        tmem_ld32(yacc + 32 * h, yv);
                        tmem_ld_wait();
                        if (h == 1) release();
                        out16(4 * h, yv, nullptr);
                        out16(4 * h + 2, yv + 16, nullptr);
                    }
                } else {  // steep: Y and Yoff, 16 columns of each per round trip
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        uint32_t yv[16], ov[16];
                        tmem_ld16(yacc + 16 * h, yv);
                        tmem_ld16(oacc + 16 * h, ov);
                        tmem_ld_wait();
                        if (h == 3) release();
                        out16(2 * h, yv, ov);
                    }
                }
                if (GATED && valid) {
                    p.row_parts[tok * 2 * p.h + 2 * head] = ssq[0];
                    p.row_parts[tok * 2 * p.h + 2 * head + 1] = ssq[1];
                }
            }
            if (p.y_tma) {  // the head's 128 x 64 tile leaves in one bulk store
                fence_async_smem();
                asm volatile("bar.sync %0, 128;" ::"r"(2 + hf) : "memory");
                if (q == 0) {
                    ok = __all_sync(0xffffffffu, ok && !*abort);
                    if (ok && head_ok && lane == 0) {
                        tma_store_3d(&mapY, sX, head * kP, tp0, b);
                        bulk_commit();
                    }
                    __syncwarp();
                }
            }
            if (ok) {  // the C region of stage sp is free once its y tile has been read
                if (lane == 0) {
                    if (p.y_tma && q == 0) bulk_wait_read0();
                    mbar_arrive(&empty_c[sp]);
                }
                __syncwarp();
            }
        };

        // X~ (fast blocks, in place over x) or X' (steep blocks, over the state copy once the C.H
        // MMA has read it) of block k for the state and output MMAs, and the D x term written into
        // this head's columns of block k's output accumulator, which the output MMAs then add to
        // (fast blocks: 2^(a - cs) D x, in the accumulator's scale; steep blocks: D x)
        auto form_x = [&](int k, bool fast, float c2, float a, float tot, float dtv) {
            const int s = k % kNStage;
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (k / kNStage) & 1, abort));
            if (!ok) return;
            uint8_t* sXk = sm + s * kStage + kOffX + hf * kTileQP;
            uint8_t* dst = sXk;
            float wgt, dsc;
            if (fast) {  // X~[s=r, :] = 2^(a - cs_r) dt_r x[r, :]
                const float e = ex2(a - c2);
                wgt = e * dtv;
                dsc = e * Dh;
            } else {  // X'[s=r, :] = 2^(tot - cs_r) dt_r x[r, :]
                ok = __all_sync(0xffffffffu, mbar_wait(yo_done, nsteep & 1, abort));
                ++nsteep;
                if (!ok) return;
                wgt = ex2(tot - c2) * dtv;
                dsc = Dh;
                dst = myH;
            }
            const float2 w2 = make_float2(wgt, wgt), d2 = make_float2(dsc, dsc);
            const uint32_t dacc = tmem + lane_base + kTY0 + 128 * (k & 1) + 64 * hf;
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // 32 columns at a time
                uint32_t dv[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int cc = 4 * h + c;
                    const uint4 xv = *reinterpret_cast<const uint4*>(sXk + sw128(r, cc));
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 xf = bf2(xw[e]);
                        o[e] = pack2(mul2(xf, w2));
                        const float2 dd = mul2(xf, d2);
                        dv[8 * c + 2 * e] = __float_as_uint(dd.x);
                        dv[8 * c + 2 * e + 1] = __float_as_uint(dd.y);
                    }
                    *reinterpret_cast<uint4*>(dst + sw128(r, cc)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
                tmem_st32(dacc + 32 * h, dv);
            }
            tmem_st_wait();
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&x_ready[k & 1]);
        };

        // Iteration k: decay scan and mode of block k; after a fast block, a fast block k then forms
        // X~, reads the state back and runs block k-1's epilogue, in the order their inputs arrive;
        // otherwise the read-back, block k-1's epilogue (a steep block also uses the other output
        // accumulator), then X~ or X' of block k.  Every warp runs every iteration (named barriers
        // 1 and 2 + hf); a failed wait skips work only.
        for (int k = 0; k <= nch; ++k) {
            float dtv = 0.0f, c2 = 0.0f, a = 0.0f, tot = 0.0f;
            bool fast = true;
            if (k < nch) {
                dtv = dt_next;
                const int t1 = (c_begin + k + 1) * kQ + r;
                dt_next = (head_ok && k + 1 < nch && t1 < p.L) ? p.dt[(tok0 + t1) * p.sdt + head] : 0.0f;
                const float sc = warp_incl_scan(dtv * A2, lane);
                float* part = tab + kTabPart + 8 * (k & 1);
                if (lane == 31) part[4 * hf + q] = sc;
                asm volatile("bar.sync 1, 256;" ::: "memory");
                float pre = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) pre += i < q ? part[4 * hf + i] : 0.0f;
                c2 = sc + pre;
                float a0, t0, a1, t1s;
                const bool f0 = fast_head(part, &a0, &t0);
                const bool f1 = fast_head(part + 4, &a1, &t1s);
                fast = f0 && f1;
                a = hf ? a1 : a0;
                tot = hf ? t1s : t0;
                if (threadIdx.x == 8 * 32) {  // one thread publishes the mode to the builders and the MMA lane
                    tab[kTabMode + (k & 1)] = fast ? 1.0f : 0.0f;
                    mbar_arrive(&mode_rdy[k & 1]);
                }
                // a fast block after a fast block forms X~ before the read-back: it needs only its
                // stage's x and the output accumulator whose epilogue (block k-2) this loop has run,
                // so the state MMA may start as soon as the read-back is done
                if (fast && fast_prev) form_x(k, fast, c2, a, tot, dtv);

                // ---- read-back: the state at the block's start, as bf16 for the C.H term and back
                // into TMEM for the state MMA (fast: both scaled by 2^a; steep: 1 and 2^tot)
                if (ok && k > 0) ok = __all_sync(0xffffffffu, mbar_wait(h_free, (k - 1) & 1, abort));
                if (ok) {
                    tc_fence_after();
                    const float beta = fast ? ex2(a) : 1.0f;
                    const float sb = s_in * beta, sg = s_in * (fast ? beta : ex2(tot));
                    const float2 sb2 = make_float2(sb, sb), sg2 = make_float2(sg, sg);
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {  // 32 state columns per TMEM round trip
                        uint32_t v[32];
                        tmem_ld32(sacc + 32 * h2, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint4 w;
                            w.x = pack2(mul2(sb2, make_float2(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1]))));
                            w.y = pack2(mul2(sb2, make_float2(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3]))));
                            w.z = pack2(mul2(sb2, make_float2(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5]))));
                            w.w = pack2(mul2(sb2, make_float2(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]))));
                            *reinterpret_cast<uint4*>(myH + sw128(r, 4 * h2 + c)) = w;
                        }
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float2 d = mul2(sg2, make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])));
                            v[j] = __float_as_uint(d.x);
                            v[j + 1] = __float_as_uint(d.y);
                        }
                        tmem_st32(sacc + 32 * h2, v);
                    }
                    tmem_st_wait();
                    fence_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(h_ready);
                }
            }
            // otherwise block k-1's epilogue comes first (a steep block uses both output accumulators,
            // and a steep block's X' goes over the state copy once the C.H MMA has read it)
            if (k < nch && fast && fast_prev) {
                if (k > 0) epilogue(k - 1);
            } else {
                if (k > 0) epilogue(k - 1);
                if (k < nch) form_x(k, fast, c2, a, tot, dtv);
            }
            if (!ok) raise_timeout(abort, p.status);
            if (k == nch) break;
            c2_prev = c2;
            a_prev = a;
            fast_prev = fast;
            s_in = fast ? ex2(tot - a) : 1.0f;  // state MMA result -> state at the next block's start
        }

        if (p.y_tma && q == 0 && lane == 0) bulk_wait0();  // this head's y tiles are in global memory
        if (seg == p.nseg - 1 && p.final_state) {  // state after the last block (its MMAs are done)
            ok = __all_sync(0xffffffffu, ok && !*abort);
            if (ok) {
                tc_fence_after();
                float* dst = p.final_state + (int64_t)b * p.state_stride + (int64_t)head * PN;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t v[32];
                    tmem_ld32(sacc + 32 * h2, v);
                    tmem_ld_wait();
                    if (head_ok) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) dst[(32 * h2 + j) * kN + r] = s_in * __uint_as_float(v[j]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTCols);
}

// Segment end states from a zero start, for every segment but the last:
//   S_seg = sum_s 2^(cs_end - cs_s) dt_s B_s x_s^T        (cs in log2 units, over the segment)
// The segment's blocks are visited last to first.  With D the decay of the
// blocks already visited (those after the current one), token s of the block
// gets the weight 2^(D + tot - cs_s) <= 1, and every block's B^T X'' is
// accumulated into one TMEM accumulator: no per-block state update.  X'' is
// formed in place over x in the stage, which the MMA's commit then frees.
// A CTA takes HC heads of one group (4 when the group allows: one MMA of N = 256
// then serves four heads and reads B^T once for all four); S of head j sits
// in TMEM columns [64 j, 64 j + 64), row n = state dim.
template <int HC>
struct SegCfg {
    static constexpr int kStageBytes = kTileQN + HC * kTileQP;  // B | x of HC heads
    static constexpr int kOffSmall = kNStage * kStageBytes;
    static constexpr int kSmem = kOffSmall + 4 * HC * 4 + 8 * 8 + 16;
    static constexpr int kThreads = 64 + 128 * HC;
};
static_assert(SegCfg<4>::kSmem <= 232448, "segment-state kernel exceeds 227 KB of shared memory");

template <int HC>
__global__ void __launch_bounds__(SegCfg<HC>::kThreads, 1)
    ssd_seg_state_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapB,
                         const ScanTcParams p)
{
    using Cfg = SegCfg<HC>;
    extern __shared__ __align__(1024) uint8_t sm[];
    float* wtot = reinterpret_cast<float*>(sm + Cfg::kOffSmall);  // [HC heads][4]
    uint64_t* full = reinterpret_cast<uint64_t*>(wtot + 4 * HC);
    uint64_t* empty = full + kNStage;  // stage read by the MMA (commit)
    uint64_t* xr = empty + kNStage;    // X'' of the stage written (compute warps)
    uint64_t* done = xr + kNStage;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int grpc = blockIdx.x, sub = blockIdx.y, b = blockIdx.z;
    const int head0 = HC * grpc;
    int c_begin, c_end;
    sub_range(p, sub, &c_begin, &c_end);
    const int nch = max(c_end - c_begin, 0);
    const int grp = head0 / p.hpg;  // all HC heads read one group
    const int64_t tok0 = (int64_t)b * p.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_launch_dependents();  // the chunk scan may start its first segment beside this grid

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNStage; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
            mbar_init(&xr[i], 4 * HC);
        }
        mbar_init(done, 1);
        *abort = (smem_u32(sm) & 1023u) ? 1 : 0;
        if (*abort) raise_timeout(abort, p.status);
        fence_mbar_init();
        prefetch_tmap(&mapX);
        prefetch_tmap(&mapB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 64 * HC);
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
                if (k >= kNStage && !mbar_wait(&empty[s], ((k / kNStage) - 1) & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                const int row = (int)(tok0 + (int64_t)(c_end - 1 - k) * kQ);
                uint8_t* base = sm + s * Cfg::kStageBytes;
                mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
                tma_load_2d(base, &mapB, &full[s], grp * kN, row);
                tma_load_2d(base + kTileQN / 2, &mapB, &full[s], grp * kN + 64, row);
#pragma unroll
                for (int j = 0; j < HC; ++j)  // heads past the last one reload it (their dt is zero)
                    tma_load_2d(base + kTileQN + j * kTileQP, &mapX, &full[s], min(head0 + j, p.h - 1) * kP, row);
            }
            for (int j = max(0, k - kNStage); j < k; ++j) mbar_wait(&full[j % kNStage], (j / kNStage) & 1, nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0 && !*abort) {  // MMA issuer: S += B^T [X''_0 | ... | X''_(HC-1)]
            const uint32_t id_s = idesc_bf16(128, 64 * HC, 1, 1);
            for (int k = 0; k < nch; ++k) {
                const int s = k % kNStage;
                if (!mbar_wait(&full[s], (k / kNStage) & 1, abort) || !mbar_wait(&xr[s], (k / kNStage) & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t aB = smem_u32(sm + s * Cfg::kStageBytes);
                const uint32_t aXP = aB + kTileQN;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmem, desc_sw128(aB + kk * 2048, kTileQN / 2, 1024), desc_sw128(aXP + kk * 2048, kTileQP, 1024),
                           id_s, (k | kk) != 0);
                mma_commit(&empty[s]);
            }
            mma_commit(done);
            mbar_wait(done, 0, nullptr);  // every issued MMA is done before TMEM can be released (bounded)
        }
    } else {  // compute warps: thread (quarter q, lane) = token / state row r, head hf of the group
        const int cw = warp - 2, q = warp & 3, hf = cw >> 2;
        const int r = q * 32 + lane;
        const int head = head0 + hf;
        const bool head_ok = head < p.h;
        const float A2 = head_ok ? p.A[head] * kLog2e : 0.0f;
        const uint32_t bar_cnt = 128 * HC;
        float D2 = 0.0f;
        float dt_next = 0.0f;
        if (head_ok && nch > 0) {
            const int t0 = (c_end - 1) * kQ;
            if (t0 + r < p.L) dt_next = p.dt[(tok0 + t0 + r) * p.sdt + head];
        }
        bool ok = true;
        for (int k = 0; k < nch; ++k) {  // every warp runs every iteration (named barrier 1)
            const int s = k % kNStage;
            const int t0 = (c_end - 1 - k) * kQ;
            const float dtv = dt_next;
            if (k + 1 < nch) {
                const int t1 = t0 - kQ;
                dt_next = (head_ok && t1 + r < p.L) ? p.dt[(tok0 + t1 + r) * p.sdt + head] : 0.0f;
            }
            const float sc = warp_incl_scan(dtv * A2, lane);
            float* wt = wtot + 4 * hf;
            if (lane == 31) wt[q] = sc;
            asm volatile("bar.sync 1, %0;" ::"r"(bar_cnt) : "memory");
            float pre = 0.0f, tot = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float w = wt[j];
                pre += j < q ? w : 0.0f;
                tot += w;
            }
            asm volatile("bar.sync 1, %0;" ::"r"(bar_cnt) : "memory");
            const float c2 = sc + pre;
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (k / kNStage) & 1, abort));
            if (ok) {  // X''[r, :] = 2^(D + tot - cs_r) dt_r x[r, :], in place
                const float wgt = ex2(D2 + tot - c2) * dtv;
                const float2 w2 = make_float2(wgt, wgt);
                uint8_t* sX = sm + s * Cfg::kStageBytes + kTileQN + hf * kTileQP;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 xv = *reinterpret_cast<const uint4*>(sX + sw128(r, c));
                    uint4 o;
                    o.x = pack2(mul2(bf2(xv.x), w2));
                    o.y = pack2(mul2(bf2(xv.y), w2));
                    o.z = pack2(mul2(bf2(xv.z), w2));
                    o.w = pack2(mul2(bf2(xv.w), w2));
                    *reinterpret_cast<uint4*>(sX + sw128(r, c)) = o;
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xr[s]);
            } else {
                raise_timeout(abort, p.status);
            }
            D2 += tot;
        }
        ok = __all_sync(0xffffffffu, ok && mbar_wait(done, 0, abort));
        if (ok) {
            tc_fence_after();
            float* dst = p.states + (((int64_t)b * p.h + head) * p.nslot + sub + 1) * (kP * kN);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t sv[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + 64 * hf + 32 * h2, sv);
                tmem_ld_wait();
                if (head_ok && !*abort) {  // an empty sub-segment contributes a zero state
#pragma unroll
                    for (int j = 0; j < 32; ++j) dst[(32 * h2 + j) * kN + r] = nch > 0 ? __uint_as_float(sv[j]) : 0.0f;
                }
            }
            if (head_ok && r == 0 && !*abort) p.seg_decay[((int64_t)b * p.h + head) * (p.nslot - 1) + sub] = D2;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem, 64 * HC);
    }
}

struct Plan {
    int nchunks, nseg, cps;
    int nsub;      // segment-state sub-segments per segment but the last
    int c0;        // blocks of segment 0
    double cost;   // modelled makespan, in chunk-scan blocks
};

// Free times of the SMs as (time, count) pairs, for list-scheduling whole grids of equal CTAs.
struct SmPool {
    std::map<double, int64_t> free_at;
    explicit SmPool(int sms) { free_at[0.0] = sms; }
    // Dispatch n CTAs in launch order onto the earliest free SMs; a CTA holds its SM from then
    // on, starts its work no earlier than `floor` and runs `dur`.  Returns the latest end and the
    // latest dispatch time.
    std::pair<double, double> take(int64_t n, double floor, double dur)
    {
        double last_end = 0.0, last_disp = 0.0;
        while (n > 0) {
            auto it = free_at.begin();
            const double t = it->first;
            const int64_t k = std::min(n, it->second);
            if ((it->second -= k) == 0) free_at.erase(it);
            const double end = std::max(t, floor) + dur;
            free_at[end] += k;
            last_end = std::max(last_end, end);
            last_disp = std::max(last_disp, t);
            n -= k;
        }
        return {last_end, last_disp};
    }
};

// Model costs in units of one 128-token block of the chunk scan with every SM busy (about 3.8 us
// on B200 for a block of two heads whose decay fits the factored form).
// The constants were fitted to plans timed on B200 over the scan and block shapes of 3 to 64 heads.
constexpr double kCtaStart = 1.0;    // chunk CTA: TMEM, barriers, pipeline fill
constexpr double kFoldSlot = 0.2;    // chunk CTA: folding one earlier sub-segment state (two heads)
constexpr double kSegStart = 0.5;    // segment-state CTA: TMEM, barriers, pipeline fill
constexpr double kSegGridEnd = 0.5;  // the segment-state grid's drain before the chunk scan may fold
constexpr double kSteep = 1.6;       // a block of a head pair that needs the exact decay form

// Makespan of one plan: the segment-state grid is dispatched first, then the chunk scan (a
// programmatic dependent, so only once every segment-state CTA is resident), segment by segment;
// CTAs of segments > 0 start their blocks when the segment-state grid has finished.  Heads with a
// steep decay make some CTAs kSteep times slower, wherever they land; the modelled makespan is
// the later of the uniform one and the end of such a CTA dispatched last in its segment.
double plan_cost(int sms, int64_t ctas, int64_t sctas, double seg_block, int nchunks, int ns, int nsub, int c0,
                 int c1)
{
    SmPool pool(sms);
    double seg_end = 0.0, seg_disp = 0.0;
    if (ns > 1) {
        for (int g = 0; g < 2; ++g) {  // sub-segments of segment 0, then those of the others
            const int len = g == 0 ? c0 : c1;
            const int64_t n = sctas * nsub * (g == 0 ? 1 : ns - 2);
            if (n == 0) continue;
            const auto r = pool.take(n, 0.0, seg_block * ((len + nsub - 1) / nsub + kSegStart));
            seg_end = std::max(seg_end, r.first);
            seg_disp = std::max(seg_disp, r.second);
        }
        seg_end += kSegGridEnd;
    }
    double cost = 0.0;
    for (int k = 0; k < ns; ++k) {
        const int len = k == 0 ? c0 : std::min(c1, nchunks - c0 - (k - 1) * c1);
        const double floor = k == 0 ? seg_disp : seg_end;
        const double start = kCtaStart + kFoldSlot * k * nsub;
        const auto r = pool.take(ctas, floor, len + start);
        cost = std::max(cost, std::max(r.first, std::max(r.second, floor) + kSteep * len + start));
    }
    return cost;
}

Plan plan_for_uncached(const ScanArgs& a, int sms)
{
    // Long sequences are cut into segments whose CTAs run side by side: a segment-state pass
    // computes each earlier segment's end state from a zero start (split into nsub sub-segments,
    // one CTA each, to shorten it), and every chunk-scan CTA folds the end states before its
    // segment.  Segment 0 needs no carried state: it starts at once and may take more blocks.
    Plan pl;
    pl.nchunks = (a.L + kQ - 1) / kQ;
    const int64_t ctas = (int64_t)a.batch * ((a.h + 1) / 2);  // chunk CTAs per segment: head pairs
    const bool quad = a.G == 1 || a.hpg % 4 == 0;
    const int64_t sctas = (int64_t)a.batch * (quad ? (a.h + 3) / 4 : (a.h + 1) / 2);  // per sub-segment
    const double seg_block = quad ? 0.43 : 0.34;  // a segment-state block, four (two) heads per CTA
    pl.nseg = 1;
    pl.nsub = 1;
    pl.cps = pl.c0 = pl.nchunks;
    pl.cost = plan_cost(sms, ctas, sctas, seg_block, pl.nchunks, 1, 1, pl.nchunks, pl.nchunks);
    // Measured on B200, beyond what the model sees: when one segment's CTAs fill three quarters
    // of the SMs, a single segment is fastest; when two or more segments fit on the SMs at once,
    // plans whose chunk-scan and segment-state CTAs all fit in one wave beat every plan that
    // needs a second one, so only those are searched.
    if (4 * ctas >= 3 * (int64_t)sms) return pl;
    const bool one_wave = sms / ctas >= 2;
    for (int ns = 2; ns <= pl.nchunks && ns <= 64; ++ns) {
        if (one_wave && ctas * ns > sms) break;
        const int even = (pl.nchunks + ns - 1) / ns;
        for (int nsub = 1; nsub <= 4; ++nsub) {
            if (one_wave && ctas + sctas * nsub * (ns - 1) > sms) break;
            // segment 0 of c0 >= even blocks, the others of c1 blocks each (the last one shorter,
            // never empty)
            for (int c0 = even; c0 <= std::min(pl.nchunks - (ns - 1), 2 * even + 2); ++c0) {
                const int rest = pl.nchunks - c0;
                const int c1 = (rest + ns - 2) / (ns - 1);
                if (rest - (ns - 2) * c1 <= 0) continue;
                const double cost = plan_cost(sms, ctas, sctas, seg_block, pl.nchunks, ns, nsub, c0, c1);
                if (cost < pl.cost - 1e-9) {
                    pl.cost = cost;
                    pl.nseg = ns;
                    pl.nsub = nsub;
                    pl.c0 = c0;
                    pl.cps = c1;
                }
            }
        }
    }
    return pl;
}

// Plans depend only on the shape and the SM count; the search is cached per shape.
Plan plan_for(const ScanArgs& a, int sms)
{
    static std::mutex mu;
    static std::map<std::tuple<int, int, int, int, int, int>, Plan> cache;
    const auto key = std::make_tuple(a.batch, a.L, a.h, a.G, a.hpg, sms);
    {
        std::lock_guard<std::mutex> lock(mu);
        const auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    const Plan pl = plan_for_uncached(a, sms);
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() < 4096) cache[key] = pl;
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
    const size_t nslot = (size_t)(pl.nseg - 1) * pl.nsub + 1;
    return align256(bh * nslot * kP * kN * 4) + align256(bh * (nslot - 1) * 4);
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
    ScanTcParams p{};
    p.L = a.L; p.h = a.h; p.nseg = pl.nseg; p.cps = pl.cps; p.nchunks = pl.nchunks; p.hpg = a.hpg;
    p.c0 = pl.c0;
    p.nsub = pl.nsub;
    p.nslot = (pl.nseg - 1) * pl.nsub + 1;
    p.dt = a.dt; p.sdt = a.sdt; p.A = a.A; p.D = a.D; p.y = a.y; p.sy = a.sy;
    // y leaves through bulk tensor stores when it is 16-byte aligned with 16-byte row pitches
    CUtensorMap mapY, mapZ;
    std::memset(&mapY, 0, sizeof(mapY));
    std::memset(&mapZ, 0, sizeof(mapZ));
    const bool y_tma = (reinterpret_cast<uintptr_t>(a.y) & 15u) == 0 && (a.sy * 2) % 16 == 0 &&
                       make_tmap_bf16_3d(&mapY, a.y, (uint64_t)a.h * kP, (uint64_t)a.L, (uint64_t)a.batch,
                                         (uint64_t)a.sy * 2, (uint64_t)a.sy * 2 * a.L, 64, kQ);
    p.y_tma = y_tma ? 1 : 0;
    if (gate && !make_tmap_bf16(&mapZ, gate->z, (uint64_t)a.h * kP, (uint64_t)rows, (uint64_t)gate->sz * 2, 64, kQ))
        return cudaErrorInvalidValue;
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
        p.seg_decay = reinterpret_cast<float*>(static_cast<char*>(ws) + align256(bh * p.nslot * kP * kN * 4));
    }
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<unsigned long long> attr_set{0};  // one bit per device
    if (dev >= 0 && dev < 64 && !(attr_set.load() >> dev & 1ull)) {
        cudaError_t e = cudaFuncSetAttribute(ssd_chunk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kChunkSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ssd_chunk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kChunkSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ssd_seg_state_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     SegCfg<4>::kSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ssd_seg_state_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     SegCfg<2>::kSmem);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(1ull << dev);
    }
    const dim3 cgrid((a.h + 1) / 2, a.batch, pl.nseg);
    if (pl.nseg == 1) {
        if (gate) ssd_chunk_kernel<true><<<cgrid, kChunkThreads, kChunkSmem, s>>>(mapX, mapB, mapC, mapY, mapZ, p);
        else ssd_chunk_kernel<false><<<cgrid, kChunkThreads, kChunkSmem, s>>>(mapX, mapB, mapC, mapY, mapZ, p);
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
        p.wait_all = 0;
        for (const auto& in : ins)
            if (ys.first < in.second && in.first < ys.second) p.wait_all = 1;
    }
    if (a.G == 1 || a.hpg % 4 == 0)  // four heads of one group per CTA
        ssd_seg_state_kernel<4><<<dim3((a.h + 3) / 4, p.nslot - 1, a.batch), SegCfg<4>::kThreads, SegCfg<4>::kSmem, s>>>(
            mapX, mapB, p);
    else
        ssd_seg_state_kernel<2><<<dim3((a.h + 1) / 2, p.nslot - 1, a.batch), SegCfg<2>::kThreads, SegCfg<2>::kSmem, s>>>(
            mapX, mapB, p);
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
    if (gate) return cudaLaunchKernelEx(&cfg, ssd_chunk_kernel<true>, mapX, mapB, mapC, mapY, mapZ, p);
    return cudaLaunchKernelEx(&cfg, ssd_chunk_kernel<false>, mapX, mapB, mapC, mapY, mapZ, p);
}

}  // namespace mm

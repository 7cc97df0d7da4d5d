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
//   2. state_pass : segment start states by a short sequential combine
//   3. chunk_scan : every segment from its true start state, carrying the
//                   state across blocks in registers (tcgen05)
// Only segment boundary states touch HBM.
//
// chunk_scan, one head per CTA (320 threads): warp 0 TMA producer, warp 1
// TMEM owner and tcgen05.mma issuer, warps 2-9 compute.  Compute thread
// (quarter q, lane l, half hf) owns TMEM lane r = 32q + l, i.e. token r of the
// block for Y and state row n = r for S, and half hf of the columns.
// TMEM columns: G = C B^T (128) | M = masked G as the bf16 A operand (64) |
// Y (64) | Y_off (64) | S = B^T X' (64).
#include <cuda.h>

#include <cmath>

#include "mm_internal.cuh"
#include "sm100.cuh"

namespace mm {

using namespace sm100;

namespace {

constexpr int kQ = 128;                       // tokens per block
constexpr int kP = 64;                        // head dim
constexpr int kN = 128;                       // state dim
constexpr int kTileQN = kQ * kN * 2;          // C or B block: two 64-column panels
constexpr int kTileQP = kQ * kP * 2;          // x, X' or H block: one panel
constexpr int kStage = 2 * kTileQN + kTileQP; // C | B | x
constexpr int kNStage = 2;
constexpr int kOffXP = kNStage * kStage;
constexpr int kOffH = kOffXP + kTileQP;
constexpr int kOffSmall = kOffH + kTileQP;
constexpr int kSmemBytes = kOffSmall + 2048 + 1024;

constexpr uint32_t kTG = 0, kTM = 128, kTY = 192, kTYO = 256, kTS = 320, kTCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

struct ScanTcParams {
    int L, h, nseg, cps, nchunks, hpg;
    const float* dt;
    int64_t sdt;
    const float* A;
    const float* D;
    void* y;
    int64_t sy;
    float* states;     // [b*h][nseg][P*N]: slot k = start state of segment k
    float* seg_decay;  // [b*h][nseg]: log2 of the decay over segment k
    const float* init_state;
    float* final_state;
    int64_t state_stride;
    int* status;
    // gated output (optional): y -> (y * SiLU(z)) * norm_w, sum of squares of y * SiLU(z) into row_sumsq
    const __nv_bfloat16* z;
    int64_t sz;
    const __nv_bfloat16* norm_w;
    float* row_parts;
};

__device__ __forceinline__ void named_sync_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128-byte-swizzled panel.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

template <bool FULL>
__global__ void __launch_bounds__(320, 1)
    ssd_tc_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapB,
                  const __grid_constant__ CUtensorMap mapC, const ScanTcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* cs2 = reinterpret_cast<float*>(sm + kOffSmall);  // [128] running log2-decay of each token
    float* dts = cs2 + kQ;                                    // [128] dt of each token (0 past the end)
    float* wtot = dts + kQ;                                   // [8] per-warp scan totals
    uint64_t* full = reinterpret_cast<uint64_t*>(wtot + 8);
    uint64_t* empty = full + kNStage;
    uint64_t* g_full = empty + kNStage;
    uint64_t* m_ready = g_full + 1;
    uint64_t* ys_full = m_ready + 1;
    uint64_t* done = ys_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int head = blockIdx.x, seg = blockIdx.y, b = blockIdx.z;
    const int c_begin = seg * p.cps;
    const int c_end = min(p.nchunks, c_begin + p.cps);
    const int nch = c_end - c_begin;
    const int grp = head / p.hpg;
    const int64_t tok0 = (int64_t)b * p.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNStage; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(g_full, 1);
        mbar_init(m_ready, 8);
        mbar_init(ys_full, 1);
        mbar_init(done, 1);
        *abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mapX);
        prefetch_tmap(&mapB);
        if (FULL) prefetch_tmap(&mapC);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {  // ------------------------------------------------ TMA producer
            constexpr uint32_t bytes = FULL ? kStage : (kTileQN + kTileQP);
            int k = 0;
            for (; k < nch; ++k) {
                const int s = k % kNStage;
                if (!mbar_wait(&empty[s], ((k / kNStage) & 1) ^ 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                const int row = (int)(tok0 + (int64_t)(c_begin + k) * kQ);
                uint8_t* base = sm + s * kStage;
                mbar_arrive_expect_tx(&full[s], bytes);
                if (FULL) {
                    tma_load_2d(base, &mapC, &full[s], grp * kN, row);
                    tma_load_2d(base + kTileQN / 2, &mapC, &full[s], grp * kN + 64, row);
                }
                tma_load_2d(base + kTileQN, &mapB, &full[s], grp * kN, row);
                tma_load_2d(base + kTileQN + kTileQN / 2, &mapB, &full[s], grp * kN + 64, row);
                tma_load_2d(base + 2 * kTileQN, &mapX, &full[s], head * kP, row);
            }
            for (int j = max(0, k - kNStage); j < k; ++j) mbar_wait(&full[j % kNStage], (j / kNStage) & 1, abort);
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ------------------------------------------------ MMA issuer
            const uint32_t id_g = idesc_bf16(128, 128, 0, 0);     // C (K-major) x B (K-major)
            const uint32_t id_y = idesc_bf16(128, 64, 0, 1);      // M (TMEM) / C (K-major) x MN-major
            const uint32_t id_s = idesc_bf16(128, 64, 1, 1);      // B^T (MN-major) x X' (MN-major)
            const uint32_t aXP = smem_u32(sm + kOffXP), aH = smem_u32(sm + kOffH);
            for (int k = 0; k < nch; ++k) {
                const int s = k % kNStage;
                if (!mbar_wait(&full[s], (k / kNStage) & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t aC = smem_u32(sm + s * kStage), aB = aC + kTileQN, aX = aB + kTileQN;
                if (FULL) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk & 3) * 32 + (kk >> 2) * (kTileQN / 2);
                        mma_ss(tmem + kTG, desc_sw128(aC + off, 16, 1024), desc_sw128(aB + off, 16, 1024), id_g,
                               kk > 0);
                    }
                    mma_commit(g_full);
                }
                if (!mbar_wait(m_ready, k & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                if (FULL) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // Y = M . X over the block's tokens
                        mma_ts(tmem + kTY, tmem + kTM + kk * 8, desc_sw128(aX + kk * 2048, 16384, 1024), id_y, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {  // Y_off = C . H_prev over the state dim
                        const uint32_t off = (kk & 3) * 32 + (kk >> 2) * (kTileQN / 2);
                        mma_ss(tmem + kTYO, desc_sw128(aC + off, 16, 1024), desc_sw128(aH + kk * 2048, 16384, 1024),
                               id_y, kk > 0);
                    }
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // S = B^T . X' over the block's tokens
                    mma_ss(tmem + kTS, desc_sw128(aB + kk * 2048, kTileQN / 2, 1024),
                           desc_sw128(aXP + kk * 2048, 16384, 1024), id_s, kk > 0);
                mma_commit(ys_full);
                mma_commit(&empty[s]);
            }
            mma_commit(done);
            mbar_wait(done, 0, nullptr);
        }
    } else {  // ------------------------------------------------------------ compute warps
        const int cw = warp - 2, q = warp & 3, hf = cw >> 2;
        const int r = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float A2 = p.A[head] * kLog2e;
        const float Dh = (FULL && p.D) ? p.D[head] : 0.0f;
        const int64_t bh = (int64_t)b * p.h + head;
        const int PN = kP * kN;

        // start state: row n = r, columns p in [32 hf, 32 hf + 32)
        float hs[32];
        {
            const float* src = nullptr;
            if (FULL) {
                if (p.nseg > 1) src = p.states + (bh * p.nseg + seg) * PN;
                else if (p.init_state) src = p.init_state + (int64_t)b * p.state_stride + (int64_t)head * PN;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) hs[j] = src ? src[(32 * hf + j) * kN + r] : 0.0f;
        }
        uint8_t* sH = sm + kOffH;
        uint8_t* sXP = sm + kOffXP;
        auto write_h = [&]() {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 v;
                v.x = pack_bf16(hs[8 * c + 0], hs[8 * c + 1]);
                v.y = pack_bf16(hs[8 * c + 2], hs[8 * c + 3]);
                v.z = pack_bf16(hs[8 * c + 4], hs[8 * c + 5]);
                v.w = pack_bf16(hs[8 * c + 6], hs[8 * c + 7]);
                *reinterpret_cast<uint4*>(sH + sw128(r, 4 * hf + c)) = v;
            }
        };
        if (FULL) write_h();
        float seg_log2 = 0.0f;

        for (int k = 0; k < nch; ++k) {
            const int s = k % kNStage;
            const int t0 = (c_begin + k) * kQ;
            const bool valid = t0 + r < p.L;
            const float dtv = valid ? p.dt[(tok0 + t0 + r) * p.sdt + head] : 0.0f;
            // inclusive scan of dt*A (log2 units) over the 128 tokens of the block
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
            const float c2 = sc + pre;  // log2 decay from the block start through token r
            if (hf == 0) {
                cs2[r] = c2;
                dts[r] = dtv;
            }
            named_sync_compute();

            if (!mbar_wait(&full[s], (k / kNStage) & 1, abort)) {
                raise_timeout(abort, p.status);
                break;
            }
            // X' = exp(cs_end - cs_r) dt_r x_r for this thread's 32 columns; keep x for the D term
            const uint8_t* sX = sm + s * kStage + 2 * kTileQN;
            uint4 xs[4];
            const float wgt = exp2f(tot - c2) * dtv;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                xs[c] = *reinterpret_cast<const uint4*>(sX + sw128(r, 4 * hf + c));
                uint4 o;
                o.x = pack_bf16(bf_lo(xs[c].x) * wgt, bf_hi(xs[c].x) * wgt);
                o.y = pack_bf16(bf_lo(xs[c].y) * wgt, bf_hi(xs[c].y) * wgt);
                o.z = pack_bf16(bf_lo(xs[c].z) * wgt, bf_hi(xs[c].z) * wgt);
                o.w = pack_bf16(bf_lo(xs[c].w) * wgt, bf_hi(xs[c].w) * wgt);
                *reinterpret_cast<uint4*>(sXP + sw128(r, 4 * hf + c)) = o;
            }
            fence_async_smem();

            if (FULL) {
                if (!mbar_wait(g_full, k & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                // M[t=r, s] = G[r, s] exp(cs_r - cs_s) dt_s for s <= r, else 0; columns [64 hf, 64 hf + 64)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int s0 = 64 * hf + 32 * j;
                    uint32_t pk[16];
                    if (s0 <= q * 32 + 31) {  // warp-uniform: some row of this warp reaches column s0
                        uint32_t gv[32];
                        tmem_ld32(tmem + lane_base + kTG + s0, gv);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int sa = s0 + e, sb = s0 + e + 1;
                            const float va = sa <= r ? __uint_as_float(gv[e]) * exp2f(c2 - cs2[sa]) * dts[sa] : 0.0f;
                            const float vb =
                                sb <= r ? __uint_as_float(gv[e + 1]) * exp2f(c2 - cs2[sb]) * dts[sb] : 0.0f;
                            pk[e >> 1] = pack_bf16(va, vb);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    }
                    tmem_st16(tmem + lane_base + kTM + s0 / 2, pk);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(m_ready);

            if (!mbar_wait(ys_full, k & 1, abort)) {
                raise_timeout(abort, p.status);
                break;
            }
            tc_fence_after();
            if (FULL) {
                uint32_t yv[32], ov[32];
                tmem_ld32(tmem + lane_base + kTY + 32 * hf, yv);
                tmem_ld32(tmem + lane_base + kTYO + 32 * hf, ov);
                tmem_ld_wait();
                const float ey = exp2f(c2);
                if (valid) {
                    const int64_t tok = tok0 + t0 + r;
                    const int col = head * kP + 32 * hf;
                    __nv_bfloat16* yo = static_cast<__nv_bfloat16*>(p.y) + tok * p.sy + col;
                    float ssq = 0.0f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t xw[4] = {xs[c].x, xs[c].y, xs[c].z, xs[c].w};
                        uint4 zw4 = make_uint4(0, 0, 0, 0), nw4 = make_uint4(0, 0, 0, 0);
                        if (p.z) {
                            zw4 = *reinterpret_cast<const uint4*>(p.z + tok * p.sz + col + 8 * c);
                            nw4 = *reinterpret_cast<const uint4*>(p.norm_w + col + 8 * c);
                        }
                        const uint32_t zw[4] = {zw4.x, zw4.y, zw4.z, zw4.w};
                        const uint32_t nw[4] = {nw4.x, nw4.y, nw4.z, nw4.w};
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = 8 * c + 2 * e;
                            float a0 = __uint_as_float(yv[j]) + ey * __uint_as_float(ov[j]) + Dh * bf_lo(xw[e]);
                            float a1 = __uint_as_float(yv[j + 1]) + ey * __uint_as_float(ov[j + 1]) + Dh * bf_hi(xw[e]);
                            if (p.z) {
                                const float z0 = bf_lo(zw[e]), z1 = bf_hi(zw[e]);
                                a0 *= __fdividef(z0, 1.0f + __expf(-z0));
                                a1 *= __fdividef(z1, 1.0f + __expf(-z1));
                                ssq = fmaf(a0, a0, fmaf(a1, a1, ssq));
                                a0 *= bf_lo(nw[e]);
                                a1 *= bf_hi(nw[e]);
                            }
                            o[e] = pack_bf16(a0, a1);
                        }
                        reinterpret_cast<uint4*>(yo)[c] = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                    if (p.z) p.row_parts[tok * 2 * p.h + 2 * head + hf] = ssq;
                }
            }
            {
                uint32_t sv[32];
                tmem_ld32(tmem + lane_base + kTS + 32 * hf, sv);
                tmem_ld_wait();
                const float dec = exp2f(tot);
#pragma unroll
                for (int j = 0; j < 32; ++j) hs[j] = fmaf(dec, hs[j], __uint_as_float(sv[j]));
            }
            if (FULL) {
                write_h();
                fence_async_smem();
            }
            tc_fence_before();
            seg_log2 += tot;
        }

        if (!*abort) {
            if (FULL) {
                if (seg == p.nseg - 1 && p.final_state) {
                    float* dst = p.final_state + (int64_t)b * p.state_stride + (int64_t)head * PN;
#pragma unroll
                    for (int j = 0; j < 32; ++j) dst[(32 * hf + j) * kN + r] = hs[j];
                }
            } else {
                float* dst = p.states + (bh * p.nseg + seg + 1) * PN;
#pragma unroll
                for (int j = 0; j < 32; ++j) dst[(32 * hf + j) * kN + r] = hs[j];
                if (r == 0 && hf == 0) p.seg_decay[bh * p.nseg + seg] = seg_log2;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTCols);
}

// Segment start states: slot 0 = initial state (or zero); slot k = state after
// segment k-1, combined in order from the local end states K_a left in slots
// 1..nseg-1.  One thread per state element.
__global__ void ssd_state_pass_kernel(float* states, const float* seg_decay, const float* init, int64_t state_stride,
                                      int64_t bh_total, int h, int nseg)
{
    constexpr int PN = kP * kN;
    const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (idx >= bh_total * PN) return;
    const int64_t bh = idx / PN;
    const int e = (int)(idx % PN);
    const int64_t b = bh / h, i = bh % h;
    float cur = init ? init[b * state_stride + i * PN + e] : 0.0f;
    float* base = states + bh * nseg * PN + e;
    base[0] = cur;
    for (int k = 1; k < nseg; ++k) {
        cur = fmaf(exp2f(seg_decay[bh * nseg + k - 1]), cur, base[(int64_t)k * PN]);
        base[(int64_t)k * PN] = cur;
    }
}

struct Plan {
    int nchunks, nseg, cps;
};

Plan plan_for(const ScanArgs& a, int sms)
{
    Plan pl;
    pl.nchunks = (a.L + kQ - 1) / kQ;
    const int64_t bh = (int64_t)a.batch * a.h;
    double best = 1e30;
    pl.nseg = 1;
    pl.cps = pl.nchunks;
    for (int ns = 1; ns <= pl.nchunks && ns <= 64; ++ns) {
        const int cps = (pl.nchunks + ns - 1) / ns;
        const int nseg = (pl.nchunks + cps - 1) / cps;
        if (nseg != ns) continue;
        const double waves = std::ceil((double)(bh * nseg) / sms);
        double cost = waves * cps;
        if (nseg > 1) cost += 0.4 * std::ceil((double)(bh * (nseg - 1)) / sms) * cps + 1.0;
        if (cost < best - 1e-9) {
            best = cost;
            pl.nseg = nseg;
            pl.cps = cps;
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
    return a.P == kP && a.N == kN && a.chunk % kQ == 0 && a.batch > 0 && a.L > 0 && a.h > 0 && a.G > 0 &&
           (int64_t)a.batch * a.L < (1ll << 31);
}

size_t scan_tc_workspace(const ScanArgs& a)
{
    const Plan pl = plan_for(a, num_sms());
    if (pl.nseg == 1) return 256;
    const size_t bh = (size_t)a.batch * a.h;
    return align256(bh * pl.nseg * kP * kN * 4) + align256(bh * pl.nseg * 4);
}

int scan_tc_kernel_count(const ScanArgs& a) { return plan_for(a, num_sms()).nseg > 1 ? 3 : 1; }

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

    ScanTcParams p{};
    p.L = a.L; p.h = a.h; p.nseg = pl.nseg; p.cps = pl.cps; p.nchunks = pl.nchunks; p.hpg = a.hpg;
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
        cudaError_t e = cudaFuncSetAttribute(ssd_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ssd_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set |= 1ull << dev;
    }
    if (pl.nseg > 1) {
        ssd_tc_kernel<false><<<dim3(a.h, pl.nseg - 1, a.batch), 320, kSmemBytes, s>>>(mapX, mapB, mapC, p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        const int64_t n = (int64_t)bh * kP * kN;
        ssd_state_pass_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p.states, p.seg_decay, a.init_state,
                                                                           a.state_stride, (int64_t)bh, a.h, pl.nseg);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    ssd_tc_kernel<true><<<dim3(a.h, pl.nseg, a.batch), 320, kSmemBytes, s>>>(mapX, mapB, mapC, p);
    return cudaGetLastError();
}

}  // namespace mm

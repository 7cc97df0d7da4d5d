// Tensor-core projection GEMM for sm_100a: out = A . B^T with bf16 operands,
// fp32 accumulation in TMEM, TMA-fed shared-memory stages, and a tile loop
// per CTA.  Serves in_proj (A = u, B = the four row blocks of the W_in
// width view, routed to z | x | B | C and an fp32 dt buffer) and out_proj
// (A = normalised activations, B = W_out with its K-prefix [0, d)); the width
// view is a set of row offsets and a K extent, never a weight copy
// ("MatMamba: A Matryoshka State Space Model", nested sub-block paragraph:
// W_x becomes W_x[0:d_i] by slicing along d_inner).
//
// CTA layout (320 threads): warp 0 schedules tiles and issues TMA loads, warp 1
// owns TMEM and issues tcgen05.mma from one lane, warps 2-9 drain the
// accumulator in two groups of four that take alternate 32-column chunks (one
// TMEM lane = one output row per thread) and store.  Two TMEM accumulators let
// the drain of tile i overlap the MMAs of tile i+1.
//
// Scheduling: the grid has one CTA per tile, but a running CTA keeps taking the
// tiles of CTAs that have not started yet (cluster launch control), so the SMs
// that drain their tiles faster take more of them and all finish together.
#include <cuda.h>

#include <atomic>
#include <cstring>

#include "mm_internal.cuh"
#include "sm100.cuh"

namespace mm {

using namespace sm100;

namespace {

__device__ __forceinline__ float bf_lo_u(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi_u(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

constexpr int kBM = 128;  // rows of a tile = TMEM lanes
constexpr int kBK = 64;   // one 128-byte swizzle atom of bf16 along K
constexpr int kStageLd = 36;  // fp32 row pitch of the conv walks' staging rows (32 columns + pad)
constexpr int kUsePairs = 1;  // wide tiles on CTA pairs (cta_group::2) where launch_gemm_tc selects them
constexpr int kTileRing = 6;  // launch-control answers in flight (producer leads the drain by <= 4 tiles)

struct TcSeg {
    void* out;
    int64_t ldo;
    int b_row0;  // row of the B tensor map holding this segment's column 0
    int n;       // columns in the segment
    int ntiles;  // ceil(n / BN)
    int out_f32;
    int accumulate;
    int vec_ok;  // 16-byte vector stores allowed
    int tma;     // tiles leave through bulk tensor operations (OutMaps::m[segment]): 1 bf16 store,
                 // 2 fp32 store, 3 fp32 add into the output (accumulate)
    int kind;    // GemmEpi
    int conv_row0;
};

// Output tensor maps of the segments whose tiles leave through bulk tensor stores
// (bf16, 64 x 128 boxes, 128-byte swizzle).
struct OutMaps {
    CUtensorMap m[kMaxSeg];
};

struct TcParams {
    int M, K, ktiles, mtiles, ntiles, nseg;
    // split K: tiles come in ksplit K slices of kper k-tiles each; every slice adds its partial
    // product into the (fp32, bulk-add) output, so only single-segment accumulating outputs split
    int ksplit, kper;
    int shift;  // halo rows at the top of each tile (K-1 with a conv segment, else 0)
    int rows;   // output rows per tile = 128 - shift
    // Paired tiles (the first pair_tiles tiles of a row block): columns [n0, n0 + BN/2) of segment
    // pair_a (a plain bf16 store) in accumulator columns [0, BN/2) and the same columns of segment
    // pair_b (conv) in [BN/2, BN), so that every tile's drain mixes cheap stores and conv walks.
    // Both segments then have ntiles = 0 in the walk over the rest.
    int pair_tiles, pair_a, pair_b;
    TcSeg seg[kMaxSeg];
    GemmExtra ex;
    int* status;
    int pdl;  // launched as a programmatic dependent: wait for the previous kernel before reading
};

template <int BN>
struct TileInfo {
    int mt, seg, n0, nvalid, b_row;
    int seg2, b_row2;  // paired tile: the conv segment and its B row (else seg2 = -1)
    int k0, k1;        // k-tiles [k0, k1) of this tile's K slice
};

// Tile j of row block mt (mt may be one past the last row block: a pair's odd CTA then has a tile
// of rows past M, which load as zeros and store nothing).
template <int BN>
__device__ __forceinline__ TileInfo<BN> tile_info_mj(const TcParams& p, int mt, int j)
{
    TileInfo<BN> t;
    t.k0 = 0;
    t.k1 = p.ktiles;
    t.mt = mt;
    t.seg2 = -1;
    t.b_row2 = 0;
    if (j < p.pair_tiles) {
        t.seg = p.pair_a;
        t.seg2 = p.pair_b;
        t.n0 = j * (BN / 2);
        t.nvalid = min(BN / 2, p.seg[t.seg].n - t.n0);
        t.b_row = p.seg[t.seg].b_row0 + t.n0;
        t.b_row2 = p.seg[t.seg2].b_row0 + t.n0;
        return t;
    }
    j -= p.pair_tiles;
    int s = 0;
    while (s < p.nseg - 1 && j >= p.seg[s].ntiles) j -= p.seg[s++].ntiles;
    t.seg = s;
    t.n0 = j * BN;
    t.nvalid = min(BN, p.seg[s].n - t.n0);
    t.b_row = p.seg[s].b_row0 + t.n0;
    return t;
}

// Tile index -> (K slice, row block, N tile), K slices slowest.  Row-block major: the N tiles of a
// row block are consecutive, so CTAs working at the same time share its A rows in L2.
template <int BN>
__device__ __forceinline__ TileInfo<BN> tile_info(const TcParams& p, int tile)
{
    const int per_slice = p.mtiles * p.ntiles;
    const int ks = tile / per_slice;
    tile -= ks * per_slice;
    TileInfo<BN> t = tile_info_mj<BN>(p, tile / p.ntiles, tile % p.ntiles);
    t.k0 = ks * p.kper;
    t.k1 = min(p.ktiles, t.k0 + p.kper);
    return t;
}

// a / (1 + 2^(-a log2 e)) from the MUFU approximations of 2^x and 1/x; -0 for very negative a.
__device__ __forceinline__ float silu_fast(float a)
{
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(a * -1.4426950408889634f));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
    return a * r;
}

__device__ __forceinline__ void store_bf16_chunk(__nv_bfloat16* o, int ncols, bool vec, const float (&v)[32])
{
    if (ncols == 32 && vec) {
        uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o4[q] = make_uint4(pack_bf16(v[8 * q + 0], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                               pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < ncols) o[i] = __float2bfloat16_rn(v[i]);
    }
}

// PAIR: the kernel runs as clusters of two CTAs sharing each MMA (M = 256 over the pair).  CTA r
// of a cluster takes row block 2 m + r of tile pair (m, j): it loads its own A rows and half of the
// tile's B rows (the store rows of a paired tile in the even CTA and its conv rows in the odd one;
// otherwise the first and second halves of the N columns the MMA uses), and drains its own
// accumulator rows.  The even CTA issues the MMAs; both CTAs' loads complete its stage barriers,
// its commits reach both CTAs, and the odd CTA's drain warps release the accumulator with remote
// arrives.  Per SM, a pair tile loads 128 A rows and 128 B rows per K step for the work that one
// CTA alone loads 128 and 256 for.  The walk over tile pairs is static.
template <int BN, int STAGES, bool CONV, bool PAIR>
__global__ void __launch_bounds__(320, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                   const __grid_constant__ CUtensorMap mapB2, const __grid_constant__ OutMaps omaps, const TcParams p)
{
    constexpr int A_BYTES = kBM * kBK * 2;
    constexpr int B_BYTES = BN * kBK * 2;
    constexpr int STAGE_BYTES = A_BYTES + (PAIR ? B_BYTES / 2 : B_BYTES);  // this CTA's bytes of a stage
    constexpr uint32_t TMEM_COLS = 2 * BN;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // Per drain group: [128 rows][kStageLd] fp32, a 32-column chunk of accumulators for the conv
    // walks; the same bytes hold [128 rows][128 bytes] in the 128-byte swizzle (piece c of row r at
    // c ^ (r % 8)), a 64-column bf16 (or 32-column fp32) unit for the bulk stores.
    constexpr int kGroupStage = CONV ? kBM * kStageLd * 4 : kBM * 128;  // both multiples of 1024
    float* stage = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
    // answers of the launch-control requests (one per tile position, kTileRing in flight at most)
    uint4* cresp = reinterpret_cast<uint4*>(smem + STAGES * STAGE_BYTES + 2 * kGroupStage);
    uint64_t* full = reinterpret_cast<uint64_t*>(cresp + kTileRing);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* done = tempty + 2;
    uint64_t* cfull = done + 1;          // answer j has landed
    uint64_t* cempty = cfull + kTileRing;  // answer j has been read by the MMA lane and the 8 drain warps
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cempty + kTileRing);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0;  // the pair's even CTA (0) issues its MMAs
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);  // the pair: the even CTA's arrive; both CTAs' loads complete it
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], PAIR ? 16 : 8);  // the pair: both CTAs' drain warps
        }
        for (int j = 0; j < kTileRing; ++j) {
            mbar_init(&cfull[j], 1);
            mbar_init(&cempty[j], 9);
        }
        mbar_init(done, 1);
        *abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mapA);
        prefetch_tmap(&mapB);
        if (p.pair_tiles) prefetch_tmap(&mapB2);
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(tmem_slot, TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();  // both CTAs' barriers are initialised before any arrives on them
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Programmatic dependent launch: the set-up above may overlap the previous kernel's tail; nothing
    // that kernel writes is read before it has completed.  A following dependent may start its own
    // set-up once every CTA of this grid has started.
    if (p.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // tiles: (K slice, row block, N tile), K slices slowest
    const int total = p.mtiles * p.ntiles * p.ksplit;
    // the pair's static walk: tile pair tp = (row-block pair tp / ntiles, N tile tp % ntiles); CTA r
    // takes tile (2 (tp / ntiles) + r) ntiles + tp % ntiles
    const int total_pairs = ((p.mtiles + 1) / 2) * p.ntiles;
    const int ncl = (int)gridDim.x / 2, cl = (int)blockIdx.x / 2;
    auto pair_info = [&](int tp) -> TileInfo<BN> {
        return tile_info_mj<BN>(p, (tp / p.ntiles) * 2 + (int)rank, tp % p.ntiles);
    };
    const uint32_t tempty_even = PAIR ? cluster_addr(tempty, 0) : 0;  // the even CTA's barriers
    const uint32_t full_even = PAIR ? cluster_addr(full, 0) : 0;
    auto release_acc = [&](int b) {  // this drain warp is done with accumulator b
        if (PAIR) mbar_arrive_remote(tempty_even + 8u * b);
        else mbar_arrive(&tempty[b]);
    };
    // the MMA's N for a tile: a paired tile's BN; otherwise its columns rounded up to 16 (32 for a pair)
    auto mma_n = [&](const TileInfo<BN>& t) -> int {
        if (t.seg2 >= 0) return BN;
        const int n = (t.nvalid + 15) & ~15;
        return PAIR ? max(n, 32) : n;
    };
    // The tile of position j + 1 (`total` once the walk is over) from the scheduler's answer j;
    // each reader then releases the answer's slot (the MMA lane alone, or a drain warp once all
    // its lanes have read).  The wait ignores the abort flag, so every reader of an answer that
    // landed follows the same tile sequence and the drain groups' named barriers stay in step.
    auto next_tile = [&](int j, bool single) -> int {
        const int cs = j % kTileRing;
        bool got = mbar_wait(&cfull[cs], (j / kTileRing) & 1, nullptr);
        if (!single) got = __all_sync(0xffffffffu, got);
        const int nx = got ? clc_cancelled_x(&cresp[cs]) : -1;
        if (!single) __syncwarp();
        if (single || lane == 0) mbar_arrive(&cempty[cs]);
        return nx < 0 ? total : nx;
    };

    if (warp == 0) {
        if (PAIR && lane == 0) {  // ---------------- TMA producer of a pair CTA
            int it = 0;
            for (int j = 0; cl + j * ncl < total_pairs && !*abort; ++j) {
                const TileInfo<BN> t = pair_info(cl + j * ncl);
                const int arow = t.mt * p.rows - p.shift;  // rows outside [0, M) load as zeros
                const int brow = t.seg2 >= 0 ? (rank ? t.b_row2 : t.b_row) : t.b_row + (int)rank * (mma_n(t) / 2);
                for (int kt = 0; kt < p.ktiles; ++kt, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort)) {
                        raise_timeout(abort, p.status);
                        break;
                    }
                    uint8_t* sa = smem + s * STAGE_BYTES;
                    // the even CTA expects both CTAs' bytes; the odd CTA's loads can only land after
                    // the previous phase completed (its stage was freed by an MMA that waited for it)
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
                    tma_load_2d_pair(sa, &mapA, full_even + 8u * s, kt * kBK, arow);
                    tma_load_2d_pair(sa + A_BYTES, &mapB2, full_even + 8u * s, kt * kBK, brow);
                }
            }
            // the even CTA sees every load of both CTAs land (bounded); the odd CTA's loads have
            // landed before the even CTA reaches the closing cluster barrier
            if (rank == 0)
                for (int i = max(0, it - STAGES); i < it; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, nullptr);
        } else if (!PAIR && lane == 0) {  // ---------------- tile scheduler and TMA producer
            // Tile position 0 is this CTA's own index; the tile of position j + 1 is the index of a
            // CTA that had not started yet, cancelled by a launch-control request made while tile j
            // loads.  An answer that cancelled nothing ends the walk (the grid has one CTA per tile).
            int it = 0, j = 0, tile = blockIdx.x;
            bool asked = false;  // an answer is in flight
            while (tile < total && !*abort) {
                const int cs = j % kTileRing;
                if (!mbar_wait(&cempty[cs], ((j / kTileRing) & 1) ^ 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                mbar_arrive_expect_tx(&cfull[cs], 16);
                clc_try_cancel(&cresp[cs], &cfull[cs]);
                asked = true;
                const TileInfo<BN> t = tile_info<BN>(p, tile);
                const int arow = t.mt * p.rows - p.shift;  // may be negative: rows above 0 load as zeros
                for (int kt = t.k0; kt < t.k1; ++kt, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort)) {
                        raise_timeout(abort, p.status);
                        break;
                    }
                    uint8_t* sa = smem + s * STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
                    tma_load_2d(sa, &mapA, &full[s], kt * kBK, arow);
                    if (t.seg2 >= 0) {  // two half-height boxes: the store rows, then the conv rows
                        tma_load_2d(sa + A_BYTES, &mapB2, &full[s], kt * kBK, t.b_row);
                        tma_load_2d(sa + A_BYTES + B_BYTES / 2, &mapB2, &full[s], kt * kBK, t.b_row2);
                    } else {
                        tma_load_2d(sa + A_BYTES, &mapB, &full[s], kt * kBK, t.b_row);
                    }
                }
                if (!mbar_wait(&cfull[cs], (j / kTileRing) & 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                asked = false;
                const int nx = clc_cancelled_x(&cresp[cs]);
                tile = nx < 0 ? total : nx;
                ++j;
            }
            // the last answer and every issued load land before the CTA can exit (bounded)
            if (asked) mbar_wait(&cfull[j % kTileRing], (j / kTileRing) & 1, nullptr);
            for (int i = max(0, it - STAGES); i < it; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, nullptr);
        }
    } else if (warp == 1) {
        if (PAIR && lane == 0 && rank == 0) {  // ---------------- MMA issuer of the pair
            int it = 0;
            for (int j = 0; cl + j * ncl < total_pairs && !*abort; ++j) {
                const TileInfo<BN> t = pair_info(cl + j * ncl);
                const int buf = j & 1;
                if (!mbar_wait(&tempty[buf], ((j >> 1) & 1) ^ 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * BN;
                const uint32_t idesc = idesc_bf16(2 * kBM, mma_n(t), 0, 0);
                for (int kt = 0; kt < p.ktiles; ++kt, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&full[s], (it / STAGES) & 1, abort)) {
                        raise_timeout(abort, p.status);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_ss_pair(d_tmem, desc_sw128(a0 + kk * 32, 16, 1024), desc_sw128(b0 + kk * 32, 16, 1024),
                                    idesc, (kt != 0 || kk != 0) ? 1u : 0u);
                    mma_commit_pair(&empty[s]);
                }
                mma_commit_pair(&tfull[buf]);
            }
            // every issued MMA has finished before TMEM can be released (bounded)
            mma_commit_pair(done);
            mbar_wait(done, 0, nullptr);
        } else if (!PAIR && lane == 0) {  // ---------------- MMA issuer
            int it = 0, tc = 0;
            for (int tile = blockIdx.x; tile < total && !*abort; ++tc) {
                const TileInfo<BN> t = tile_info<BN>(p, tile);
                const int buf = tc & 1;
                if (!mbar_wait(&tempty[buf], ((tc >> 1) & 1) ^ 1, abort)) {
                    raise_timeout(abort, p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * BN;
                const uint32_t idesc = idesc_bf16(kBM, mma_n(t), 0, 0);
                for (int kt = t.k0; kt < t.k1; ++kt, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&full[s], (it / STAGES) & 1, abort)) {
                        raise_timeout(abort, p.status);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_ss(d_tmem, desc_sw128(a0 + kk * 32, 16, 1024), desc_sw128(b0 + kk * 32, 16, 1024), idesc,
                               (kt != t.k0 || kk != 0) ? 1u : 0u);
                    mma_commit(&empty[s]);
                }
                mma_commit(&tfull[buf]);
                tile = next_tile(tc, true);
            }
            // every issued MMA has finished before TMEM can be released (bounded)
            mma_commit(done);
            mbar_wait(done, 0, nullptr);
        }
    } else {  // ---------------- epilogue: warps 2..9, two groups alternating 32-column chunks
        const int q = warp & 3;
        const int eg = (warp - 2) >> 2;
        const int r = q * 32 + lane;  // tile row = TMEM lane
        const GemmExtra& ex = p.ex;
        int tc = 0;
        // the walk: the pair's static one over tile pairs, else this CTA's own tile, then the
        // scheduler's answers
        for (int tile = PAIR ? cl : (int)blockIdx.x; PAIR ? tile < total_pairs : tile < total;
             tile = PAIR ? tile + ncl : next_tile(tc, false), ++tc) {
            const TileInfo<BN> t = PAIR ? pair_info(tile) : tile_info<BN>(p, tile);
            const int buf = tc & 1;
            const TcSeg& sg = p.seg[t.seg];
            const bool paired = t.seg2 >= 0;
            const TcSeg& cs = p.seg[paired ? t.seg2 : t.seg];  // the segment of the chunk loop's columns
            const int cbase = paired ? BN / 2 : 0;            // and their first accumulator column
            const int64_t m = (int64_t)t.mt * p.rows - p.shift + r;  // token of this row
            const bool row_ok = r >= p.shift && m < p.M;
            // the row scale does not depend on the accumulator: its loads go out before the wait
            float scale = 1.0f;
            if (ex.row_parts && row_ok) {
                const float* rp = ex.row_parts + m * ex.nparts;
                float ss = 0.0f;
                if ((ex.nparts & 3) == 0) {  // rows of partials are 16-byte aligned
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int j = 0; j < ex.nparts; j += 4) {
                        const float4 v4 = *reinterpret_cast<const float4*>(rp + j);
                        acc.x += v4.x; acc.y += v4.y; acc.z += v4.z; acc.w += v4.w;
                    }
                    ss = (acc.x + acc.y) + (acc.z + acc.w);
                } else {
                    for (int j = 0; j < ex.nparts; ++j) ss += rp[j];
                }
                scale = rsqrtf(ss * ex.rs_inv_n + ex.rs_eps);
            }
            // Conv tiles: this thread's walk stores outputs at rows [wr0, wr0 + 16) of the tile
            // (wr0 = 16 rb, rb = 2 q + lane / 16) from a window of rows [wr0 - 3, wr0 + 16).  Outputs
            // [w_ilo, w_ihi) are stored: the top walk's first rows are the tile's halo, and rows past
            // the last token are no tokens.  w_m0, w_tp0: the token of row wr0 and its position in its
            // sequence.  Path 1: every stored output's three history rows are earlier rows of its own
            // sequence in the window (and none is one of the last K-1 of its sequence when the conv
            // state is written); path 2: the walk meets a sequence start or the end of the tokens;
            // path 0: anything else.
            const int wrb = 2 * q + (lane >> 4), wr0 = 16 * wrb;
            const int lc = 2 * (lane & 15);  // the walk's column pair within a chunk
            int64_t w_m0 = 0;
            int w_tp0 = 0, w_ilo = 0, w_ihi = 0, w_path = 0;
            if (CONV && cs.kind == kEpiConv) {
                w_m0 = (int64_t)t.mt * p.rows - p.shift + wr0;
                w_tp0 = (int)(((w_m0 % ex.L) + ex.L) % ex.L);
                w_ilo = wr0 < p.shift ? p.shift - wr0 : 0;
                const int64_t left = (int64_t)p.M - w_m0;  // tokens from row wr0 on
                w_ihi = left <= 0 ? 0 : (left < 16 ? (int)left : 16);
                const int tpf = (w_tp0 + w_ilo) % ex.L;  // position of the first stored output
                const bool vec = cs.vec_ok && p.shift == 3;
                const int tail = ex.conv_state_out ? 3 : 0;
                if (vec && w_ihi == 16 && tpf >= 3 && tpf + (15 - w_ilo) + tail < ex.L) w_path = 1;
                else if (vec && ex.L >= 19 && w_ihi > w_ilo) w_path = 2;
            }
            // filters and biases of the pair in the group's chunk j (zeros when the walk does not use them)
            auto load_filters = [&](int j, uint2& fa, uint2& fb, uint32_t& fbi) {
                const int cc = 32 * eg + 64 * j + lc;  // column of the pair in the chunk loop's columns
                fa = fb = make_uint2(0, 0);
                fbi = 0;
                if (CONV && cs.kind == kEpiConv && w_path && cc + 1 < t.nvalid) {
                    const __nv_bfloat16* cw = static_cast<const __nv_bfloat16*>(ex.conv_w);
                    const __nv_bfloat16* cb = static_cast<const __nv_bfloat16*>(ex.conv_b);
                    const int crow = cs.conv_row0 + t.n0 + cc;
                    fa = *reinterpret_cast<const uint2*>(cw + (int64_t)crow * 4);
                    fb = *reinterpret_cast<const uint2*>(cw + (int64_t)(crow + 1) * 4);
                    fbi = (uint32_t)__bfloat16_as_ushort(cb[crow]) | ((uint32_t)__bfloat16_as_ushort(cb[crow + 1]) << 16);
                }
            };
            // the first two chunks' filters go out before the accumulator wait; each chunk then
            // fetches the filters of the chunk after next
            uint2 fwa[2], fwb[2];
            uint32_t fbias[2];
            load_filters(0, fwa[0], fwb[0], fbias[0]);
            load_filters(1, fwa[1], fwb[1], fbias[1]);
            // dt biases of the group's first 16-column chunk of a softplus tile, loaded before the wait
            float dtb[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) dtb[i] = 0.0f;
            if (sg.kind == kEpiSoftplus) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (16 * eg + i < t.nvalid) dtb[i] = ex.dt_bias[t.n0 + 16 * eg + i];
            }
            // a failed wait skips this tile's work but keeps the group's named barriers in step
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], (tc >> 1) & 1, abort));
            if (!ok) raise_timeout(abort, p.status);
            tc_fence_after();
            if (sg.kind == kEpiSoftplus) {
                // dt columns (a few dozen at most): 16-column chunks, group eg takes chunks eg, eg + 2, ...
                for (int c0 = 16 * eg; c0 < t.nvalid; c0 += 32) {
                    if (!ok) continue;
                    uint32_t raw[16];
                    tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + buf * BN + c0, raw);
                    tmem_ld_wait();
                    if (row_ok) {
                        float* o = static_cast<float*>(sg.out) + m * sg.ldo + t.n0 + c0;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < t.nvalid) {
                                const float bias = c0 == 16 * eg ? dtb[i] : ex.dt_bias[t.n0 + c0 + i];
                                const float a = __uint_as_float(raw[i]) + bias;
                                o[i] = a > 20.0f ? a : log1pf(__expf(a));
                            }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) release_acc(buf);
                continue;
            }
            const int64_t tile_row0 = (int64_t)t.mt * p.rows - p.shift;  // token of tile row 0
            if (sg.tma >= 2 && tile_row0 >= 0 && tile_row0 < p.M) {
                // fp32 outputs: 32-column units (group eg takes units eg, eg + 2, ...), rows staged in
                // the 128-byte-swizzled layout, then one bulk store or bulk add per unit.  Each output
                // element gets exactly one add per launch, the same fp32 add as a read-modify-write.
                uint8_t* stg = reinterpret_cast<uint8_t*>(stage) + eg * kGroupStage;
                for (int u = eg; 32 * u < t.nvalid; u += 2) {
                    asm volatile("bar.sync %0, 128;" ::"r"(2 + eg) : "memory");  // staging rows free
                    if (ok) {
                        uint32_t raw[32];
                        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + buf * BN + 32 * u, raw);
                        tmem_ld_wait();
                        float v[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
                        if (ex.row_parts) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] *= scale;
                        }
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<float4*>(stg + r * 128 + ((c ^ (r & 7)) << 4)) =
                                make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                    }
                    fence_async_smem();
                    asm volatile("bar.sync %0, 128;" ::"r"(2 + eg) : "memory");
                    if (ok && q == 2 && lane == 0) {  // one issuer per group
                        if (sg.tma == 3) tma_reduce_add_2d(&omaps.m[t.seg], stg, t.n0 + 32 * u, (int)tile_row0);
                        else tma_store_2d(&omaps.m[t.seg], stg, t.n0 + 32 * u, (int)tile_row0);
                        bulk_commit();
                        bulk_wait_read0();
                    }
                }
                asm volatile("bar.sync %0, 128;" ::"r"(2 + eg) : "memory");  // last unit's rows read
                tc_fence_before();
                __syncwarp();
                if (lane == 0) release_acc(buf);
                continue;
            }
            if (sg.tma == 1 && tile_row0 >= 0 && tile_row0 < p.M) {
                // 64-column units (group eg takes units eg, eg + 2, ...): rows staged as bf16 in the
                // 128-byte-swizzled layout, then one bulk store per unit.  Halo rows above the tile's
                // outputs rewrite the identical values the previous row block wrote.  A paired tile
                // stores its first half this way and goes on to its conv half.
                uint8_t* stg = reinterpret_cast<uint8_t*>(stage) + eg * kGroupStage;
                for (int u = eg; 64 * u < t.nvalid; u += 2) {
                    // the previous unit's store has read the staging rows (its issuer waited)
                    asm volatile("bar.sync %0, 128;" ::"r"(2 + eg) : "memory");
                    if (ok) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint32_t raw[32];
                            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + buf * BN + 64 * u + 32 * hh, raw);
                            tmem_ld_wait();
                            float v[32];
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
                            if (ex.row_parts) {
#pragma unroll
                                for (int i = 0; i < 32; ++i) v[i] *= scale;
                            }
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const uint4 w = make_uint4(pack_bf16(v[8 * c + 0], v[8 * c + 1]), pack_bf16(v[8 * c + 2], v[8 * c + 3]),
                                                           pack_bf16(v[8 * c + 4], v[8 * c + 5]), pack_bf16(v[8 * c + 6], v[8 * c + 7]));
                                const int chunk = 4 * hh + c;
                                *reinterpret_cast<uint4*>(stg + r * 128 + ((chunk ^ (r & 7)) << 4)) = w;
                            }
                        }
                    }
                    fence_async_smem();
                    asm volatile("bar.sync %0, 128;" ::"r"(2 + eg) : "memory");
                    if (ok && q == 2 && lane == 0) {  // one issuer per group
                        tma_store_2d(&omaps.m[t.seg], stg, t.n0 + 64 * u, (int)tile_row0);
                        bulk_commit();
                        bulk_wait_read0();
                    }
                }
                // the last store has read the staging rows before the group writes them again
                asm volatile("bar.sync %0, 128;" ::"r"(2 + eg) : "memory");
                if (!paired) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) release_acc(buf);
                    continue;
                }
            } else if (paired) {  // first half of a paired tile at the top row block: plain stores
                for (int c0 = 32 * eg; c0 < t.nvalid; c0 += 64) {
                    if (!ok) continue;
                    uint32_t raw[32];
                    tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + buf * BN + c0, raw);
                    tmem_ld_wait();
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
                    if (row_ok)
                        store_bf16_chunk(static_cast<__nv_bfloat16*>(sg.out) + m * sg.ldo + t.n0 + c0,
                                         min(32, t.nvalid - c0), sg.vec_ok, v);
                }
            }
            for (int c0 = 32 * eg; c0 < t.nvalid; c0 += 64) {
                float v[32];
                if (ok) {
                    uint32_t raw[32];
                    tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + buf * BN + cbase + c0, raw);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
                    if (ex.row_parts) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= scale;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                }
                const int ncols = min(32, t.nvalid - c0);
                const int col = t.n0 + c0;
                if (CONV && cs.kind == kEpiConv) {
                    // The chunk goes through shared memory so that each thread can walk down the token
                    // axis over its column pair, keeping a window of pre-conv values in registers.
                    // Taps never cross a sequence start: there the window restarts from the given
                    // history (or zeros).
                    float* st = stage + eg * (kBM * kStageLd);
                    // the pre-conv values of columns lc, lc + 1 (lc even) in row `row` of the chunk
                    auto xat = [st](int row, int lc2) -> float2 {
                        return *reinterpret_cast<const float2*>(st + row * kStageLd + lc2);
                    };
                    // this chunk's filters and biases; the next chunk's move to the front
                    const uint2 wa = fwa[0], wb = fwb[0];
                    const uint32_t bab = fbias[0];
                    fwa[0] = fwa[1];
                    fwb[0] = fwb[1];
                    fbias[0] = fbias[1];
                    load_filters((c0 - 32 * eg) / 64 + 2, fwa[1], fwb[1], fbias[1]);
                    if (ok) {
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<float4*>(st + r * kStageLd + 4 * c) =
                                make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                    }
                    asm volatile("bar.sync %0, 128;" ::"r"(2 + eg) : "memory");
                    if (ok && lc + 1 < ncols && w_path) {
                        const float a0 = bf_lo_u(wa.x), a1 = bf_hi_u(wa.x), a2 = bf_lo_u(wa.y), a3 = bf_hi_u(wa.y);
                        const float b0 = bf_lo_u(wb.x), b1 = bf_hi_u(wb.x), b2 = bf_lo_u(wb.y), b3 = bf_hi_u(wb.y);
                        const float biasa = bf_lo_u(bab), biasb = bf_hi_u(bab);
                        // the window, rows wr0 - 3 .. wr0 + 15 of the staged chunk.  The top walk's rows
                        // -3..-1 lie before the group's staging rows (still inside the CTA's shared
                        // memory) and feed only its halo outputs, which are not stored.
                        const float* wbase = st + (wr0 - 3) * kStageLd + lc;
                        float2 xw[19];
#pragma unroll
                        for (int i = 0; i < 19; ++i) xw[i] = *reinterpret_cast<const float2*>(wbase + i * kStageLd);
                        // output i goes to row (i - w_ilo) from the first stored one
                        uint32_t* o = reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(cs.out) +
                                                                  (w_m0 + w_ilo) * cs.ldo + col + lc);
                        const int64_t step = cs.ldo / 2;  // output row pitch in bf16 pairs
                        if (w_path == 1) {
                            // every output's taps are rows of the window
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float oa = fmaf(a3, xw[i + 3].x, fmaf(a2, xw[i + 2].x, fmaf(a1, xw[i + 1].x, fmaf(a0, xw[i].x, biasa))));
                                float ob = fmaf(b3, xw[i + 3].y, fmaf(b2, xw[i + 2].y, fmaf(b1, xw[i + 1].y, fmaf(b0, xw[i].y, biasb))));
                                if (i >= w_ilo) o[(i - w_ilo) * step] = pack_bf16(silu_fast(oa), silu_fast(ob));
                            }
                        } else {
                            // A sequence whose first outputs reach into the history starts at output kst:
                            // up to 2 rows before the first stored output, or after it (one start at most:
                            // sequences are at least 19 tokens long).  Its history (the K-1 pre-conv values
                            // before its first token, oldest first) comes from the given conv state or is
                            // zero.
                            const int L = ex.L;
                            const int tpf = (w_tp0 + w_ilo) % L;
                            const int kst = tpf < 3 ? w_ilo - tpf : (L - tpf < w_ihi - w_ilo ? w_ilo + L - tpf : 16);
                            const int crow = cs.conv_row0 + col + lc;
                            float2 h0 = make_float2(0.f, 0.f), h1 = h0, h2 = h0;
                            const __nv_bfloat16* cin = static_cast<const __nv_bfloat16*>(ex.conv_state_in);
                            if (kst < 16 && cin) {
                                const __nv_bfloat16* ha = cin + (((w_m0 + kst) / L) * ex.conv_rows + crow) * 3;
                                h0 = make_float2(__bfloat162float(ha[0]), __bfloat162float(ha[3]));
                                h1 = make_float2(__bfloat162float(ha[1]), __bfloat162float(ha[4]));
                                h2 = make_float2(__bfloat162float(ha[2]), __bfloat162float(ha[5]));
                            }
                            // the three pre-conv values before output 0, oldest first
                            float2 p3 = xw[0], p2 = xw[1], p1 = xw[2];
                            if (kst == -1) {
                                p3 = h1;
                                p2 = h2;
                            } else if (kst == -2) {
                                p3 = h2;
                            }
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                if (i == kst) {
                                    p3 = h0;
                                    p2 = h1;
                                    p1 = h2;
                                }
                                const float2 cur = xw[i + 3];
                                float oa = fmaf(a3, cur.x, fmaf(a2, p1.x, fmaf(a1, p2.x, fmaf(a0, p3.x, biasa))));
                                float ob = fmaf(b3, cur.y, fmaf(b2, p1.y, fmaf(b1, p2.y, fmaf(b0, p3.y, biasb))));
                                if (i >= w_ilo && i < w_ihi) o[(i - w_ilo) * step] = pack_bf16(silu_fast(oa), silu_fast(ob));
                                p3 = p2;
                                p2 = p1;
                                p1 = cur;
                            }
                            __nv_bfloat16* cout = static_cast<__nv_bfloat16*>(ex.conv_state_out);
                            if (cout) {  // the last K-1 pre-conv inputs of each sequence ending in the walk
#pragma unroll
                                for (int sl = 0; sl < 3; ++sl) {
                                    const int i = ((L - 3 + sl - w_tp0) % L + L) % L;  // output at position L-3+sl
                                    if (i >= w_ilo && i < w_ihi) {
                                        const int64_t bq = (w_m0 + i) / L;
                                        const float2 xv = xat(wr0 + i, lc);
                                        cout[(bq * ex.conv_rows + crow) * 3 + sl] = __float2bfloat16_rn(xv.x);
                                        cout[(bq * ex.conv_rows + crow + 1) * 3 + sl] = __float2bfloat16_rn(xv.y);
                                    }
                                }
                            }
                        }
                    } else if (ok && lc < ncols && w_ihi > w_ilo) {
                        const int crow = cs.conv_row0 + col + lc;
                        const bool two = lc + 1 < ncols;
                        const __nv_bfloat16* cw = static_cast<const __nv_bfloat16*>(ex.conv_w);
                        const __nv_bfloat16* cbias = static_cast<const __nv_bfloat16*>(ex.conv_b);
                        const __nv_bfloat16* cin = static_cast<const __nv_bfloat16*>(ex.conv_state_in);
                        __nv_bfloat16* cout = static_cast<__nv_bfloat16*>(ex.conv_state_out);
                        const uint2 wa = *reinterpret_cast<const uint2*>(cw + (int64_t)crow * 4);
                        const uint2 wb = two ? *reinterpret_cast<const uint2*>(cw + (int64_t)(crow + 1) * 4) : wa;
                        const float a0 = bf_lo_u(wa.x), a1 = bf_hi_u(wa.x), a2 = bf_lo_u(wa.y), a3 = bf_hi_u(wa.y);
                        const float b0 = bf_lo_u(wb.x), b1 = bf_hi_u(wb.x), b2 = bf_lo_u(wb.y), b3 = bf_hi_u(wb.y);
                        const float biasa = __bfloat162float(cbias[crow]);
                        const float biasb = two ? __bfloat162float(cbias[crow + 1]) : 0.0f;
                        // window start: three rows above the block (inside the tile: rows >= 0)
                        const int r0 = wr0;
                        float xa3 = 0.f, xa2 = 0.f, xa1 = 0.f, xb3 = 0.f, xb2 = 0.f, xb1 = 0.f;
                        if (r0 >= 3) {
                            const float2 p3 = xat(r0 - 3, lc);
                            const float2 p2 = xat(r0 - 2, lc);
                            const float2 p1 = xat(r0 - 1, lc);
                            xa3 = p3.x; xb3 = p3.y; xa2 = p2.x; xb2 = p2.y; xa1 = p1.x; xb1 = p1.y;
                        }
                        int64_t m_r = (int64_t)t.mt * p.rows - p.shift + r0;  // token of row r0
                        int tp = (int)(((m_r % ex.L) + ex.L) % ex.L);          // its position in its sequence
#pragma unroll 4
                        for (int i = 0; i < 16; ++i, ++m_r) {
                            const int rr = r0 + i;
                            const float2 xv = xat(rr, lc);
                            if (tp == 0) {  // sequence start: history from the given state, or zeros
                                const int64_t bq = m_r / ex.L;
                                if (cin && m_r >= 0 && m_r < p.M) {
                                    const __nv_bfloat16* ha = cin + (bq * ex.conv_rows + crow) * 3;
                                    xa3 = __bfloat162float(ha[0]); xa2 = __bfloat162float(ha[1]);
                                    xa1 = __bfloat162float(ha[2]);
                                    if (two) {
                                        xb3 = __bfloat162float(ha[3]); xb2 = __bfloat162float(ha[4]);
                                        xb1 = __bfloat162float(ha[5]);
                                    }
                                } else {
                                    xa3 = xa2 = xa1 = xb3 = xb2 = xb1 = 0.0f;
                                }
                            }
                            if (rr >= p.shift && m_r < p.M) {
                                float oa = fmaf(a3, xv.x, fmaf(a2, xa1, fmaf(a1, xa2, fmaf(a0, xa3, biasa))));
                                float ob = fmaf(b3, xv.y, fmaf(b2, xb1, fmaf(b1, xb2, fmaf(b0, xb3, biasb))));
                                oa = silu_fast(oa);
                                ob = silu_fast(ob);
                                __nv_bfloat16* o = static_cast<__nv_bfloat16*>(cs.out) + m_r * cs.ldo + col + lc;
                                if (two) *reinterpret_cast<uint32_t*>(o) = pack_bf16(oa, ob);
                                else *o = __float2bfloat16_rn(oa);
                                // the new conv state: older entries shift in from the history first, then
                                // the sequence's own last inputs (this order also holds with the state
                                // updated in place)
                                if (cout && tp == 0 && ex.L < 3) {
                                    const int64_t bq = m_r / ex.L;
                                    for (int e = 0; e < 3 - ex.L; ++e) {
                                        const int64_t ba = (bq * ex.conv_rows + crow) * 3;
                                        cout[ba + e] = cin ? cin[ba + e + ex.L] : __float2bfloat16_rn(0.0f);
                                        if (two) cout[ba + 3 + e] = cin ? cin[ba + 3 + e + ex.L] : __float2bfloat16_rn(0.0f);
                                    }
                                }
                                if (cout && tp >= ex.L - 3) {  // last K-1 pre-conv inputs of the sequence
                                    const int64_t bq = m_r / ex.L;
                                    const int slot = tp - (ex.L - 3);
                                    cout[(bq * ex.conv_rows + crow) * 3 + slot] = __float2bfloat16_rn(xv.x);
                                    if (two) cout[(bq * ex.conv_rows + crow + 1) * 3 + slot] = __float2bfloat16_rn(xv.y);
                                }
                            }
                            xa3 = xa2; xa2 = xa1; xa1 = xv.x;
                            xb3 = xb2; xb2 = xb1; xb1 = xv.y;
                            tp = (tp + 1 == ex.L) ? 0 : tp + 1;
                        }
                    }
                    asm volatile("bar.sync %0, 128;" ::"r"(2 + eg) : "memory");  // the stage buffer is free again
                } else if (row_ok && ok) {
                    if (sg.out_f32) {
                        float* o = static_cast<float*>(sg.out) + m * sg.ldo + col;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < ncols) o[i] = sg.accumulate ? o[i] + v[i] : v[i];
                    } else {
                        store_bf16_chunk(static_cast<__nv_bfloat16*>(sg.out) + m * sg.ldo + col, ncols, sg.vec_ok, v);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_acc(buf);
        }
    }
    if (warp >= 2 && (warp & 3) == 2 && lane == 0) bulk_wait0();  // this group's bulk stores are complete
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();  // the pair's MMAs, loads and arrives are all done
    tc_fence_after();
    if (warp == 1) {
        if (PAIR) tmem_dealloc_pair(tmem, TMEM_COLS);
        else tmem_dealloc(tmem, TMEM_COLS);
    }
}

// --------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    // resolved once (the initialisation of a function-local static is thread-safe)
    static const EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

}  // namespace

// 2-D bf16 tensor map with a 128-byte swizzle: inner extent `inner` elements,
// `rows` rows `pitch` bytes apart, box of box_inner x box_rows.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch,
                    uint32_t box_inner, uint32_t box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 tensor map with a 128-byte swizzle (box_inner * 4 bytes must be 128).
static bool make_tmap_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch,
                          uint32_t box_inner, uint32_t box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor map with a 128-byte swizzle: extents {inner, rows, planes}, `pitch` bytes
// between rows and `plane_pitch` between planes, box of box_inner x box_rows x 1.  Rows past
// `rows` inside a plane are outside the tensor, so a box that overhangs a plane is clipped there
// (stores drop those rows) rather than reaching into the next plane.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t planes,
                       uint64_t pitch, uint64_t plane_pitch, uint32_t box_inner, uint32_t box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {inner, rows, planes};
    cuuint64_t strides[2] = {pitch, plane_pitch};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool tc_shape_ok(const GemmDesc& g)
{
    auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (g.M <= 0 || g.K <= 0 || g.nseg <= 0 || g.nseg > kMaxSeg) return false;
    if (g.K % 8 || g.lda % 8 || g.ldb % 8 || g.lda < g.K || g.ldb < g.K) return false;
    if (!al16(g.A)) return false;
    const char* base = static_cast<const char*>(g.seg[0].B);
    for (int s = 0; s < g.nseg; ++s) {
        const char* b = static_cast<const char*>(g.seg[s].B);
        if (b < base || (b - base) % (g.ldb * 2) || g.seg[s].n <= 0) return false;
        if (g.seg[s].accumulate && !g.seg[s].out_f32) return false;
        if (g.seg[s].kind == kEpiConv &&
            (g.ex.K != 4 || !g.ex.conv_w || !g.ex.conv_b || g.ex.L <= 0 || (reinterpret_cast<uintptr_t>(g.ex.conv_w) & 7u)))
            return false;
        if (g.seg[s].kind == kEpiSoftplus && (!g.ex.dt_bias || !g.seg[s].out_f32)) return false;
    }
    if (!al16(base)) return false;
    return true;
}

bool gemm_tc_supported(const GemmDesc& g) { return tc_shape_ok(g) && encode_fn() != nullptr; }

template <int BN, int STAGES, bool CONV, bool PAIR>
static cudaError_t launch_bn(const GemmDesc& g, const TcParams& p0, cudaStream_t s, int* status)
{
    TcParams p = p0;
    // Pair the conv columns of in_proj with the plain store columns of the same width: every
    // tile then drains half cheap stores and half conv walks, instead of alternating tiles whose
    // drains differ threefold (with two accumulators, the slow drains would hold up the MMAs).
    p.pair_tiles = 0;
    p.pair_a = p.pair_b = 0;
    if (CONV && BN == 256) {
        for (int a = 0; a < p.nseg && !p.pair_tiles; ++a)
            for (int b = 0; b < p.nseg; ++b)
                if (p.seg[a].kind == kEpiStore && !p.seg[a].out_f32 && !p.seg[a].accumulate &&
                    p.seg[b].kind == kEpiConv && p.seg[a].n == p.seg[b].n) {
                    p.pair_a = a;
                    p.pair_b = b;
                    p.pair_tiles = (p.seg[a].n + BN / 2 - 1) / (BN / 2);
                    break;
                }
    }
    p.ntiles = p.pair_tiles;
    for (int i = 0; i < p.nseg; ++i) {
        const bool in_pair = p.pair_tiles && (i == p.pair_a || i == p.pair_b);
        p.seg[i].ntiles = in_pair ? 0 : (p.seg[i].n + BN - 1) / BN;
        p.ntiles += p.seg[i].ntiles;
    }
    p.status = status;
    const char* base = static_cast<const char*>(g.seg[0].B);
    int64_t rows = 0;
    for (int i = 0; i < p.nseg; ++i) rows = max(rows, (int64_t)p.seg[i].b_row0 + p.seg[i].n);
    CUtensorMap mapA, mapB, mapB2;
    if (!make_tmap_bf16(&mapA, g.A, g.K, g.M, g.lda * 2, kBK, kBM)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&mapB, base, g.ldb, rows, g.ldb * 2, kBK, BN)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&mapB2, base, g.ldb, rows, g.ldb * 2, kBK, BN / 2)) return cudaErrorInvalidValue;
    OutMaps om;
    std::memset(&om, 0, sizeof(om));
    for (int i = 0; i < p.nseg; ++i) {  // plain outputs leave through bulk stores (fp32: or bulk adds)
        TcSeg& t = p.seg[i];
        t.tma = 0;
        if (t.kind != kEpiStore) continue;
        if (!t.out_f32 && !t.accumulate && t.vec_ok)
            t.tma = make_tmap_bf16(&om.m[i], t.out, (uint64_t)t.n, (uint64_t)g.M, (uint64_t)t.ldo * 2, 64, kBM) ? 1 : 0;
        else if (t.out_f32 && (reinterpret_cast<uintptr_t>(t.out) & 15u) == 0 && t.ldo % 4 == 0 &&
                 (p.shift == 0 || !t.accumulate))  // halo rows are written twice: never add them twice
            t.tma = make_tmap_f32(&om.m[i], t.out, (uint64_t)t.n, (uint64_t)g.M, (uint64_t)t.ldo * 4, 32, kBM)
                        ? (t.accumulate ? 3 : 2) : 0;
    }
    if (p.ksplit > 1 && p.seg[0].tma != 3) {  // K slices add their partials only through bulk adds
        p.ksplit = 1;
        p.kper = p.ktiles;
    }
    constexpr int smem = STAGES * (kBM + (PAIR ? BN / 2 : BN)) * kBK * 2 +
                         (CONV ? 2 * kBM * kStageLd * 4 : 2 * kBM * 128) + 1024 + 512;
    static_assert(smem <= 232448, "GEMM configuration exceeds 227 KB of shared memory");
    static_assert(!PAIR || BN == 256, "pairs run 256 x 256 MMAs");
    auto kernel = gemm_tc_kernel<BN, STAGES, CONV, PAIR>;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<unsigned long long> attr_set{0};  // one bit per device
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!(attr_set.load() >> dev & 1ull)) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(1ull << dev);
    }
    // one CTA per tile: the CTAs that start first take over the others' tiles as they go.  Pairs:
    // one cluster of two per pair of SMs, walking the tile pairs statically.
    int grid = p.mtiles * p.ntiles * p.ksplit;
    if (PAIR) {
        int sms = 148;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int pairs = ((p.mtiles + 1) / 2) * p.ntiles;
        grid = 2 * (pairs < sms / 2 ? pairs : sms / 2);
    }
    if (!p.pdl && !PAIR) {
        kernel<<<grid, 320, smem, s>>>(mapA, mapB, mapB2, om, p);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(320);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (p.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (PAIR) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, mapA, mapB, mapB2, om, p);
}

cudaError_t launch_gemm_tc(const GemmDesc& g, cudaStream_t s)
{
    TcParams p{};
    p.M = g.M;
    p.K = g.K;
    p.ktiles = (g.K + kBK - 1) / kBK;
    p.nseg = g.nseg;
    p.ex = g.ex;
    p.pdl = g.pdl;
    p.shift = 0;
    for (int i = 0; i < g.nseg; ++i)
        if (g.seg[i].kind == kEpiConv) p.shift = g.ex.K - 1;
    p.rows = kBM - p.shift;
    p.mtiles = (g.M + p.rows - 1) / p.rows;
    const char* base = static_cast<const char*>(g.seg[0].B);
    int n_total = 0;
    for (int i = 0; i < g.nseg; ++i) {
        const GemmSeg& sg = g.seg[i];
        TcSeg& t = p.seg[i];
        t.out = sg.out;
        t.ldo = sg.ldo;
        t.b_row0 = (int)((static_cast<const char*>(sg.B) - base) / (g.ldb * 2));
        t.n = sg.n;
        t.out_f32 = sg.out_f32;
        t.accumulate = sg.accumulate;
        t.vec_ok = !sg.out_f32 && (reinterpret_cast<uintptr_t>(sg.out) & 15u) == 0 && sg.ldo % 8 == 0;
        t.kind = sg.kind;
        t.conv_row0 = sg.conv_row0;
        n_total += sg.n;
    }
    int* status = device_status_ptr();
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // A 128 x 256 tile and a 128 x 128 one keep the tensor core equally busy per flop (an MMA of
    // N = 256 takes twice the cycles of one of N = 128), but the wide tile loads each A row once for
    // twice the columns.  Narrow tiles only when they take no more waves over the SMs than wide ones
    // (each SM then drains half as many columns).
    const int tiles256 = p.mtiles * ((n_total + 255) / 256);
    const int tiles128 = p.mtiles * ((n_total + 127) / 128);
    auto waves = [&](int t) { return (t + sms - 1) / sms; };
    const bool conv = p.shift > 0;
    bool wide = waves(tiles256) < waves(tiles128);
    // Too few tiles for the SMs and a long K: a single accumulating fp32 output splits K into
    // slices whose partial products add into it (bulk tensor adds, performed in L2).
    p.ksplit = 1;
    p.kper = p.ktiles;
    if (g.nseg == 1 && g.seg[0].out_f32 && g.seg[0].accumulate && g.seg[0].kind == kEpiStore && !conv &&
        tiles256 * 2 <= sms && p.ktiles >= 4) {
        wide = true;
        const int ks = min(sms / tiles256, p.ktiles / 2);  // at least two k-tiles per slice
        p.kper = (p.ktiles + ks - 1) / ks;
        p.ksplit = (p.ktiles + p.kper - 1) / p.kper;
    }
    // Wide tiles with a long enough K run on CTA pairs (measured on B200: the block's out_proj,
    // K = 1536, 40.1 -> 38.9 us, but slower with K = 192; in_proj with its conv drain, K = 2048,
    // 457 -> 420 us, but 105 -> 113 us with K = 768, where the pairs' static walk loses more to the
    // uneven drains than the halved B loads gain).
    if (wide && kUsePairs && p.ksplit == 1 && p.mtiles >= 2 && p.ktiles >= (conv ? 32 : 8))
        return conv ? launch_bn<256, 5, true, true>(g, p, s, status) : launch_bn<256, 6, false, true>(g, p, s, status);
    if (wide)
        return conv ? launch_bn<256, 3, true, false>(g, p, s, status)
                    : launch_bn<256, 4, false, false>(g, p, s, status);
    return conv ? launch_bn<128, 5, true, false>(g, p, s, status) : launch_bn<128, 6, false, false>(g, p, s, status);
}

}  // namespace mm

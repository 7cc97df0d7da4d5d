// C-ABI entry points: host-side validation, width views, workspace carving and
// launch sequences.  Every step of the computation runs in this library's
// kernels; nothing here computes on the host.
#include <atomic>
#include <cstring>
#include <mutex>

#include "mm_internal.cuh"

using namespace mm;

// Status word a kernel writes when a bounded wait gives up (one per device).
__device__ int g_mm_device_status;

namespace mm {
int* device_status_ptr()
{
    static std::atomic<int*> ptrs[64] = {};  // host threads may look it up at the same time
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int* ptr = ptrs[dev].load(std::memory_order_acquire);
    if (!ptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mm_device_status) != cudaSuccess) return nullptr;
        ptr = static_cast<int*>(p);
        ptrs[dev].store(ptr, std::memory_order_release);
    }
    return ptr;
}
}  // namespace mm

namespace {

constexpr size_t kAlign = 256;

size_t esize(int dtype) { return dtype == MM_BF16 ? 2 : 4; }

// Shape limits of the launches: sequences go on a grid's y or z dimension (at most 65535 of them per
// call), and the projections and scans index tokens (batch * L) with 32-bit rows.
constexpr int kMaxBatch = 65535;
bool batch_ok(int batch, int L)
{
    return batch > 0 && L > 0 && batch <= kMaxBatch && (int64_t)batch * L < (1ll << 31);
}
bool dtype_ok(int dtype) { return dtype == MM_F32 || dtype == MM_BF16; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// True when the byte ranges [a, a + na) and [b, b + nb) share a byte (null or empty ranges never do).
bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb)
{
    if (!a || !b || !na || !nb) return false;
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

// Sequential carving of the caller's workspace into 256-byte aligned pieces.
struct Carver {
    char* base;
    size_t used = 0;
    explicit Carver(void* b) : base(static_cast<char*>(b)) {}
    void* take(size_t bytes)
    {
        void* p = base ? base + used : nullptr;
        used += round_up(bytes);
        return p;
    }
};

struct View {  // resolved width view
    int Dm, E, P, N, G, GN, H, K, d, h, nconv, hpg;
};

int check_params(const mm_block_params* p)
{
    if (!p) return MM_ERR_NULL;
    if (!dtype_ok(p->dtype)) return MM_ERR_DTYPE;
    if (p->d_model <= 0 || p->d_inner <= 0 || p->d_head <= 0 || p->d_state <= 0 || p->ngroups <= 0) return MM_ERR_SHAPE;
    if (p->d_conv < 2 || p->d_conv > 8) return MM_ERR_SHAPE;
    if (p->d_inner % p->d_head) return MM_ERR_SHAPE;
    const int H = p->d_inner / p->d_head;
    if (H % p->ngroups) return MM_ERR_SHAPE;
    if (p->d_state > 256 || p->d_state % 8) return MM_ERR_SHAPE;
    if (!(p->norm_eps >= 0.0f)) return MM_ERR_SHAPE;
    const void* ptrs[] = {p->W_in, p->conv_w, p->conv_b, p->dt_bias, p->A, p->D, p->norm_w, p->W_out};
    for (const void* q : ptrs)
        if (!q) return MM_ERR_NULL;
    if (p->dtype == MM_BF16) {
        if (p->d_model % 8 || p->d_head % 8) return MM_ERR_SHAPE;
        const void* al[] = {p->W_in, p->W_out, p->norm_w};
        for (const void* q : al)
            if (!aligned16(q)) return MM_ERR_ALIGN;
    }
    return MM_OK;
}

int resolve(const mm_block_params* p, int m, View& v)
{
    int rc = check_params(p);
    if (rc) return rc;
    if (m <= 0 || m > p->d_model) return MM_ERR_INVALID_WIDTH;
    const long long num = (long long)p->d_inner * m;
    if (num % p->d_model) return MM_ERR_INVALID_WIDTH;
    const int d = (int)(num / p->d_model);
    if (d % p->d_head) return MM_ERR_INVALID_WIDTH;
    v.Dm = p->d_model; v.E = p->d_inner; v.P = p->d_head; v.N = p->d_state; v.G = p->ngroups;
    v.GN = v.G * v.N; v.H = v.E / v.P; v.K = p->d_conv; v.d = d; v.h = d / v.P; v.nconv = d + 2 * v.GN;
    v.hpg = v.H / v.G;
    return MM_OK;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;  // most recent CUDA error a call of this thread reported

inline int cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return MM_OK;
    g_last_cuda_error = e;
    return MM_ERR_CUDA;
}

// ------------------------------------------------------------------ tracing

struct TraceRec {
    const char* name;
    int kernels;
    cudaEvent_t start, stop;
};
struct Trace {
    TraceRec* recs = nullptr;
    int cap = 0, n = 0;
};
Trace g_trace;

// Runs one launch stage; with tracing on, brackets it with events on stream s.
template <class F>
cudaError_t stage(const char* name, int kernels, cudaStream_t s, F&& launch)
{
    if (!g_trace.recs || g_trace.n >= g_trace.cap) return launch();
    TraceRec& r = g_trace.recs[g_trace.n];
    cudaError_t e = cudaEventRecord(r.start, s);
    if (e != cudaSuccess) return e;
    e = launch();
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(r.stop, s);
    if (e != cudaSuccess) return e;
    r.name = name;
    r.kernels = kernels;
    ++g_trace.n;
    return cudaSuccess;
}
#define MM_TRY(expr)                          \
    do {                                      \
        int _rc = cuda_status(expr);          \
        if (_rc) return _rc;                  \
    } while (0)

cudaError_t run_gemm(int dtype, const GemmDesc& g, cudaStream_t s)
{
    if (dtype == MM_BF16 && gemm_tc_supported(g)) return launch_gemm_tc(g, s);
    return launch_gemm_simt(dtype, g, s);
}

bool scan_uses_tc(int dtype, const ScanArgs& a) { return dtype == MM_BF16 && scan_tc_supported(a); }

size_t scan_ws_bytes(int dtype, const ScanArgs& a) { return scan_uses_tc(dtype, a) ? scan_tc_workspace(a) : 0; }

int scan_kernels(int dtype, const ScanArgs& a) { return scan_uses_tc(dtype, a) ? scan_tc_kernel_count(a) : 1; }

cudaError_t run_scan(int dtype, const ScanArgs& a, void* ws, size_t ws_bytes, cudaStream_t s)
{
    if (scan_uses_tc(dtype, a)) return launch_scan_tc(a, ws, ws_bytes, s);
    return launch_scan_seq(dtype, a, s);
}

// Scan arguments of the block: x | B | C live in the post-conv buffer.
ScanArgs block_scan_args(const View& v, const mm_block_params* p, const void* xbc, const float* dt, int batch, int L,
                         int chunk, const float* s_in, float* s_out, void* y)
{
    ScanArgs a{};
    const size_t es = esize(p->dtype);
    a.x = xbc; a.sx = v.nconv;
    a.dt = dt; a.sdt = v.h;
    a.A = p->A;
    a.B = static_cast<const char*>(xbc) + (size_t)v.d * es; a.sB = v.nconv;
    a.C = static_cast<const char*>(xbc) + (size_t)(v.d + v.GN) * es; a.sC = v.nconv;
    a.D = p->D;
    a.batch = batch; a.L = L; a.h = v.h; a.P = v.P; a.N = v.N; a.G = v.G; a.hpg = v.hpg; a.chunk = chunk;
    a.init_state = s_in; a.state_stride = (int64_t)v.H * v.P * v.N;
    a.y = y; a.sy = v.d;
    a.final_state = s_out;
    return a;
}

struct BlockBufs {
    void *zxbc, *xbc, *y, *nrm, *scan_ws;
    float *dt_raw, *dt;
    size_t scan_ws_bytes;
};

BlockBufs carve_block(Carver& c, const View& v, const mm_block_params* p, int batch, int L, int chunk)
{
    const size_t es = esize(p->dtype);
    const size_t T = (size_t)batch * L;
    BlockBufs b{};
    b.zxbc = c.take(T * (v.d + v.nconv) * es);
    b.dt_raw = static_cast<float*>(c.take(T * v.h * 4));
    b.xbc = c.take(T * v.nconv * es);
    b.dt = static_cast<float*>(c.take(T * v.h * 4));
    b.y = c.take(T * v.d * es);
    b.nrm = c.take(T * v.d * es);
    ScanArgs probe = block_scan_args(v, p, b.xbc, b.dt, batch, L, chunk, nullptr, nullptr, b.y);
    b.scan_ws_bytes = scan_ws_bytes(p->dtype, probe);
    b.scan_ws = c.take(b.scan_ws_bytes);
    return b;
}

// in_proj through the width view: columns z | x | B | C go to zxbc, dt_raw to an fp32 buffer.
GemmDesc in_proj_desc(const View& v, const mm_block_params* p, const void* u, int64_t T, void* zxbc, float* dt_raw)
{
    const size_t es = esize(p->dtype);
    const char* W = static_cast<const char*>(p->W_in);
    char* Z = static_cast<char*>(zxbc);
    const int64_t ld = v.d + v.nconv;
    GemmDesc g{};
    g.A = u; g.lda = v.Dm; g.ldb = v.Dm; g.M = (int)T; g.K = v.Dm; g.nseg = 4;
    g.seg[0] = GemmSeg{W, Z, ld, v.d, 0, 0};
    g.seg[1] = GemmSeg{W + (size_t)v.E * v.Dm * es, Z + (size_t)v.d * es, ld, v.d, 0, 0};
    g.seg[2] = GemmSeg{W + (size_t)2 * v.E * v.Dm * es, Z + (size_t)2 * v.d * es, ld, 2 * v.GN, 0, 0};
    g.seg[3] = GemmSeg{W + (size_t)(2 * v.E + 2 * v.GN) * v.Dm * es, dt_raw, v.h, v.h, 1, 0};
    return g;
}

// out_proj through the K-prefix view W_out[:, 0:d] (row stride E).
GemmDesc out_proj_desc(const View& v, const mm_block_params* p, const void* nrm, int64_t T, void* out, int accumulate)
{
    GemmDesc g{};
    g.A = nrm; g.lda = v.d; g.ldb = v.E; g.M = (int)T; g.K = v.d; g.nseg = 1;
    g.seg[0] = GemmSeg{p->W_out, out, v.Dm, v.Dm, accumulate, accumulate};
    return g;
}

// ------------------------------------------------------------------ fused bf16 block
//
// in_proj applies conv + SiLU and softplus(dt) in its epilogue (pre-conv
// values stay in fp32 TMEM), the scan applies the SiLU(z) gate and norm_w and
// accumulates each token's sum of squares, and out_proj scales its rows by the
// resulting 1/RMS: three stages instead of six, no pre-conv or y round trip.

bool fused_ok(const mm_block_params* p, const View& v, int chunk)
{
    return p->dtype == MM_BF16 && v.K == 4 && v.P == 64 && v.N == 128 && chunk % 128 == 0 && v.Dm % 8 == 0 &&
           (reinterpret_cast<uintptr_t>(p->conv_w) & 7u) == 0 && (reinterpret_cast<uintptr_t>(p->norm_w) & 15u) == 0;
}

struct FusedBufs {
    void *z, *xbc, *nrm, *scan_ws;
    float *dt, *rowsq;
    size_t scan_ws_bytes;
};

FusedBufs carve_fused(Carver& c, const View& v, const mm_block_params* p, int batch, int L, int chunk)
{
    const size_t T = (size_t)batch * L;
    FusedBufs b{};
    b.z = c.take(T * v.d * 2);
    b.xbc = c.take(T * v.nconv * 2);
    b.dt = static_cast<float*>(c.take(T * v.h * 4));
    b.nrm = c.take(T * v.d * 2);
    b.rowsq = static_cast<float*>(c.take(T * 2 * v.h * 4));
    ScanArgs probe = block_scan_args(v, p, b.xbc, b.dt, batch, L, chunk, nullptr, nullptr, b.nrm);
    b.scan_ws_bytes = scan_tc_workspace(probe);
    b.scan_ws = c.take(b.scan_ws_bytes);
    return b;
}

GemmDesc in_proj_fused_desc(const View& v, const mm_block_params* p, const void* u, int batch, int L,
                            const FusedBufs& b, const void* c_in, void* c_out)
{
    const char* W = static_cast<const char*>(p->W_in);
    const size_t row = (size_t)v.Dm * 2;
    GemmDesc g{};
    g.A = u; g.lda = v.Dm; g.ldb = v.Dm; g.M = batch * L; g.K = v.Dm; g.nseg = 4;
    g.seg[0] = GemmSeg{W, b.z, v.d, v.d, 0, 0, kEpiStore, 0};
    g.seg[1] = GemmSeg{W + (size_t)v.E * row, b.xbc, v.nconv, v.d, 0, 0, kEpiConv, 0};
    g.seg[2] = GemmSeg{W + (size_t)2 * v.E * row, static_cast<char*>(b.xbc) + (size_t)v.d * 2, v.nconv, 2 * v.GN, 0, 0,
                       kEpiConv, v.E};
    g.seg[3] = GemmSeg{W + (size_t)(2 * v.E + 2 * v.GN) * row, b.dt, v.h, v.h, 1, 0, kEpiSoftplus, 0};
    g.ex.conv_w = p->conv_w; g.ex.conv_b = p->conv_b; g.ex.dt_bias = p->dt_bias;
    g.ex.L = L; g.ex.K = v.K; g.ex.conv_rows = v.E + 2 * v.GN;
    g.ex.conv_state_in = c_in; g.ex.conv_state_out = c_out;
    return g;
}

int block_impl_fused(const mm_block_params* p, const View& v, const void* u, int batch, int L, int chunk, void* out,
                     int out_accumulate, const float* s_in, const void* c_in, float* s_out, void* c_out, Carver& c,
                     cudaStream_t s)
{
    const int64_t T = (int64_t)batch * L;
    FusedBufs b = carve_fused(c, v, p, batch, L, chunk);
    const GemmDesc gin = in_proj_fused_desc(v, p, u, batch, L, b, c_in, c_out);
    MM_TRY(stage("in_proj_conv", 1, s, [&] { return launch_gemm_tc(gin, s); }));
    ScanArgs a = block_scan_args(v, p, b.xbc, b.dt, batch, L, chunk, s_in, s_out, b.nrm);
    ScanGate gate{b.z, v.d, p->norm_w, b.rowsq};
    MM_TRY(stage("ssd_scan_gate", scan_tc_kernel_count(a), s,
                 [&] { return launch_scan_tc_gated(a, gate, b.scan_ws, b.scan_ws_bytes, s); }));
    GemmDesc go = out_proj_desc(v, p, b.nrm, T, out, out_accumulate);
    go.ex.row_parts = b.rowsq;
    go.ex.nparts = 2 * v.h;
    go.ex.rs_inv_n = 1.0f / (float)v.d;
    go.ex.rs_eps = p->norm_eps;
    go.pdl = 1;  // out_proj may set up during the chunk scan's tail, then waits for it
    MM_TRY(stage("out_proj_norm", 1, s, [&] { return launch_gemm_tc(go, s); }));
    return MM_OK;
}

bool fused_supported(const mm_block_params* p, const View& v, int batch, int L, int chunk)
{
    if (!fused_ok(p, v, chunk)) return false;
    Carver c(nullptr);
    FusedBufs b = carve_fused(c, v, p, batch, L, chunk);
    // probe with an aligned stand-in for u (the entry points require 16-byte aligned u)
    const GemmDesc gin = in_proj_fused_desc(v, p, p->W_in, batch, L, b, nullptr, nullptr);
    ScanArgs a = block_scan_args(v, p, b.xbc, b.dt, batch, L, chunk, nullptr, nullptr, b.nrm);
    return gemm_tc_supported(gin) && scan_tc_supported(a);
}

size_t block_ws_bytes(const mm_block_params* p, const View& v, int batch, int L, int chunk)
{
    Carver c(nullptr);
    if (fused_supported(p, v, batch, L, chunk)) carve_fused(c, v, p, batch, L, chunk);
    else carve_block(c, v, p, batch, L, chunk);
    return c.used;
}

// The block on device buffers.  out_accumulate = 1: out is an fp32 buffer and
// the projection is added to it (residual stream of the stack).
int block_impl_unfused(const mm_block_params* p, const View& v, const void* u, int batch, int L, int chunk, void* out,
               int out_accumulate, const float* s_in, const void* c_in, float* s_out, void* c_out, Carver& c,
               cudaStream_t s)
{
    const int64_t T = (int64_t)batch * L;
    BlockBufs b = carve_block(c, v, p, batch, L, chunk);
    MM_TRY(stage("in_proj", 1, s, [&] { return run_gemm(p->dtype, in_proj_desc(v, p, u, T, b.zxbc, b.dt_raw), s); }));
    const int conv_rows = v.E + 2 * v.GN;
    MM_TRY(stage("conv_silu_dt", 1, s, [&] {
        return launch_conv_silu_dt(p->dtype, b.zxbc, v.d + v.nconv, v.d, b.dt_raw, p->conv_w, p->conv_b, p->dt_bias,
                                   v.E, v.d, v.nconv, v.h, v.K, batch, L, c_in, conv_rows, b.xbc, b.dt, s);
    }));
    if (c_out)
        MM_TRY(stage("conv_state", 1, s, [&] {
            return launch_conv_state_out(p->dtype, b.zxbc, v.d + v.nconv, v.d, v.E, v.d, v.nconv, v.K, batch, L, c_in,
                                         conv_rows, c_out, s);
        }));
    ScanArgs a = block_scan_args(v, p, b.xbc, b.dt, batch, L, chunk, s_in, s_out, b.y);
    MM_TRY(stage("ssd_scan", scan_kernels(p->dtype, a), s,
                 [&] { return run_scan(p->dtype, a, b.scan_ws, b.scan_ws_bytes, s); }));
    MM_TRY(stage("gate_rmsnorm", 1, s, [&] {
        return launch_gate_rmsnorm(p->dtype, b.y, v.d, b.zxbc, v.d + v.nconv, p->norm_w, p->norm_eps, v.d, (int)T,
                                   b.nrm, v.d, s);
    }));
    MM_TRY(stage("out_proj", 1, s,
                 [&] { return run_gemm(p->dtype, out_proj_desc(v, p, b.nrm, T, out, out_accumulate), s); }));
    return MM_OK;
}

int block_impl(const mm_block_params* p, const View& v, const void* u, int batch, int L, int chunk, void* out,
               int out_accumulate, const float* s_in, const void* c_in, float* s_out, void* c_out, Carver& c,
               cudaStream_t s)
{
    if (fused_supported(p, v, batch, L, chunk))
        return block_impl_fused(p, v, u, batch, L, chunk, out, out_accumulate, s_in, c_in, s_out, c_out, c, s);
    return block_impl_unfused(p, v, u, batch, L, chunk, out, out_accumulate, s_in, c_in, s_out, c_out, c, s);
}

int check_chunk(int chunk) { return chunk > 0 ? MM_OK : MM_ERR_SHAPE; }

}  // namespace

extern "C" {

const char* mm_status_string(int status)
{
    switch (status) {
        case MM_OK: return "ok";
        case MM_ERR_INVALID_WIDTH: return "invalid Matryoshka width";
        case MM_ERR_SHAPE: return "invalid shape or stride";
        case MM_ERR_DTYPE: return "invalid dtype";
        case MM_ERR_ALIGN: return "misaligned pointer or stride";
        case MM_ERR_WORKSPACE: return "workspace missing or too small";
        case MM_ERR_CUDA: return "CUDA runtime error";
        case MM_ERR_TIMEOUT: return "bounded device wait timed out";
        case MM_ERR_NULL: return "required pointer is NULL";
        case MM_ERR_UNSUPPORTED: return "unsupported configuration";
        default: return "unknown status";
    }
}

int mm_version(void) { return 100; }

const char* mm_last_cuda_error(void) { return cudaGetErrorName(g_last_cuda_error); }

int mm_device_status(void* stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MM_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_mm_device_status, sizeof(int)) != cudaSuccess) return MM_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(g_mm_device_status, &zero, sizeof(int)) != cudaSuccess) return MM_ERR_CUDA;
    return v;
}

int mm_width(const mm_block_params* p, int m_i, int* d_out, int* h_out)
{
    View v;
    int rc = resolve(p, m_i, v);
    if (rc) return rc;
    if (d_out) *d_out = v.d;
    if (h_out) *h_out = v.h;
    return MM_OK;
}

int matmamba_block_workspace(const mm_block_params* p, int batch, int L, int m_i, int chunk, size_t* bytes)
{
    View v;
    int rc = resolve(p, m_i, v);
    if (rc) return rc;
    if (!bytes) return MM_ERR_NULL;
    if (!batch_ok(batch, L)) return MM_ERR_SHAPE;
    if ((rc = check_chunk(chunk))) return rc;
    *bytes = block_ws_bytes(p, v, batch, L, chunk);
    return MM_OK;
}

int matmamba_block_fwd(const mm_block_params* p, const void* u, int batch, int L, int m_i, int chunk, void* out,
                       const float* ssm_state_in, const void* conv_state_in, float* ssm_state_out,
                       void* conv_state_out, void* workspace, size_t ws_bytes, void* stream)
{
    View v;
    int rc = resolve(p, m_i, v);
    if (rc) return rc;
    if (!u || !out) return MM_ERR_NULL;
    if (!batch_ok(batch, L)) return MM_ERR_SHAPE;
    if ((rc = check_chunk(chunk))) return rc;
    if (p->dtype == MM_BF16 && (!aligned16(u) || !aligned16(out))) return MM_ERR_ALIGN;
    // a state output may not share a byte with its input: CTAs write one sequence's output while
    // others still read their input
    const size_t ssm_bytes = (size_t)batch * v.H * v.P * v.N * 4;
    const size_t conv_bytes = (size_t)batch * (v.E + 2 * v.GN) * (v.K - 1) * esize(p->dtype);
    if (ranges_overlap(ssm_state_out, ssm_bytes, ssm_state_in, ssm_bytes) ||
        ranges_overlap(conv_state_out, conv_bytes, conv_state_in, conv_bytes))
        return MM_ERR_SHAPE;
    size_t need;
    matmamba_block_workspace(p, batch, L, m_i, chunk, &need);
    if (!workspace || ws_bytes < need) return MM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return MM_ERR_ALIGN;
    Carver c(workspace);
    return block_impl(p, v, u, batch, L, chunk, out, 0, ssm_state_in, conv_state_in, ssm_state_out, conv_state_out, c,
                      static_cast<cudaStream_t>(stream));
}

// Streams and events of the host-buffer entry point, created once per device (no device memory):
// copies in and out run on their own streams so that sub-batch i's compute overlaps the upload of
// sub-batch i+1 and the download of sub-batch i-1.
namespace {
constexpr int kMaxSub = 8;
struct HostPipe {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr, up[kMaxSub] = {}, comp[kMaxSub] = {};
    bool ready = false;
};
HostPipe g_pipes[64];
// Calls on one device take turns: they share that device's copy streams and events.
std::mutex g_pipe_mu[64];

cudaError_t host_pipe(HostPipe** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    HostPipe& hp = g_pipes[dev];
    if (!hp.ready) {
        const unsigned ef = cudaEventDisableTiming;
        if ((e = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&hp.start, ef)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&hp.done, ef)) != cudaSuccess) return e;
        for (int i = 0; i < kMaxSub; ++i) {
            if ((e = cudaEventCreateWithFlags(&hp.up[i], ef)) != cudaSuccess) return e;
            if ((e = cudaEventCreateWithFlags(&hp.comp[i], ef)) != cudaSuccess) return e;
        }
        hp.ready = true;
    }
    *out = &hp;
    return cudaSuccess;
}
}  // namespace

int matmamba_block_fwd_host(const mm_block_params* p, const void* u_host, int batch, int L, int m_i, int chunk,
                            void* out_host, void* u_dev, void* out_dev, void* workspace, size_t ws_bytes, void* stream)
{
    if (!u_host || !out_host || !u_dev || !out_dev) return MM_ERR_NULL;
    View v;
    int rc = resolve(p, m_i, v);
    if (rc) return rc;
    if (!batch_ok(batch, L)) return MM_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t row_bytes = (size_t)L * v.Dm * esize(p->dtype);  // one sequence of u or out
    size_t need;
    if ((rc = matmamba_block_workspace(p, batch, L, m_i, chunk, &need))) return rc;
    if (!workspace || ws_bytes < need) return MM_ERR_WORKSPACE;
    // sub-batches of whole sequences (sequences are independent); each must fit the workspace
    int nsub = batch < 4 ? batch : 4;
    for (; nsub > 1; --nsub) {
        const int per = (batch + nsub - 1) / nsub;
        size_t sub_need;
        if (!matmamba_block_workspace(p, per, L, m_i, chunk, &sub_need) && sub_need <= ws_bytes) break;
    }
    int dev = 0;
    MM_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return cuda_status(cudaErrorInvalidDevice);
    std::lock_guard<std::mutex> turn(g_pipe_mu[dev]);
    HostPipe* hp;
    MM_TRY(host_pipe(&hp));
    MM_TRY(cudaEventRecord(hp->start, s));  // earlier work on s (users of u_dev / out_dev) comes first
    MM_TRY(cudaStreamWaitEvent(hp->in, hp->start, 0));
    MM_TRY(cudaStreamWaitEvent(hp->out, hp->start, 0));
    const int per = (batch + nsub - 1) / nsub;
    for (int i = 0, b0 = 0; b0 < batch; ++i, b0 += per) {
        const int nb = batch - b0 < per ? batch - b0 : per;
        const size_t off = (size_t)b0 * row_bytes, bytes = (size_t)nb * row_bytes;
        char* ud = static_cast<char*>(u_dev) + off;
        char* od = static_cast<char*>(out_dev) + off;
        MM_TRY(cudaMemcpyAsync(ud, static_cast<const char*>(u_host) + off, bytes, cudaMemcpyHostToDevice, hp->in));
        MM_TRY(cudaEventRecord(hp->up[i], hp->in));
        MM_TRY(cudaStreamWaitEvent(s, hp->up[i], 0));
        rc = matmamba_block_fwd(p, ud, nb, L, m_i, chunk, od, nullptr, nullptr, nullptr, nullptr, workspace, ws_bytes,
                                stream);
        if (rc) {
            cudaStreamSynchronize(hp->in);
            cudaStreamSynchronize(s);
            cudaStreamSynchronize(hp->out);
            return rc;
        }
        MM_TRY(cudaEventRecord(hp->comp[i], s));
        MM_TRY(cudaStreamWaitEvent(hp->out, hp->comp[i], 0));
        MM_TRY(cudaMemcpyAsync(static_cast<char*>(out_host) + off, od, bytes, cudaMemcpyDeviceToHost, hp->out));
    }
    MM_TRY(cudaEventRecord(hp->done, hp->out));
    MM_TRY(cudaStreamWaitEvent(s, hp->done, 0));
    MM_TRY(cudaStreamSynchronize(s));
    return MM_OK;
}

static int scan_args_check(int dtype, const void* x, int64_t x_stride, const float* dt, int64_t dt_stride,
                           const float* A, const void* B, int64_t B_stride, const void* C, int64_t C_stride, int batch,
                           int L, int h, int P, int N, int G, int hpg, int chunk, int64_t state_stride, const void* y,
                           int64_t y_stride, bool need_state)
{
    if (!dtype_ok(dtype)) return MM_ERR_DTYPE;
    if (!x || !dt || !A || !B || !C || !y) return MM_ERR_NULL;
    if (!batch_ok(batch, L) || h <= 0 || P <= 0 || N <= 0 || G <= 0 || hpg <= 0) return MM_ERR_SHAPE;
    if (N > 256) return MM_ERR_SHAPE;
    if ((h - 1) / hpg >= G) return MM_ERR_SHAPE;
    if (x_stride < (int64_t)h * P || y_stride < (int64_t)h * P || dt_stride < h || B_stride < (int64_t)G * N ||
        C_stride < (int64_t)G * N)
        return MM_ERR_SHAPE;
    if (need_state && state_stride < (int64_t)h * P * N) return MM_ERR_SHAPE;
    if (chunk <= 0) return MM_ERR_SHAPE;
    if (dtype == MM_BF16) {
        if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(y)) return MM_ERR_ALIGN;
        if (x_stride % 8 || y_stride % 8 || B_stride % 8 || C_stride % 8) return MM_ERR_ALIGN;
    }
    return MM_OK;
}

static ScanArgs make_scan_args(const void* x, int64_t x_stride, const float* dt, int64_t dt_stride, const float* A,
                               const void* B, int64_t B_stride, const void* C, int64_t C_stride, const float* D,
                               int batch, int L, int h, int P, int N, int G, int hpg, int chunk,
                               const float* init_state, int64_t state_stride, void* y, int64_t y_stride,
                               float* final_state)
{
    ScanArgs a{};
    a.x = x; a.sx = x_stride; a.dt = dt; a.sdt = dt_stride; a.A = A; a.B = B; a.sB = B_stride; a.C = C;
    a.sC = C_stride; a.D = D; a.batch = batch; a.L = L; a.h = h; a.P = P; a.N = N; a.G = G; a.hpg = hpg;
    a.chunk = chunk; a.init_state = init_state; a.state_stride = state_stride; a.y = y; a.sy = y_stride;
    a.final_state = final_state;
    return a;
}

int ssd_scan_workspace(int dtype, int batch, int L, int h, int P, int N, int G, int chunk, size_t* bytes)
{
    if (!bytes) return MM_ERR_NULL;
    if (!dtype_ok(dtype)) return MM_ERR_DTYPE;
    if (!batch_ok(batch, L) || h <= 0 || P <= 0 || N <= 0 || G <= 0 || chunk <= 0) return MM_ERR_SHAPE;
    const int hpg = (h + G - 1) / G;
    ScanArgs a = make_scan_args(nullptr, (int64_t)h * P, nullptr, h, nullptr, nullptr, (int64_t)G * N, nullptr,
                                (int64_t)G * N, nullptr, batch, L, h, P, N, G, hpg, chunk, nullptr, (int64_t)h * P * N,
                                nullptr, (int64_t)h * P, nullptr);
    *bytes = round_up(scan_ws_bytes(dtype, a));
    return MM_OK;
}

int ssd_scan(int dtype, const void* x, int64_t x_stride, const float* dt, int64_t dt_stride, const float* A,
             const void* B, int64_t B_stride, const void* C, int64_t C_stride, const float* D, int batch, int L,
             int h, int P, int N, int G, int heads_per_group, int chunk, const float* init_state,
             int64_t state_stride, void* y, int64_t y_stride, float* final_state, void* workspace, size_t ws_bytes,
             void* stream)
{
    int rc = scan_args_check(dtype, x, x_stride, dt, dt_stride, A, B, B_stride, C, C_stride, batch, L, h, P, N, G,
                             heads_per_group, chunk, state_stride, y, y_stride, init_state || final_state);
    if (rc) return rc;
    {  // final_state may not share a byte with init_state (one CTA's output is another's input)
        const size_t st_bytes = ((size_t)(batch - 1) * state_stride + (size_t)h * P * N) * 4;
        if (ranges_overlap(final_state, st_bytes, init_state, st_bytes)) return MM_ERR_SHAPE;
    }
    ScanArgs a = make_scan_args(x, x_stride, dt, dt_stride, A, B, B_stride, C, C_stride, D, batch, L, h, P, N, G,
                                heads_per_group, chunk, init_state, state_stride, y, y_stride, final_state);
    const size_t need = scan_ws_bytes(dtype, a);
    if (need && (!workspace || ws_bytes < need)) return MM_ERR_WORKSPACE;
    if (need && reinterpret_cast<uintptr_t>(workspace) % kAlign) return MM_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return cuda_status(stage("ssd_scan", scan_kernels(dtype, a), s, [&] { return run_scan(dtype, a, workspace, ws_bytes, s); }));
}

int mm_linear(int dtype, const void* A, int64_t lda, int M, int K, const void* W, int64_t ldw, int N, void* out,
              int64_t ldo, int out_f32, int accumulate, void* stream)
{
    if (!dtype_ok(dtype)) return MM_ERR_DTYPE;
    if (!A || !W || !out) return MM_ERR_NULL;
    if (M < 0 || K <= 0 || N <= 0 || lda < K || ldw < K || ldo < N) return MM_ERR_SHAPE;
    if (accumulate && !out_f32) return MM_ERR_SHAPE;
    if (dtype == MM_F32 && !out_f32) out_f32 = 0;
    if (dtype == MM_BF16 && (!aligned16(A) || !aligned16(W) || lda % 8 || ldw % 8)) return MM_ERR_ALIGN;
    if (M == 0) return MM_OK;
    GemmDesc g{};
    g.A = A; g.lda = lda; g.ldb = ldw; g.M = M; g.K = K; g.nseg = 1;
    g.seg[0] = GemmSeg{W, out, ldo, N, out_f32 ? 1 : 0, accumulate ? 1 : 0};
    if (dtype == MM_F32) g.seg[0].out_f32 = 1;  // fp32 path: plain or accumulating fp32 stores
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return cuda_status(stage("linear", 1, s, [&] { return run_gemm(dtype, g, s); }));
}

// Buffers of one recurrent step in the caller's workspace.
struct StepBufs {
    void *zxbc, *xbc, *y, *nrm;
    float *dt_raw, *dt, *row_parts, *out32;
};

static StepBufs carve_step(Carver& c, const View& v, const mm_block_params* p, int batch)
{
    const size_t es = esize(p->dtype);
    StepBufs b{};
    b.zxbc = c.take((size_t)batch * (v.d + v.nconv) * es);
    b.dt_raw = static_cast<float*>(c.take((size_t)batch * v.h * 4));
    b.xbc = c.take((size_t)batch * v.nconv * es);
    b.dt = static_cast<float*>(c.take((size_t)batch * v.h * 4));
    b.y = c.take((size_t)batch * v.d * es);
    b.nrm = c.take((size_t)batch * v.d * es);
    b.row_parts = static_cast<float*>(c.take((size_t)batch * 2 * v.h * 4));
    b.out32 = static_cast<float*>(c.take((size_t)batch * v.Dm * 4));
    return b;
}

static size_t step_ws(const View& v, const mm_block_params* p, int batch)
{
    Carver c(nullptr);
    carve_step(c, v, p, batch);
    return c.used;
}

// The gate and norm fold into the step's scan and out_proj (bf16, d_head 64, d_state 128, 16-byte
// aligned state rows, tensor-core out_proj).  out_proj then adds its K slices (few rows, a long K)
// into an fp32 buffer with the 1/RMS row scale, which is rounded to the output afterwards.
static bool step_gated_ok(const View& v, const mm_block_params* p, const float* ssm_state, const GemmDesc& go)
{
    return p->dtype == MM_BF16 && v.P == 64 && v.N == 128 && (reinterpret_cast<uintptr_t>(ssm_state) & 15u) == 0 &&
           gemm_tc_supported(go);
}

int ssd_step_workspace(const mm_block_params* p, int batch, int m_i, size_t* bytes)
{
    View v;
    int rc = resolve(p, m_i, v);
    if (rc) return rc;
    if (!bytes) return MM_ERR_NULL;
    if (!batch_ok(batch, 1)) return MM_ERR_SHAPE;
    *bytes = step_ws(v, p, batch);
    return MM_OK;
}

int ssd_step(const mm_block_params* p, float* ssm_state, void* conv_state, const void* u_t, int batch, int m_i,
             void* out_t, void* workspace, size_t ws_bytes, void* stream)
{
    View v;
    int rc = resolve(p, m_i, v);
    if (rc) return rc;
    if (!ssm_state || !conv_state || !u_t || !out_t) return MM_ERR_NULL;
    if (!batch_ok(batch, 1)) return MM_ERR_SHAPE;
    if (p->dtype == MM_BF16 && (!aligned16(u_t) || !aligned16(out_t))) return MM_ERR_ALIGN;
    if (!workspace || ws_bytes < step_ws(v, p, batch)) return MM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return MM_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Carver c(workspace);
    const StepBufs b = carve_step(c, v, p, batch);
    MM_TRY(stage("step_in_proj", 1, s,
                 [&] { return run_gemm(p->dtype, in_proj_desc(v, p, u_t, batch, b.zxbc, b.dt_raw), s); }));
    MM_TRY(stage("step_conv_dt", 1, s, [&] {
        return launch_step_conv_dt(p->dtype, b.zxbc, v.d + v.nconv, v.d, b.dt_raw, p->conv_w, p->conv_b, p->dt_bias,
                                   v.E, v.d, v.nconv, v.h, v.K, batch, conv_state, v.E + 2 * v.GN, b.xbc, b.dt, s);
    }));
    GemmDesc go = out_proj_desc(v, p, b.nrm, batch, b.out32, 1);
    go.ex.row_parts = b.row_parts;
    go.ex.nparts = 2 * v.h;
    go.ex.rs_inv_n = 1.0f / (float)v.d;
    go.ex.rs_eps = p->norm_eps;
    if (step_gated_ok(v, p, ssm_state, go)) {
        MM_TRY(stage("step_scan_gate", 1, s, [&] {
            return launch_step_scan_gated(b.xbc, v.nconv, v.d, b.dt, p->A, p->D, ssm_state, v.H, v.h, v.GN, v.hpg,
                                          batch, b.zxbc, v.d + v.nconv, p->norm_w, b.nrm, b.row_parts, s);
        }));
        MM_TRY(stage("step_out_proj_norm", 2, s, [&] {
            cudaError_t e = cudaMemsetAsync(b.out32, 0, (size_t)batch * v.Dm * 4, s);
            if (e == cudaSuccess) e = launch_gemm_tc(go, s);
            if (e == cudaSuccess) e = launch_from_f32(p->dtype, b.out32, out_t, (int64_t)batch * v.Dm, s);
            return e;
        }));
        return MM_OK;
    }
    MM_TRY(stage("step_scan", 1, s, [&] {
        return launch_step_scan(p->dtype, b.xbc, v.nconv, v.d, b.dt, p->A, p->D, ssm_state, v.H, v.h, v.P, v.N, v.GN,
                                v.hpg, batch, b.y, s);
    }));
    MM_TRY(stage("step_gate_rmsnorm", 1, s, [&] {
        return launch_gate_rmsnorm(p->dtype, b.y, v.d, b.zxbc, v.d + v.nconv, p->norm_w, p->norm_eps, v.d, batch,
                                   b.nrm, v.d, s);
    }));
    MM_TRY(stage("step_out_proj", 1, s,
                 [&] { return run_gemm(p->dtype, out_proj_desc(v, p, b.nrm, batch, out_t, 0), s); }));
    return MM_OK;
}

static int stack_check(const mm_block_params* layers, int nlayers, const int* m_per_layer, int batch, int L, int chunk,
                       size_t* need)
{
    if (!layers || !m_per_layer) return MM_ERR_NULL;
    if (nlayers <= 0 || !batch_ok(batch, L)) return MM_ERR_SHAPE;
    int rc;
    if ((rc = check_chunk(chunk))) return rc;
    size_t block_max = 0;
    for (int l = 0; l < nlayers; ++l) {
        View v;
        if ((rc = resolve(&layers[l], m_per_layer[l], v))) return rc;
        if (layers[l].d_model != layers[0].d_model || layers[l].dtype != layers[0].dtype) return MM_ERR_SHAPE;
        const size_t need_l = block_ws_bytes(&layers[l], v, batch, L, chunk);
        block_max = need_l > block_max ? need_l : block_max;
    }
    const size_t T = (size_t)batch * L;
    const int Dm = layers[0].d_model;
    *need = round_up(T * Dm * 4) + round_up(T * Dm * esize(layers[0].dtype)) + block_max;
    return MM_OK;
}

int matmamba_stack_workspace(const mm_block_params* layers, int nlayers, const int* m_per_layer, int batch, int L,
                             int chunk, size_t* bytes)
{
    if (!bytes) return MM_ERR_NULL;
    return stack_check(layers, nlayers, m_per_layer, batch, L, chunk, bytes);
}

int matmamba_stack_fwd(const mm_block_params* layers, const void* const* prenorm_w, float prenorm_eps, int nlayers,
                       const int* m_per_layer, const void* u, int batch, int L, int chunk, void* out, void* workspace,
                       size_t ws_bytes, void* stream)
{
    size_t need;
    int rc = stack_check(layers, nlayers, m_per_layer, batch, L, chunk, &need);
    if (rc) return rc;
    if (!prenorm_w || !u || !out) return MM_ERR_NULL;
    for (int l = 0; l < nlayers; ++l)
        if (!prenorm_w[l]) return MM_ERR_NULL;
    if (!(prenorm_eps >= 0.0f)) return MM_ERR_SHAPE;
    if (!workspace || ws_bytes < need) return MM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return MM_ERR_ALIGN;
    const int dtype = layers[0].dtype;
    if (dtype == MM_BF16 && (!aligned16(u) || !aligned16(out))) return MM_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t T = (int64_t)batch * L;
    const int Dm = layers[0].d_model;
    Carver c(workspace);
    float* resid = static_cast<float*>(c.take((size_t)T * Dm * 4));
    void* normed = c.take((size_t)T * Dm * esize(dtype));
    const size_t block_base = c.used;
    MM_TRY(stage("stack_load", 1, s, [&] { return launch_to_f32(dtype, u, resid, T * Dm, s); }));
    for (int l = 0; l < nlayers; ++l) {
        View v;
        resolve(&layers[l], m_per_layer[l], v);
        MM_TRY(stage("prenorm", 1, s, [&] {
            return launch_rmsnorm_rows_f32in(dtype, resid, prenorm_w[l], prenorm_eps, Dm, (int)T, normed, s);
        }));
        c.used = block_base;
        if ((rc = block_impl(&layers[l], v, normed, batch, L, chunk, resid, 1, nullptr, nullptr, nullptr, nullptr, c,
                             s)))
            return rc;
    }
    MM_TRY(stage("stack_store", 1, s, [&] { return launch_from_f32(dtype, resid, out, T * Dm, s); }));
    return MM_OK;
}

int mm_trace_enable(int capacity)
{
    if (capacity < 0) return MM_ERR_SHAPE;
    if (g_trace.recs) {
        for (int i = 0; i < g_trace.cap; ++i) {
            cudaEventDestroy(g_trace.recs[i].start);
            cudaEventDestroy(g_trace.recs[i].stop);
        }
        delete[] g_trace.recs;
        g_trace = Trace{};
    }
    if (capacity == 0) return MM_OK;
    g_trace.recs = new TraceRec[capacity];
    g_trace.cap = capacity;
    for (int i = 0; i < capacity; ++i) {
        if (cudaEventCreate(&g_trace.recs[i].start) != cudaSuccess ||
            cudaEventCreate(&g_trace.recs[i].stop) != cudaSuccess) {
            g_trace.cap = i;
            mm_trace_enable(0);
            return MM_ERR_CUDA;
        }
    }
    return MM_OK;
}

int mm_trace_collect(mm_trace_entry* entries, int max_entries, int* n_entries, int* total_kernels)
{
    if (!entries || !n_entries) return MM_ERR_NULL;
    int n = 0, kern = 0;
    for (int i = 0; i < g_trace.n; ++i) {
        TraceRec& r = g_trace.recs[i];
        float ms = 0.0f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
            return MM_ERR_CUDA;
        kern += r.kernels;
        int j = 0;
        while (j < n && std::strncmp(entries[j].name, r.name, sizeof(entries[j].name) - 1) != 0) ++j;
        if (j == n) {
            if (n >= max_entries) continue;
            std::memset(&entries[n], 0, sizeof(entries[n]));
            std::strncpy(entries[n].name, r.name, sizeof(entries[n].name) - 1);
            ++n;
        }
        entries[j].stages += 1;
        entries[j].kernels += r.kernels;
        entries[j].total_ms += ms;
    }
    g_trace.n = 0;
    *n_entries = n;
    if (total_kernels) *total_kernels = kern;
    return MM_OK;
}

}  // extern "C"

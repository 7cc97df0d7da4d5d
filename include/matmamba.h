/*
 * matmamba.h -- C ABI of the MatMamba block library for NVIDIA B200 (sm_100a).
 *
 * The library evaluates the MatMamba block ("MatMamba: A Matryoshka State
 * Space Model", block-definition and nested sub-block paragraphs): a Mamba2
 * block whose inner width, heads and per-head parameters are cut to a prefix
 * chosen per call by the Matryoshka width m_i.  One set of full-width weights
 * serves every width; a width is a strided view of those weights, never a
 * copy.
 *
 * Conventions shared by every entry point
 *  - All tensors are row-major.  Device pointers unless stated otherwise.
 *  - The caller owns all memory.  The library allocates nothing; scratch
 *    space is a caller-provided device workspace whose size comes from the
 *    matching *_workspace query (256-byte aligned pointer required).
 *  - Calls are asynchronous on the given CUDA stream (a cudaStream_t passed
 *    as void*, NULL = legacy default stream).  Output buffers must not alias
 *    inputs unless a parameter says so.
 *  - Limits per call: at most 65535 sequences (batch) and fewer than 2^31
 *    tokens (batch * L); larger calls return MM_ERR_SHAPE.
 *  - Every call returns an mm_status.  Shapes, widths, dtypes, alignment and
 *    workspace size are checked on the host before anything is launched; a
 *    rejected call launches nothing and leaves every buffer untouched.
 *    MM_ERR_CUDA reports a launch or runtime error from the CUDA runtime.
 *  - dtype MM_BF16 runs the tensor-core path (bf16 storage, fp32
 *    accumulation and fp32 scan state); MM_F32 runs an fp32 CUDA-core path
 *    (fp32 storage and arithmetic throughout).
 *  - Host threads: entry points may be called from several host threads at
 *    once.  Calls that share a buffer (a workspace, a state, an output) must
 *    be ordered by the caller, as for any two kernels; matmamba_block_fwd_host
 *    calls on one device take turns by themselves; tracing (mm_trace_*) is
 *    for one host thread.
 *  - Symbols: d_model = D_m, E = d_inner, P = d_head, N = d_state,
 *    G = ngroups, GN = G*N, H = E/P heads, K = d_conv.  At width m:
 *    d = E*m/D_m channels, h = d/P heads, nconv = d + 2*GN conv channels.
 */
#ifndef MATMAMBA_H
#define MATMAMBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MM_OK = 0,
    MM_ERR_INVALID_WIDTH = 1, /* m_i is not a valid Matryoshka width            */
    MM_ERR_SHAPE = 2,         /* a size or stride is out of range               */
    MM_ERR_DTYPE = 3,         /* unknown dtype                                   */
    MM_ERR_ALIGN = 4,         /* a pointer or stride breaks the stated alignment */
    MM_ERR_WORKSPACE = 5,     /* workspace NULL or smaller than the query        */
    MM_ERR_CUDA = 6,          /* CUDA runtime reported an error                  */
    MM_ERR_TIMEOUT = 7,       /* a bounded device-side wait gave up              */
    MM_ERR_NULL = 8,          /* a required pointer is NULL                      */
    MM_ERR_UNSUPPORTED = 9    /* valid shape with no kernel in this build        */
} mm_status;

typedef enum { MM_F32 = 0, MM_BF16 = 1 } mm_dtype;

/*
 * Full-width parameters of one block.  Pointers are device pointers to
 * contiguous row-major arrays of the given shapes; weights marked "dtype" are
 * stored in params.dtype, the per-head vectors always in fp32.
 *   W_in   (2E + 2GN + H, D_m) dtype   rows in the order z | x | B | C | dt
 *   conv_w (E + 2GN, K)        dtype   rows x | B | C; tap K-1 multiplies the
 *                                      current token (cross-correlation)
 *   conv_b (E + 2GN)           dtype
 *   dt_bias, A, D (H)          fp32    A holds the (negative) decay rates
 *   norm_w (E)                 dtype   RMSNorm weight
 *   W_out  (D_m, E)            dtype
 * The width-m view uses W_in rows [0,d) u [E,E+d) u [2E,2E+2GN) u
 * [2E+2GN, 2E+2GN+h), conv rows [0,d) u [E,E+2GN), entries [0,h) of the
 * per-head vectors, norm_w[0,d) and columns [0,d) of W_out (nested sub-block
 * paragraph: (d_inner, .) parameters keep their first d_i rows, (n_heads)
 * parameters their first h_i entries; B and C do not depend on d_inner and
 * stay whole).
 * Requirements (else MM_ERR_SHAPE / MM_ERR_ALIGN / MM_ERR_NULL before any
 * launch): E % P == 0, H % G == 0, 2 <= K <= 8, N % 8 == 0, N <= 256,
 * norm_eps >= 0, no null weight pointer; bf16 also needs D_m % 8 == 0,
 * P % 8 == 0 and W_in, W_out, norm_w 16-byte aligned.  A valid width m has
 * 0 < m <= D_m, E*m divisible by D_m and d = E*m/D_m divisible by P
 * (MM_ERR_INVALID_WIDTH otherwise).
 * Which kernels run: bf16 blocks with K == 4, P == 64, N == 128, chunk a
 * multiple of 128, conv_w 8-byte and norm_w 16-byte aligned take the fused
 * tensor-core path (in_proj + conv + dt in one GEMM, scan + gate, out_proj +
 * 1/RMS); everything else takes the unfused path: separate conv, gate and
 * norm kernels on CUDA cores, with the tensor-core GEMM and scan where their
 * shape rules hold (bf16) and CUDA-core GEMM and scan otherwise.
 */
typedef struct mm_block_params {
    int d_model;
    int d_inner;
    int d_head;
    int d_state;
    int ngroups;
    int d_conv;
    int dtype;      /* mm_dtype */
    float norm_eps; /* RMSNorm epsilon (added to the mean square) */
    const void* W_in;
    const void* conv_w;
    const void* conv_b;
    const float* dt_bias;
    const float* A;
    const float* D;
    const void* norm_w;
    const void* W_out;
} mm_block_params;

/* Human-readable name of a status code (static string, never NULL). */
const char* mm_status_string(int status);

/* Name of the most recent CUDA error behind an MM_ERR_CUDA returned to the
 * calling host thread ("cudaSuccess" if none). */
const char* mm_last_cuda_error(void);

/* Library version: major*10000 + minor*100 + patch. */
int mm_version(void);

/*
 * Device-side status of the current device: synchronizes `stream`, returns
 * MM_OK, or MM_ERR_TIMEOUT if a kernel's bounded wait (at most about two
 * seconds on one barrier) gave up since the last call, and clears the word.
 * Kernels never trap; a timed-out kernel skips its remaining work and exits,
 * so its outputs are then undefined.
 */
int mm_device_status(void* stream);

/*
 * Width rule (nested sub-block paragraph; Mix'n'Match paragraph: any m_i that
 * gives an integer number of heads is valid).  Host only.
 * Valid iff 0 < m_i <= D_m, E*m_i divisible by D_m, and d = E*m_i/D_m
 * divisible by P.  On success writes d and h (either pointer may be NULL).
 */
int mm_width(const mm_block_params* p, int m_i, int* d_out, int* h_out);

/* Workspace bytes for matmamba_block_fwd with these arguments.  Host only. */
int matmamba_block_workspace(const mm_block_params* p, int batch, int L, int m_i, int chunk, size_t* bytes);

/*
 * Forward pass of the block at width m_i ("MatMamba: A Matryoshka State Space
 * Model", block-definition paragraph and nested sub-block paragraph):
 *   [z | x | B | C | r] = W_in-view . u_t
 *   x,B,C <- SiLU(causal depthwise conv, K taps, + conv_b)
 *   dt = softplus(r + dt_bias)
 *   H_t = exp(dt A) H_{t-1} + dt B_t x_t^T,  y_t = C_t^T H_t + D x_t  (per head)
 *   n = RMSNorm(y * SiLU(z)) * norm_w[0:d];  out_t = W_out[:, 0:d] . n_t
 *   u    (batch, L, D_m) dtype      out (batch, L, D_m) dtype
 *   chunk: block length of the chunked scan (positive; the result does not
 *          depend on it beyond rounding; the bf16 path needs a multiple of 128
 *          and evaluates 128-token sub-blocks, the fp32 path scans
 *          sequentially)
 *   ssm_state_in  (batch, H, P, N) fp32 or NULL (zero initial state)
 *   conv_state_in (batch, E + 2GN, K-1) dtype or NULL (zero history); entry
 *                 [.., k] is the pre-conv input k-(K-1) tokens before u[:,0]
 *   ssm_state_out, conv_state_out: same shapes, or NULL.  Only heads [0,h)
 *                 and conv rows [0,d) u [E,E+2GN) are written; every other
 *                 byte keeps its previous contents.  *_out must not alias
 *                 *_in.
 * L >= 1, batch >= 1.
 */
int matmamba_block_fwd(const mm_block_params* p, const void* u, int batch, int L, int m_i, int chunk, void* out,
                       const float* ssm_state_in, const void* conv_state_in, float* ssm_state_out,
                       void* conv_state_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Same computation with u and out in HOST memory: copies u to u_dev, runs
 * matmamba_block_fwd, copies out_dev back to out_host and waits.  u_dev and
 * out_dev are caller-owned device buffers of the same shapes.  The batch is
 * cut into up to four sub-batches of whole sequences (sequences are
 * independent; a sub-batch may take another scan schedule, so results match
 * a single call up to rounding): sub-batch i computes on
 * `stream` while sub-batch i+1 is uploaded and sub-batch i-1 downloaded on two
 * copy streams the library creates once per device, so with pinned host
 * buffers the transfers in both directions overlap the compute.  The call
 * orders itself after earlier work on `stream` and returns once out_host
 * holds the result.  Calls on one device from several host threads take
 * turns (they share that device's copy streams).
 */
int matmamba_block_fwd_host(const mm_block_params* p, const void* u_host, int batch, int L, int m_i, int chunk,
                            void* out_host, void* u_dev, void* out_dev, void* workspace, size_t ws_bytes,
                            void* stream);

/*
 * Projection primitive used for in_proj and out_proj: out[m, n] (+)=
 * sum_k A[m, k] * W[n, k] for m < M, n < N, k < K.  A (M rows, pitch lda)
 * and W (N rows, pitch ldw) are K-major in `dtype`.  out has pitch ldo and
 * holds fp32 when out_f32 != 0 (bf16 inputs only; accumulate != 0 then adds
 * to it), else `dtype`.  bf16 runs on the tensor cores when the operands are
 * 16-byte aligned with pitches that are multiples of 8 elements.
 */
int mm_linear(int dtype, const void* A, int64_t lda, int M, int K, const void* W, int64_t ldw, int N, void* out,
              int64_t ldo, int out_f32, int accumulate, void* stream);

/* Workspace bytes for ssd_scan.  Host only. */
int ssd_scan_workspace(int dtype, int batch, int L, int h, int P, int N, int G, int chunk, size_t* bytes);

/*
 * Selective scan alone ("chunk + selective scan" of the block-definition
 * paragraph), with the D skip term:
 *   H_t = exp(dt_t A_i) H_{t-1} + dt_t B_t x_t^T,  y_t = C_t^T H_t + D_i x_t
 * for heads i in [0,h), head i reading group i / heads_per_group.
 * Element addresses (tokens flattened as tok = b*L + t):
 *   x[tok*x_stride + i*P + p]      dtype    (x_stride >= h*P)
 *   dt[tok*dt_stride + i]          fp32     already through softplus, > 0
 *   B[tok*B_stride + g*N + n], C[tok*C_stride + g*N + n]  dtype
 *   y[tok*y_stride + i*P + p]      dtype
 *   A, D: (>= h) fp32; D may be NULL (no skip term)
 *   init_state, final_state: fp32 [b*state_stride + (i*P + p)*N + n], each
 *   may be NULL (zero initial state / not returned); state_stride >= h*P*N.
 * chunk as for matmamba_block_fwd.  bf16 strides must be multiples of 8
 * elements and the base pointers 16-byte aligned.
 */
int ssd_scan(int dtype, const void* x, int64_t x_stride, const float* dt, int64_t dt_stride, const float* A,
             const void* B, int64_t B_stride, const void* C, int64_t C_stride, const float* D, int batch, int L,
             int h, int P, int N, int G, int heads_per_group, int chunk, const float* init_state,
             int64_t state_stride, void* y, int64_t y_stride, float* final_state, void* workspace,
             size_t ws_bytes, void* stream);

/*
 * ssd_scan without a workspace argument, for callers that cannot allocate
 * device memory around a call: an engine whose allocator owns all device
 * memory from start-up, a plugin handed only its input and output buffers, or
 * a latency-critical loop that must avoid the device-wide synchronisation
 * cudaMalloc / cudaFree may cause.  The paper has no counterpart; it is a
 * deployment convenience of this library.
 * Same arguments and results as ssd_scan.  Scratch comes from a fixed device
 * array of MM_SCAN_STATIC_SCRATCH_BYTES inside the library (held by every GPU
 * that loads it, until exit); a call whose scan needs more than that (its
 * ssd_scan_workspace figure for the same arguments) returns MM_ERR_WORKSPACE
 * and launches nothing.  Allocates nothing itself.
 * All calls on a device share the array and it keeps the last call's
 * contents (the scan writes every scratch byte before reading it): calls that
 * overlap on the GPU race and must be serialised by the caller.  The first
 * call on a device looks up the array's device address and caches it; make
 * that first call before any stream capture.
 */
#define MM_SCAN_STATIC_SCRATCH_BYTES ((size_t)32 << 20) /* 32 MiB per device */

int ssd_scan_static(int dtype, const void* x, int64_t x_stride, const float* dt, int64_t dt_stride, const float* A,
                    const void* B, int64_t B_stride, const void* C, int64_t C_stride, const float* D, int batch,
                    int L, int h, int P, int N, int G, int heads_per_group, int chunk, const float* init_state,
                    int64_t state_stride, void* y, int64_t y_stride, float* final_state, void* stream);

/*
 * Failure-path self-test (no counterpart in the paper): launches one CTA that
 * waits on an mbarrier nothing arrives on, through the same bounded wait the
 * tensor-core kernels use, with a limit of timeout_us microseconds (1 ..
 * 1,000,000).  The wait gives up, the kernel records MM_ERR_TIMEOUT in the
 * device status word and returns; mm_device_status then reports it (and
 * clears it) and the context stays usable.  Returns MM_ERR_SHAPE for a limit
 * out of range, MM_ERR_CUDA if the launch fails, else MM_OK.
 */
int mm_selftest_wait_timeout(unsigned timeout_us, void* stream);

/* Workspace bytes for ssd_step.  Host only. */
int ssd_step_workspace(const mm_block_params* p, int batch, int m_i, size_t* bytes);

/*
 * One recurrent token of the block at width m_i for every sequence (linear-
 * time recurrent inference, "Mamba: Linear-Time Sequence Modeling with
 * Selective State Spaces", summary page):
 *   u_t (batch, D_m) dtype -> out_t (batch, D_m) dtype
 *   ssm_state  (batch, H, P, N) fp32, in/out
 *   conv_state (batch, E + 2GN, K-1) dtype, in/out, oldest tap first; the
 *              step rolls it by one token.
 * Only heads [0,h) and conv rows [0,d) u [E,E+2GN) are read or written.
 * Equals matmamba_block_fwd on one token with the same states.
 */
int ssd_step(const mm_block_params* p, float* ssm_state, void* conv_state, const void* u_t, int batch, int m_i,
             void* out_t, void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes for matmamba_stack_fwd.  Host only. */
int matmamba_stack_workspace(const mm_block_params* layers, int nlayers, const int* m_per_layer, int batch, int L,
                             int chunk, size_t* bytes);

/*
 * Stacked model ("MatMamba: A Matryoshka State Space Model", stacking
 * paragraph) with a pre-norm residual: for l in [0, nlayers)
 *   u <- u + block_l(RMSNorm(u) * prenorm_w[l], m_per_layer[l])
 * with no final norm.  layers: host array of nlayers parameter sets (same
 * dims and dtype); prenorm_w: host array of nlayers device pointers to
 * (D_m) weights in that dtype; m_per_layer: host array of widths (one per
 * layer: a single width or a Mix'n'Match choice).  The residual stream is
 * kept in fp32 in the workspace; out (batch, L, D_m) dtype.
 */
int matmamba_stack_fwd(const mm_block_params* layers, const void* const* prenorm_w, float prenorm_eps,
                       int nlayers, const int* m_per_layer, const void* u, int batch, int L, int chunk, void* out,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * Tracing.  While enabled, every launch stage of the library (one named
 * step such as "in_proj" or "ssd_scan", which may be several kernels) records
 * a CUDA event before and after itself on the stream it runs on.  Events are
 * created with cudaEventCreate (no device memory).  Single host thread only.
 *   mm_trace_enable(capacity): capacity > 0 starts a trace holding up to that
 *     many stages (older entries are kept, later ones dropped); 0 stops and
 *     frees it.
 *   mm_trace_collect: synchronizes on the recorded events and writes per-name
 *     totals (at most max_entries) and the number of kernels launched.
 *     The trace is then cleared and stays enabled.
 */
typedef struct mm_trace_entry {
    char name[32];
    int stages;      /* traced stages with this name           */
    int kernels;     /* kernel launches inside those stages     */
    double total_ms; /* sum of event-to-event times             */
} mm_trace_entry;

int mm_trace_enable(int capacity);
int mm_trace_collect(mm_trace_entry* entries, int max_entries, int* n_entries, int* total_kernels);

#ifdef __cplusplus
}
#endif

#endif /* MATMAMBA_H */

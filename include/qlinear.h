/*
 * qlinear.h -- C ABI of libqlinear.so: forward pass y = W x of a weight-only
 * low-bit quantized linear layer whose W stays compressed in device memory and
 * is decoded on the fly by sm_100a (B200) kernels.
 *
 * Two weight formats:
 *
 *  BenQ 6-bit ("Qwen3.8-27B -- BenQ 6-bit", section "What BenQ stores"):
 *    every weight is a 6-bit code (1 sign bit + 5 magnitude-tier bits) indexing
 *    its output row's own table of 64 signed bf16 magnitudes; decode is exactly
 *    lut.gather(1, codes).  Codes are packed 4 per 3 bytes (the card's
 *    "packing to 6-bit" remark made concrete): code k of a row occupies bits
 *    [6k, 6k+6) of the row's little-endian bitstream, bit q of the stream being
 *    bit q%8 of byte q/8.  W is N x K (out x in).
 *
 *  MDBF ("MDBF (Multi-Envelope Double Binary Factorization)", section
 *    "Algorithm"): W ~= sum_p F_p G_p with F = S_A (.) (A_amp Q_U^T) and
 *    G = S_B (.) (Q_V B_amp^T); S_A (n x r) and S_B (r x m) are +-1 matrices
 *    stored one bit per element (LSB first along each row, bit 1 = +1, rows
 *    padded to a byte stride; padding bits are ignored), the four envelopes are
 *    fp16.  W is n x m (out x in).
 *
 * Conventions shared by every entry point
 *  - Pointers named as device pointers are caller-owned device memory.  The
 *    library never allocates, frees or keeps them.  Host pointers are read
 *    during the call only.
 *  - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t;
 *    NULL is the legacy default stream).  No call synchronizes the device.
 *  - Activations x are bf16, row-major [B][K] (BenQ) or [B][m] (MDBF).  Outputs
 *    y are row-major [B][N] / [B][n], fp32 or bf16 (round-to-nearest-even of the
 *    fp32 result) as chosen by `y_dtype`; accumulation is always fp32.
 *  - Argument errors are detected on the host before any launch and return
 *    QL_ERR_INVALID_ARG, QL_ERR_UNSUPPORTED or QL_ERR_ALIGNMENT with nothing
 *    launched; a failed launch returns QL_ERR_CUDA.  ql_last_error() gives a
 *    message for the calling thread's last non-OK status.
 *  - Device-side waits in the pipelined kernels are bounded.  A wait that runs
 *    out sets a device-side flag and the kernel returns early (its output is
 *    then undefined); ql_check() reports it as QL_ERR_TIMEOUT.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QL_API __attribute__((visibility("default")))
#else
#define QL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ql_stream_t; /* same object as cudaStream_t */

typedef enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1, /* null pointer, non-positive or inconsistent size */
  QL_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement    */
  QL_ERR_ALIGNMENT = 3,   /* a pointer or stride breaks a stated alignment    */
  QL_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed             */
  QL_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out               */
} ql_status;

typedef enum { QL_OUT_F32 = 0, QL_OUT_BF16 = 1 } ql_out_dtype;

/* ---------------------------------------------------------------- BenQ ----- */

/*
 * benq_linear -- y[b][n] = sum_k lut[n][code(n,k)] * x[b][k]
 *   ("What BenQ stores": decode is lut.gather(1, codes), fused here into the
 *   contraction so the decoded W is never written to memory).
 *
 *   codes  device, uint8 [N][3K/4]: packed codes, row stride exactly 3K/4 bytes.
 *   lut    device, bf16 bits [N][64]: row n's table; entry c is the value of code c.
 *   x      device, bf16 bits [B][K].
 *   y      device, [B][N] of y_dtype; fully overwritten.
 *   B, N, K  batch rows, output features, input features.  K % 4 == 0.
 *
 *   B <= 16 runs the decode GEMV (one pass over the codes, bandwidth bound);
 *   B > 16 runs the tensor-core GEMM (tcgen05, W tiles decoded into shared
 *   memory), which needs K % 64 == 0 and N % 256 == 0 (else QL_ERR_UNSUPPORTED).
 *   Alignment: codes, lut, x, y 16-byte aligned (QL_ERR_ALIGNMENT otherwise).
 */
QL_API ql_status benq_linear(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y,
                      ql_out_dtype y_dtype, int B, int N, int K, ql_stream_t stream);

/*
 * benq_linear_ws -- benq_linear with a caller workspace for the GEMM's last
 *   wave.  No counterpart in the pages: this is scheduling.  The GEMM runs whole
 *   output tiles in waves over the SM pairs; when the last wave would leave at
 *   least half of them idle, it splits each of its tiles into up to 8 K ranges,
 *   writes fp32 partials to `workspace` and sums them in a fixed order (results
 *   are deterministic and, for a given device, independent of the stream).
 *   Results equal benq_linear's up to fp32 summation order.
 *
 *   workspace  device, 256-byte aligned, ws_bytes >= benq_linear_workspace_bytes
 *              (B, N, K) to enable the split; NULL with ws_bytes == 0 runs exactly
 *              benq_linear.  A smaller non-NULL workspace also runs without the
 *              split.  Owned by the caller; must not be used by another call
 *              running at the same time.  Other arguments as benq_linear.
 *   Errors: QL_ERR_INVALID_ARG if only one of workspace / ws_bytes is set,
 *   QL_ERR_ALIGNMENT if the workspace is not 256-byte aligned.
 */
QL_API ql_status benq_linear_ws(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y,
                                ql_out_dtype y_dtype, int B, int N, int K, void *workspace, size_t ws_bytes,
                                ql_stream_t stream);

/*
 * benq_mlp_gate_up -- the gated MLP of two BenQ projections of the same input,
 *     h[b][n] = silu(g[b][n]) * u[b][n],  g = x W_g^T,  u = x W_u^T,  silu(v) = v / (1 + e^-v)
 *   (the MLP of the card's model family; the gate itself is not printed on the pages).
 *   W_g and W_u are N x K BenQ layers stored as for benq_linear (codes_g / lut_g, codes_u /
 *   lut_u); x bf16 [B][K]; h [B][N] of h_dtype (bf16: round to nearest even of the fp32 value).
 *   g and u are accumulated exactly as benq_linear computes them; the gate is taken in fp32
 *   (library expf, IEEE division).  B == 1 with K % 1024 == 0 (K <= 20480) and N even runs as one
 *   fused kernel that needs no workspace; other shapes run both projections (GEMV or tensor-core
 *   GEMM) into the workspace and a gate kernel.
 *   workspace  device, 256-byte aligned, ws_bytes >= benq_mlp_workspace_bytes(B, N, K); NULL with 0
 *              when that is 0.  Owned by the caller, not shared with a concurrent call.
 *   Errors: as benq_linear (alignment of every pointer 16 bytes, B > 16 needs K % 64 == 0 and
 *   N % 256 == 0), QL_ERR_INVALID_ARG for a workspace smaller than required.
 */
QL_API ql_status benq_mlp_gate_up(const uint8_t *codes_g, const uint16_t *lut_g, const uint8_t *codes_u,
                                  const uint16_t *lut_u, const uint16_t *x, void *h, ql_out_dtype h_dtype, int B,
                                  int N, int K, void *workspace, size_t ws_bytes, ql_stream_t stream);

/* Workspace bytes benq_mlp_gate_up needs for these sizes (0 when the fused batch-1 kernel runs). */
QL_API size_t benq_mlp_workspace_bytes(int B, int N, int K);

/*
 * benq_linear_multi -- several BenQ layers that read the same input, y_s = x W_s^T for
 *   s < S ("What BenQ stores": each layer stored as for benq_linear), as the attention
 *   projections q, k and v of a decoder layer are.  At B == 1, with K % 1024 == 0 (K <= 20480)
 *   and every N % 4 == 0, all layers run in one launch of the batch-1 GEMV, which walks the row
 *   tiles of every layer as one range (a small layer then shares the SMs with the others instead
 *   of leaving them idle); each y_s equals benq_linear's result for that layer bit for bit.
 *   Other shapes run the layers one after another through benq_linear.
 *   layers  host array of S entries {codes, lut, y, N}: device pointers and the layer's output
 *           features, each as for benq_linear (16-byte aligned).
 *   S       1 <= S <= 4.
 *   x       device, bf16 bits [B][K], shared by all layers; y_s [B][N_s] of y_dtype.
 *   Errors: as benq_linear for every layer; QL_ERR_INVALID_ARG for S outside [1, 4].
 */
typedef struct {
  const uint8_t *codes;   /* [N][3K/4] packed codes */
  const uint16_t *lut;    /* [N][64] bf16 tables */
  void *y;                /* [B][N] output */
  int N;                  /* output features */
} benq_layer;
QL_API ql_status benq_linear_multi(const benq_layer *layers, int S, const uint16_t *x, ql_out_dtype y_dtype,
                                   int B, int K, ql_stream_t stream);

/* Workspace bytes benq_linear_ws uses for these sizes on the current device
 * (0 when B <= 16 or when no split applies).  Needs a CUDA device. */
QL_API size_t benq_linear_workspace_bytes(int B, int N, int K);

/*
 * benq_encode -- quantizes a bf16 matrix to BenQ storage ("Why equal-width shells": 32 magnitude
 *   tiers as equal-width shells of each row's range, member-mean levels refined Lloyd-style,
 *   nearest-level assignment; the uncalibrated path, no calibration data):
 *     D = max_k |W[n][k]| / 32, tier t = min(floor(|w| / D), 31) in fp64;
 *     level t = fp64 mean of the magnitudes in tier t (the shell midpoint (t + 1/2) D when empty),
 *               rounded fp64 -> fp32 -> bf16 to nearest even;
 *     lloyd_iters rounds of: assign every magnitude to its nearest level (lower tier on an exact
 *               tie), level = fp64 mean of its members (unchanged without members), rounded the same;
 *     code = 32 + t for w >= 0 (zero and -0 included), 31 - t for w < 0 with t the nearest level,
 *     table [-L31 .. -L0, L0 .. L31]; an all-zero row gets zero levels and codes 32.
 *   W      device bf16 [N][K] (read);  codes  device uint8 [N][3K/4] (written, the layout
 *          benq_linear reads);  lut  device bf16 [N][64] (written).  K % 4 == 0, 0 <= lloyd_iters <= 1000.
 *   W must be finite (NaN or Inf weights give unspecified codes).
 *   The result is exact and independent of scheduling when every row's nonzero magnitudes span less
 *   than a factor 2^30 (the tier sums are then exact in fp64); beyond that the tier means are
 *   rounded in an unspecified order.
 */
QL_API ql_status benq_encode(const uint16_t *W, uint8_t *codes, uint16_t *lut, int N, int K, int lloyd_iters,
                             ql_stream_t stream);

/*
 * benq_dequant_debug -- W[n][k] = lut[n][code(n,k)] as bf16 bits, row-major
 *   [N][K].  Bit-exact by construction; meant for checking, not speed.
 *   Same codes / lut layout as benq_linear; K % 4 == 0.
 */
QL_API ql_status benq_dequant_debug(const uint8_t *codes, const uint16_t *lut, uint16_t *W, int N,
                             int K, ql_stream_t stream);

/* Storage cost of one BenQ layer: 6 code bits + 64*16/K table bits per weight
 * (the card's bits/weight table).  Host only. */
QL_API double benq_bits_per_weight(int K);

/* ---------------------------------------------------------------- MDBF ----- */

/* One residual path.  Every pointer is device memory; the struct itself is host memory. */
typedef struct {
  const uint8_t *S_A;     /* [n][ldSA] packed signs of the n x r matrix S_A */
  const uint8_t *S_B;     /* [r][ldSB] packed signs of the r x m matrix S_B */
  size_t ldSA, ldSB;      /* row strides in bytes, >= ceil(r/8), >= ceil(m/8) */
  const uint16_t *A_amp;  /* fp16 bits [n][l] */
  const uint16_t *B_amp;  /* fp16 bits [m][l] */
  const uint16_t *Q_U;    /* fp16 bits [r][l] */
  const uint16_t *Q_V;    /* fp16 bits [r][l] */
} mdbf_path;

/* Bytes of device workspace mdbf_linear needs for these sizes (0 on invalid sizes).  For
 * batches that run on the tensor cores (see mdbf_linear) the size depends on how many CTA pairs
 * the current device holds at once: query it with the device current that will run the call
 * (without a device it returns the size of a run that does not split the last wave). */
QL_API size_t mdbf_workspace_bytes(int P, int n, int m, int r, int l, int B);

/*
 * mdbf_linear -- y[b][a] = sum_p sum_j (F_p G_p)[a][j] x[b][j], evaluated
 *   without forming W, as two sign-matrix products per path
 *   ("Algorithm": F = S_A (.) (A_amp Q_U^T), G = S_B (.) (Q_V B_amp^T)):
 *     t[k][b]   = sum_i Q_V[k][i] * sum_j S_B[k][j] * (B_amp[j][i] * x[b][j])
 *     y[b][a]  += sum_i A_amp[a][i] * sum_k S_A[a][k] * (Q_U[k][i] * t[k][b]).
 *
 *   paths      host array of P paths (device pointers inside).
 *   P, n, m, r, l  paths, out features, in features, rank, envelope rank;
 *              1 <= r <= min(n, m) (the page's rank clamp), l >= 1.
 *   x          device, bf16 bits [B][m].
 *   y          device, [B][n] of y_dtype; fully overwritten.
 *   workspace  device scratch of ws_bytes >= mdbf_workspace_bytes(...), 256-byte
 *              aligned; contents on entry are ignored and on return undefined.
 *   Execution: l * B <= 64 runs the decode kernels once (sign products on the warp MMA with
 *   the dense operand split into bf16 high and low parts).  Larger batches with l <= 32 and
 *   n, m, r >= 64 run as two tensor-core GEMMs, T = X G^T and y = T F^T, each factor element
 *   rebuilt in fp16 inside the GEMM (fp32 accumulation).  Powers of two keep every fp16 value
 *   in range: each factor is rebuilt times 2^-e (e >= 0 from the envelope column maxima, so that
 *   no element's bound sum_i max|L_i| max|R_i| exceeds 2^15), each token row of x is scaled so
 *   that x and T fit fp16, and y is scaled back exactly; any envelope magnitudes are accepted.
 *   All other batches run through the decode kernels floor(64 / l) rows at a time.
 *   Limits: l <= 64 (else QL_ERR_UNSUPPORTED), P <= 8.
 */
QL_API ql_status mdbf_linear(const mdbf_path *paths, int P, int n, int m, int r, int l,
                      const uint16_t *x, void *y, ql_out_dtype y_dtype, int B, void *workspace,
                      size_t ws_bytes, ql_stream_t stream);

/*
 * mdbf_linear_multi -- S MDBF layers of the same sizes that read the same x (the gate and up
 *   projections of a gated MLP): y_s = W_s x for s < S, each exactly as mdbf_linear computes it
 *   (the same kernels and arithmetic, bit for bit).
 *   paths      host array of S * P paths, layer s's paths at [s * P, s * P + P).
 *   S, P       layers and paths per layer: 1 <= S <= 4, S * P <= 8.
 *   ys         host array of S device outputs, each [B][n] of y_dtype (4-byte aligned), fully
 *              overwritten.
 *   workspace  device scratch of ws_bytes >= mdbf_workspace_bytes(S * P, n, m, r, l, B), 256-byte
 *              aligned; contents on entry are ignored and on return undefined.
 *   Execution: where the layers run the decode kernels with the one-pass F stage (l * B <= 4, at
 *   most two paths per layer, 16-byte aligned sign rows), each of the three launches covers all
 *   layers, so S layers take three launches instead of 3 S.  Otherwise the layers run one after
 *   another as mdbf_linear calls on the same workspace.  Other sizes and limits as mdbf_linear.
 */
QL_API ql_status mdbf_linear_multi(const mdbf_path *paths, int S, int P, int n, int m, int r, int l,
                                   const uint16_t *x, void *const *ys, ql_out_dtype y_dtype, int B,
                                   void *workspace, size_t ws_bytes, ql_stream_t stream);

/*
 * mdbf_linear_noalloc -- mdbf_linear for callers that cannot allocate device memory.
 *   The paper has no counterpart: this is a deployment convenience.  Some callers can't call
 *   cudaMalloc (or must not: allocator-internal code, real-time threads that may not block in
 *   the driver, hosts with a memory budget fixed at start-up), so this entry point needs no
 *   workspace.  Its scratch is a fixed 4 MiB array compiled into the library
 *   (mdbf_noalloc_scratch_bytes()); every GPU that loads the library holds it until the process
 *   exits, and sizes whose mdbf_workspace_bytes() exceed it return QL_ERR_UNSUPPORTED.  The
 *   library allocates nothing for this call.
 *   Arguments, layouts and results are those of mdbf_linear without workspace/ws_bytes.
 *   All calls share the one array: calls that may overlap on the GPU (two streams, or two host
 *   threads with no ordering between their streams) race and must be serialised by the caller.
 *   Every scratch byte that is read is first written by the same call, so nothing needs
 *   clearing between calls.  The first call on each device looks up the array's device address
 *   with that device current (and so does the first call after the device's context has been
 *   destroyed and created again); make that first call before any stream capture.
 */
QL_API ql_status mdbf_linear_noalloc(const mdbf_path *paths, int P, int n, int m, int r, int l,
                                     const uint16_t *x, void *y, ql_out_dtype y_dtype, int B,
                                     ql_stream_t stream);

/* Size in bytes of the static scratch array mdbf_linear_noalloc uses (its size limit).  Host only. */
QL_API size_t mdbf_noalloc_scratch_bytes(void);

/*
 * mdbf_dequant_debug -- materialises W (and optionally the factors) in fp32:
 *   F[p][a][k] = s_A[a][k] * fp32(sum_i A_amp[a][i] Q_U[k][i])   (i ascending),
 *   G[p][k][j] = s_B[k][j] * fp32(sum_i Q_V[k][i] B_amp[j][i])   (i ascending),
 *   W[a][j]    = fp32( sum_p sum_k F[p][a][k] * G[p][k][j] ), the sum taken in
 *                fp64, p outer and k ascending, so the result is reproducible
 *                bit for bit.
 *   W  device fp32 [n][m] (required); F device fp32 [P][n][r] or NULL;
 *   G  device fp32 [P][r][m] or NULL.  O(P n m r) fp64 work: for checking only.
 */
QL_API ql_status mdbf_dequant_debug(const mdbf_path *paths, int P, int n, int m, int r, int l, float *W,
                             float *F, float *G, ql_stream_t stream);

/* Effective bits per weight of an MDBF layer ("Bit-width and rank"):
 *   b_eff = P [ r (n+m) + scale_bits * l (n + m + 2r) ] / (n m).  Host only. */
QL_API double mdbf_effective_bits(int n, int m, int r, int P, int l, int scale_bits);

/*
 * mdbf_select_rank -- rank for a target bits/weight by inverting b_eff
 *   ("Bit-width and rank"), rounded down, then clamped to min(n, m) ("The
 *   matrix shape caps the reachable BPW").  *r_out receives the rank and
 *   *clamped 1 when the target exceeded b_max (the layer then lands below the
 *   request).  Returns QL_ERR_INVALID_ARG when even rank 1 exceeds the target.
 *   Host only.
 */
QL_API ql_status mdbf_select_rank(int n, int m, int P, int l, int scale_bits, double target_bits,
                           int *r_out, int *clamped);

/* ---------------------------------------------------------------- misc ----- */

/* Message for the calling thread's last non-OK status ("" if none). */
QL_API const char *ql_last_error(void);

/* Waits for `stream`, then reports (and clears) a device-side timeout flag:
 * QL_OK, QL_ERR_TIMEOUT, or QL_ERR_CUDA if the stream itself failed. */
QL_API ql_status ql_check(ql_stream_t stream);

/* Self-test of the bounded device-side waits (no counterpart in the pages): launches a CTA pair
 * whose wait on a barrier that nothing arrives on gives up after ~10 ms, propagates the abort to the
 * other CTA and raises the flag ql_check() reports; the kernel then returns normally, so the next
 * ql_check(stream) returns QL_ERR_TIMEOUT and the context stays usable. */
QL_API ql_status ql_selftest_timeout(ql_stream_t stream);

/* Launch overlap (programmatic dependent launch).  No counterpart in the pages:
 * this is launch plumbing.  When enabled (the default; the environment variable
 * QL_PDL=0 at load time disables it), every kernel is launched so that it may
 * start while the kernel before it in the same stream is still finishing.  Each
 * kernel reads its WEIGHTS (codes, tables, sign bits, envelopes) before it has
 * waited for that predecessor, and reads activations / workspace and writes
 * outputs only after the wait.  Weights are therefore treated as constants: a
 * caller that writes weights with a kernel and then calls a linear entry point on
 * the same stream right after it must either disable overlap or put a host
 * synchronisation, an event wait or a copy between the two.  The setting is
 * process-wide and takes effect at the next launch.  Returns the previous
 * setting (1 enabled, 0 disabled). */
QL_API int ql_set_pdl(int enable);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_H */

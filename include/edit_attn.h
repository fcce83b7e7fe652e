/*
 * edit_attn.h -- C ABI of the B200 (sm_100a) EDiT linear compressed attention
 * library (libedit_attn.so).
 *
 * What it computes. The paper-notes page "EDiT: Efficient Diffusion
 * Transformers with Linear Compressed Attention" (ICCV 2025, arXiv
 * 2503.16726), section "Method in detail", defines one attention layer:
 *   - ConvFusion query, eq. (Q^EDiT):
 *       Q = ReLU(Linear_Q(X + Conv1x1(LeakyReLU(GN(Conv3x3(X))))))
 *     on the token sequence viewed as its H x W grid; the 3x3 conv compresses
 *     C -> c_red channels, the 1x1 conv restores c_red -> C.
 *   - Spatial Compressor, eq. (phi_SC): K = ReLU(DW(Linear_K(X))),
 *     V = DW(Linear_V(X)), DW a 3x3 depthwise conv of stride 2 (padding 1),
 *     leaving M = ceil(H/2) * ceil(W/2) key/value tokens.
 *   - Linear attention per head, eq. (y_i):
 *       y_i = (Q_i S) / (Q_i z + attn_eps),  S = sum_j K_j^T V_j,  z = sum_j K_j
 *     with heads = contiguous blocks of d = C/heads channels, no 1/sqrt(d)
 *     and no output projection.
 * Section "MM-EDiT", eq. (A^Hybrid), mixes it with softmax attention for
 * every interaction with prompt tokens, with eta = N_I / (N_I + N_T):
 *   out_img = eta * y + (1 - eta) * A(Q_I, K_P, V_P)
 *   out_txt = eta * A(Q_P, K_I, V_I) + (1 - eta) * A(Q_P, K_P, V_P)
 * where A(q,k,v) = softmax(q k^T / sqrt(d)) v per head, Q_I/K_I/V_I are the
 * EDiT query and compressed keys/values above, and Q_P/K_P/V_P are plain
 * Linear projections of the prompt tokens.
 *
 * Conventions for every entry point below.
 *   Layout:  x, out: [B, H*W, C], token n = h*W + w, channels innermost.
 *            x_txt, out_txt: [B, N_T, C].
 *   dtype:   x, out and every weight/bias share one dtype (EDIT_F32 or
 *            EDIT_BF16); all accumulation is fp32.
 *   Memory:  every pointer except the weights struct itself is DEVICE memory,
 *            owned by the caller, 16-byte aligned. The library never
 *            allocates, frees or synchronises (except edit_attn_read_status).
 *            Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *            default stream). Outputs must not alias inputs or the workspace.
 *            The library creates no streams or events either.
 *   Streams: a caller may lend a second stream (side_stream, a cudaStream_t
 *            of the same device, with EDIT_SIDE_EVENTS cudaEvent_t handles in
 *            side_events, all owned by the caller). bf16 calls then run part
 *            of their kernels there: the query's weight folding, and for
 *            layers of at most 32768 tokens (B*H*W) also the key/value branch
 *            and MM-EDiT's prompt-side attention. The side stream is forked
 *            from `stream` and joined back into it within the call, so
 *            everything still completes in `stream` order and the call can be
 *            captured in a CUDA graph. Calls that share a side stream or its
 *            events must be ordered on one `stream`. With side_stream NULL
 *            every kernel runs on `stream`, one after the other (identical
 *            results). Stage events (below) and the key-ConvFusion variant
 *            also keep every kernel on `stream`.
 *   Workspace: caller-allocated device buffer of at least the size returned by
 *            the matching *_workspace_bytes query, 256-byte aligned. Distinct
 *            concurrent calls need distinct workspaces.
 *   Errors:  the return value is 0 (EDIT_OK) or a negative EDIT_ERR_* code.
 *            Arguments are validated on the host before any launch; on a
 *            validation error nothing is enqueued. Device-side problems (a
 *            bounded wait that ran out) are recorded in the workspace status
 *            word and read back with edit_attn_read_status. Kernel faults
 *            surface at the caller's next synchronisation. Nothing traps.
 */
#ifndef EDIT_ATTN_H_
#define EDIT_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EDIT_API __attribute__((visibility("default")))
#else
#define EDIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { EDIT_F32 = 0, EDIT_BF16 = 1 } edit_dtype;

/* Events that go with a caller-provided side stream (see Streams above). */
#define EDIT_SIDE_EVENTS 4

enum {
  EDIT_OK = 0,
  EDIT_ERR_NULL = -1,      /* a required pointer is NULL                          */
  EDIT_ERR_SHAPE = -2,     /* B, H, W < 1; C % heads; c_red % gn_groups; N_T < 0 ...*/
  EDIT_ERR_ALIGN = -3,     /* pointer not 16-byte aligned (workspace: 256-byte)    */
  EDIT_ERR_DTYPE = -4,     /* unsupported dtype                                    */
  EDIT_ERR_WORKSPACE = -5, /* workspace smaller than the query returned            */
  EDIT_ERR_CUDA = -6,      /* a CUDA runtime/driver call or launch failed          */
  EDIT_ERR_TIMEOUT = -7,   /* (device) a bounded wait ran out; results invalid     */
  EDIT_ERR_UNSUPPORTED = -8, /* shape outside what the kernels are built for       */
  EDIT_ERR_SCRATCH = -9     /* request needs more than the library's fixed scratch */
};

/* Weights and declared constants of one EDiT layer. Shapes (row-major):
 *   cf3_w [c_red][3][3][C]  3x3 conv C->c_red (torch [c_red,C,3,3] permuted to
 *                           channels-last: tap (kh,kw) reads pixel (h+kh-1, w+kw-1))
 *   cf3_b [c_red]           gn_gamma, gn_beta [c_red]
 *   cf1_w [C][c_red]        1x1 conv c_red->C; cf1_b [C]
 *   q_w, k_w, v_w [C][C]    Linear, torch [out][in] layout; q_b, k_b, v_b [C]
 *   kdw_w, vdw_w [C][3][3]  depthwise stride-2 conv taps; kdw_b, vdw_b [C]
 * Constants: gn_eps (GroupNorm, biased variance), leaky_slope, attn_eps (added
 * to the linear-attention denominator). None is defaulted by the library. */
typedef struct {
  int dtype; /* edit_dtype */
  int c_red;
  int gn_groups;
  float gn_eps;
  float leaky_slope;
  float attn_eps;
  const void *cf3_w, *cf3_b;
  const void *gn_gamma, *gn_beta;
  const void *cf1_w, *cf1_b;
  const void *q_w, *q_b;
  const void *k_w, *k_b;
  const void *v_w, *v_b;
  const void *kdw_w, *kdw_b;
  const void *vdw_w, *vdw_b;
  void *workspace; /* device, 256-byte aligned, >= edit_attn_workspace_bytes() */
  size_t workspace_bytes;
  void *side_stream;                   /* optional cudaStream_t (see Streams), or NULL */
  void *side_events[EDIT_SIDE_EVENTS]; /* cudaEvent_t handles; required with side_stream */
} edit_attn_weights;

/* Bytes of workspace edit_attn_forward needs for this shape (0 on a shape or
 * dtype error). Host-only: no allocation and no launch; the plan reads the
 * current device's SM count (148 when no device is visible), so query with
 * the device current that will run the layer. */
EDIT_API size_t edit_attn_workspace_bytes(int B, int H, int W, int C, int heads, const edit_attn_weights *w);

/* One EDiT attention layer: out[B, H*W, C] from x[B, H*W, C] (equations
 * above). Enqueues all kernels on `stream` and returns without waiting. */
EDIT_API int edit_attn_forward(const void *x, int B, int H, int W, int C, int heads, const edit_attn_weights *w,
                      void *out, void *stream);

/* Ablation variants of the query / key / value processing and an optional
 * output Linear. The ablation table of the notes page (section 消融实验,
 * "Query/Key/Value processing") compares the EDiT layer (CF, SC, SC) with
 * (CF, CF, -), (-, SC, SC) and (CF, -, -), where CF is ConvFusion, SC the
 * Spatial Compressor and - no processing beyond the Linear. Readings of the
 * table used here (it names the processing, not the formulas):
 *   q_proc  EDIT_PROC_CF:   Q = ReLU(Linear_Q(X + Conv1x1(LeakyReLU(GN(Conv3x3(X))))))
 *           EDIT_PROC_NONE: Q = ReLU(Linear_Q(X))
 *   k_proc  EDIT_PROC_SC:   K = ReLU(DW_K(Linear_K(X)))              (M keys)
 *           EDIT_PROC_CF:   K = ReLU(Linear_K(X + Conv1x1_K(LeakyReLU(GN_K(Conv3x3_K(X))))))
 *                           with the key's own ConvFusion weights below (N keys)
 *           EDIT_PROC_NONE: K = ReLU(Linear_K(X))                    (N keys)
 *   v_proc  EDIT_PROC_SC:   V = DW_V(Linear_V(X)); EDIT_PROC_NONE: V = Linear_V(X)
 * Keys and values must have equal counts, so (k_proc, v_proc) is one of
 * (SC, SC), (CF, NONE), (NONE, NONE); any other combination returns
 * EDIT_ERR_UNSUPPORTED. The attention step is eq. (y_i) over the M or N
 * key/value tokens. With o_w non-NULL the layer ends with the attention
 * block's output Linear, out = y o_w^T + o_b (o_w [C][C] torch layout, o_b
 * [C]); the page's layer has none, so it is optional.
 * kcf3_w [c_red][3][3][C], kcf3_b, kgn_gamma, kgn_beta [c_red], kcf1_w
 * [C][c_red], kcf1_b [C] are read only when k_proc is EDIT_PROC_CF; they use
 * the c_red, gn_groups, gn_eps and leaky_slope of the edit_attn_weights.
 * Weights a variant does not read may be NULL in both structs (for example
 * all ConvFusion weights, c_red and gn_groups when neither q_proc nor k_proc
 * is EDIT_PROC_CF; the depthwise weights without the compressor). */
enum { EDIT_PROC_NONE = 0, EDIT_PROC_CF = 1, EDIT_PROC_SC = 2 };

typedef struct {
  int q_proc;
  int k_proc;
  int v_proc;
  const void *kcf3_w, *kcf3_b;
  const void *kgn_gamma, *kgn_beta;
  const void *kcf1_w, *kcf1_b;
  const void *o_w, *o_b;
} edit_attn_variant;

/* Workspace bytes of edit_attn_variant_forward (0 on a shape, dtype or
 * processing error, or a NULL variant). Host-only. */
EDIT_API size_t edit_attn_variant_workspace_bytes(int B, int H, int W, int C, int heads, const edit_attn_weights *w,
                                                  const edit_attn_variant *v);

/* One layer with the processing chosen in `v` (conventions as
 * edit_attn_forward; the workspace is w->workspace and must hold
 * edit_attn_variant_workspace_bytes). {CF, SC, SC} with o_w == NULL computes
 * exactly what edit_attn_forward computes. Stage events (the hook below) are
 * the EDiT layer's 0-8, plus 9 after the output Linear when there is one. */
EDIT_API int edit_attn_variant_forward(const void *x, int B, int H, int W, int C, int heads,
                                       const edit_attn_weights *w, const edit_attn_variant *v, void *out,
                                       void *stream);

/* Mixing weights of the MM-EDiT hybrid (eta_mode below).
 *   EDIT_ETA_RATIO  the page's approximation: eta_I = eta_P = N_I / (N_I + N_T)
 *                   (section "MM-EDiT", the sentence after eq. (A^Hybrid)).
 *   EDIT_ETA_EXACT  the normaliser that ratio stands in for (the page calls it
 *                   the exact computation but does not write it out; reading
 *                   used here): each query normalises once over all keys.
 *                   Image row i, head h: eta = (Q_i z + eps) /
 *                   (Q_i z + eps + sum_P exp(q.k/sqrt(d))), i.e. image keys
 *                   weighted by the linear kernel Q_i . K_j and prompt keys by
 *                   exp(q . k / sqrt(d)) under one denominator. Prompt row:
 *                   eta = Z_I / (Z_I + Z_P) with Z the sums of
 *                   exp(q . k / sqrt(d)) over the image / prompt keys, i.e.
 *                   one softmax over both key sets. */
enum { EDIT_ETA_RATIO = 0, EDIT_ETA_EXACT = 1 };

/* Weights of the MM-EDiT hybrid: the EDiT image-stream weights (`img`, its
 * dtype field is the dtype of everything) plus the prompt-token projections
 * tq_w, tk_w, tv_w [C][C] (torch Linear layout) and their biases [C]. The
 * workspace and side-stream fields of `img` are ignored; the ones here are
 * used. eta_mode: EDIT_ETA_RATIO (0, the page's choice) or EDIT_ETA_EXACT;
 * anything else returns EDIT_ERR_UNSUPPORTED. */
typedef struct {
  edit_attn_weights img;
  const void *tq_w, *tq_b;
  const void *tk_w, *tk_b;
  const void *tv_w, *tv_b;
  void *workspace;
  size_t workspace_bytes;
  void *side_stream;
  void *side_events[EDIT_SIDE_EVENTS];
  int eta_mode;
} mmedit_weights;

EDIT_API size_t mmedit_workspace_bytes(int B, int H, int W, int N_T, int C, int heads, const mmedit_weights *w);

/* MM-EDiT hybrid attention (section "MM-EDiT", eq. (A^Hybrid)):
 * out_img[B, H*W, C] and out_txt[B, N_T, C] from x_img[B, H*W, C] and
 * x_txt[B, N_T, C]. N_T may be 0 (then eta = 1 and out_img is the EDiT
 * layer; x_txt/out_txt may be NULL). */
EDIT_API int mmedit_hybrid_forward(const void *x_img, const void *x_txt, int B, int H, int W, int N_T, int C, int heads,
                          const mmedit_weights *w, void *out_img, void *out_txt, void *stream);

/* Copy the device status word of a workspace to *status (0 = no device-side
 * error since the last forward call on it) and synchronise `stream`. This is
 * the only call that waits. When a tensor-core kernel's bounded wait ran out
 * (EDIT_ERR_TIMEOUT), the seven int32 words after the status word (offset
 * layout.status + 4) name the first wait that gave up: site (2: MMA issuer
 * waiting for a free accumulator, 3: MMA issuer waiting for operands,
 * 4: conv MMA issuer waiting for its input patch,
 * 10 + w: producer warp w waiting for a free stage, 20 + 10 r + q: epilogue
 * warp q of pair rank r waiting for an accumulator), block, tile, k-block (or
 * tiles done), stage or accumulator, barrier parity, globaltimer low bits. */
EDIT_API int edit_attn_read_status(const void *workspace, void *stream, int *status);

/* Text for a status code (static storage). */
EDIT_API const char *edit_status_string(int status);

/* Byte offsets of the intermediates kept in an edit_attn_forward workspace,
 * for inspection after the call completes (-1 when absent). Each tensor is
 * stored in the call's dtype unless noted:
 *   U [B,H,W,c_red]; G = LeakyReLU(GN(U)) [B,H*W,c_red]; Q [B,H*W,C];
 *   KVp [B,H*W,2C] (Linear_K(X) | Linear_V(X) per token);
 *   K, V [B,M,C] token-major (fp32 calls and MM-EDiT calls only);
 *   KT [B][C][Mp], VTx [B][heads][NP][Mp] channel-major (bf16 only): token
 *     t = i*Wop + j of the compressed grid padded to Wop columns (padding
 *     tokens are 0); rows d.. of each VTx head block are not written (the
 *     KV-state kernel forms the [V | 1] operand's ones row itself);
 *   gn_stats fp32 [B][gn_groups][2] (mean, rstd);
 *   Sz fp32 [B][heads][d][d+1] (S_h with z_h as the last column).
 * Mp, Wop, NP give the padded sizes (Mp = M, Wop = ceil(W/2), NP = 0 for fp32). */
typedef struct {
  int64_t status, U, G, Q, KVp, K, V, gn_stats, Sz, KT, VTx, Mp, Wop, NP;
} edit_ws_layout;

EDIT_API int edit_attn_workspace_layout(int B, int H, int W, int C, int heads, const edit_attn_weights *w,
                               edit_ws_layout *layout);

/* The same for an edit_attn_variant_forward workspace (v NULL: the EDiT
 * layer). Without the compressor, KT and VTx hold all N tokens in one padded
 * row (Mp = Wop = N rounded up to a multiple of 8). */
EDIT_API int edit_attn_variant_workspace_layout(int B, int H, int W, int C, int heads, const edit_attn_weights *w,
                                                const edit_attn_variant *v, edit_ws_layout *layout);

/* The DiT block around the attention (a text-to-image transformer block of
 * the PixArt-Sigma kind with EDiT as its self-attention; the notes page says
 * EDiT replaces the attention of PixArt-Sigma's blocks, section 整体框架 /
 * overall framework, but does not spell the block out: the block used here is
 * that model family's, read as follows).
 *   m = sst + t6[b] = (shift_a, scale_a, gate_a, shift_f, scale_f, gate_f)
 *   x1 = x + gate_a * (EDiT(LN(x) (1 + scale_a) + shift_a) o_w^T + o_b)
 *   x2 = x1 + softmax-attention(x1 cq_w^T + cq_b, y ck_w^T + ck_b, y cv_w^T + cv_b) co_w^T + co_b
 *   out = x2 + gate_f * (GELU(LN(x2) (1 + scale_f) + shift_f) fc1_w^T + fc1_b) fc2_w^T + fc2_b)
 * LN: LayerNorm over C without affine weights (eps ln_eps); GELU: the tanh
 * form; the cross-attention is per head with scale 1/sqrt(d), over the N_T
 * caption tokens y. Shapes (row-major, dtype of attn.dtype):
 *   x, out [B, H*W, C]; y [B, N_T, C] (N_T >= 1); t6 [B, 6, C] (the sample's
 *   timestep modulation); sst [6][C]; o_w, cq_w, ck_w, cv_w, co_w [C][C] and
 *   their biases [C]; fc1_w [hidden][C], fc1_b [hidden], fc2_w [C][hidden],
 *   fc2_b [C].
 * The EDiT attention weights and constants are those of `attn` (its workspace
 * and side-stream fields are ignored; the ones here are used). bf16 needs
 * hidden % 128 == 0 and head widths d of 32, 64 or 72 (the softmax kernel's);
 * other shapes return EDIT_ERR_UNSUPPORTED. */
typedef struct {
  edit_attn_weights attn;
  const void *o_w, *o_b;
  const void *sst;
  const void *cq_w, *cq_b, *ck_w, *ck_b, *cv_w, *cv_b, *co_w, *co_b;
  const void *fc1_w, *fc1_b, *fc2_w, *fc2_b;
  int hidden;
  float ln_eps;
  void *workspace;
  size_t workspace_bytes;
  void *side_stream;
  void *side_events[EDIT_SIDE_EVENTS];
} edit_dit_block_weights;

EDIT_API size_t edit_dit_block_workspace_bytes(int B, int H, int W, int N_T, int C, int heads,
                                               const edit_dit_block_weights *w);
EDIT_API int edit_dit_block_forward(const void *x, const void *y, const void *t6, int B, int H, int W, int N_T, int C,
                                    int heads, const edit_dit_block_weights *w, void *out, void *stream);

/* Row bands: one image split over several ranks (sequence parallelism).
 *
 * The notes page scales EDiT to 8192 x 8192 images (section 延迟分析, the
 * latency table); one such layer is 262,144 tokens. Its only global steps are
 * two reductions: the GroupNorm statistics of U = Conv3x3(X) (eq. (Q^EDiT))
 * and the per-head sums S = sum_j K_j^T V_j, z = sum_j K_j of eq. (y_i).
 * Everything else reads at most a 3 x 3 neighbourhood of a pixel. So the rows
 * of one image can be split into bands, one per rank:
 *   1. each rank takes its band of x plus one halo row above and one below
 *      from its neighbours (none at the image borders) and calls
 *      edit_attn_band_partials, which writes the band's record of partial
 *      sums;
 *   2. the ranks all-gather the records, in band order;
 *   3. each rank calls edit_attn_band_finish with all records, which sums them
 *      in band order (so every rank forms the same totals) and writes the
 *      band's rows of out.
 * Shapes and rules:
 *   band   rows [row0, row0 + rows) of an image of H rows: row0 even, and
 *          row0 + rows even unless it equals H, so that no stride-2 key/value
 *          token straddles two bands.
 *   x_ext  [rows + top + bottom][W][C]: the band with its halo rows, top = 1
 *          when row0 > 0, bottom = 1 when row0 + rows < H (else 0).
 *   record device buffer of edit_attn_band_record_bytes, 256-byte aligned:
 *          fp64 GroupNorm sums [gn_groups][2] (sum, sum of squares of the
 *          band's U), then, at the next 256-byte boundary, the band's fp32
 *          [S | z] [heads][d][d + 1].
 *   records the records of all nrecords bands, in band order, each
 *          edit_attn_band_record_bytes apart (256-byte aligned).
 *   out    [rows][W][C]: the band's rows of the layer output.
 * bf16 only (EDIT_ERR_UNSUPPORTED for fp32), one image. The workspace
 * (w->workspace, at least edit_attn_band_workspace_bytes) carries the band's
 * intermediates from the first call to the second: pass the same band, x_ext
 * and workspace to both, on the same stream. Errors as for edit_attn_forward;
 * a band that breaks the rules above is EDIT_ERR_SHAPE. */
typedef struct {
  int H;    /* rows of the whole image */
  int row0; /* first row of this band */
  int rows; /* rows of this band */
} edit_band;

EDIT_API size_t edit_attn_band_workspace_bytes(int W, int C, int heads, const edit_band *band,
                                               const edit_attn_weights *w);
EDIT_API size_t edit_attn_band_record_bytes(int C, int heads, const edit_attn_weights *w);
EDIT_API int edit_attn_band_partials(const void *x_ext, int W, int C, int heads, const edit_band *band,
                                     const edit_attn_weights *w, void *record, void *stream);
EDIT_API int edit_attn_band_finish(const void *x_ext, int W, int C, int heads, const edit_band *band,
                                   const edit_attn_weights *w, const void *records, int nrecords, void *out,
                                   void *stream);

/* Measurement hooks (no counterpart on the page; used by the benchmark).
 *
 * edit_attn_set_stage_events: when `events` is non-NULL, the next forward
 * calls made by this host thread record events[i] (cudaEvent_t handles
 * created by the caller) on the call's stream at stage boundary i:
 *   0 start, 1 K|V Linear GEMM, 2 depthwise conv, 3 KV state,
 *   4 weight folding, 5 3x3 conv GEMM (the conv kernel alone), 6 GroupNorm
 *   (statistics, finalize, apply; plus the conv's last-wave fixup when
 *   used), 7 query GEMM, 8 apply GEMM; MM-EDiT adds 9 prompt projections,
 *   10 image-row softmax attention, 11 prompt-row softmax attention.
 * Recording events between kernels serialises the programmatic overlap of
 * consecutive kernels at those points, so timed steps are fastest without
 * the hook.
 * `n` is the number of handles (events beyond n are not recorded). NULL
 * clears the hook. Returns EDIT_OK or EDIT_ERR_SHAPE for n < 0.
 *
 * edit_attn_kernel_launches: number of kernels this host thread's forward
 * calls have enqueued since the library was loaded. */
enum { EDIT_STAGE_EVENTS_EDIT = 9, EDIT_STAGE_EVENTS_MM = 12 };

EDIT_API int edit_attn_set_stage_events(void *const *events, int n);

EDIT_API uint64_t edit_attn_kernel_launches(void);

/* Wait drill for the device-side failure path (no counterpart on the page).
 *
 * Every device-side wait in the library is bounded and reports
 * EDIT_ERR_TIMEOUT through the workspace status word instead of hanging. This
 * hook lets a test make one such wait run out on purpose, without a fault.
 * bf16 layers at least 128 pixels wide normalise through a cooperative
 * GroupNorm kernel (statistics, grid barrier, apply in one grid); narrower ones
 * take the statistics from column sums their conv writes (in its epilogue, or
 * in the fixup of tiles split over k).
 * While the drill is armed (gn_extra_arrivals > 0), the calling thread's bf16
 * forward calls always run the cooperative kernel, which waits at its barrier for
 * gn_extra_arrivals more blocks than it launched, and gives up after
 * limit_ns nanoseconds (1e3 .. 2e9). Each block then records EDIT_ERR_TIMEOUT
 * and the first one the wait site (word 1 = 30, word 3 = arrivals seen,
 * word 4 = arrivals expected, word 5 = blocks launched) and returns without
 * applying the normalisation; later kernels of the call still run, and their
 * results are invalid. The GPU context stays usable. The cooperative kernel
 * runs for bf16 layers with at least 8 channels per group and c_red <= 4096.
 * (0, 0) disarms it. Returns EDIT_ERR_SHAPE for arguments out of range. */
EDIT_API int edit_attn_set_wait_drill(int gn_extra_arrivals, uint64_t limit_ns);

/* Linear attention step without any caller-provided scratch (the paper has
 * no counterpart; this is a deployment convenience).
 *
 * Some callers cannot allocate device memory at the point where they run the
 * layer: code running inside a framework's memory pool that forbids ad-hoc
 * cudaMalloc, plugins handed only their input and output buffers, or hosts
 * that must not grow device memory after start-up. For them this entry point
 * computes y from q, k, v exactly like the last step of edit_attn_forward
 * (per head: S = sum_j k_j^T v_j, z = sum_j k_j, y_i = q_i S / (q_i z + eps))
 * using a scratch array compiled into the library instead of a workspace.
 *
 *   q, out [B, N, C]; k, v [B, M, C] (device, dtype `dtype`, 16-byte aligned);
 *   heads divide C; the call is asynchronous on `stream`.
 *
 * The scratch is a static device array of EDIT_NOALLOC_SCRATCH_BYTES bytes
 * that every GPU which loads the library keeps until the process exits. Each
 * [S | z] block is B * heads * d * (d + 1) * 4 bytes (d = C / heads); a call
 * uses chunks + 1 such blocks (partial sums of each chunk of keys, then the
 * combined one), at least 3, and they must fit in the scratch: larger
 * requests return EDIT_ERR_SCRATCH without launching anything. d above 128,
 * or B or heads above 65535, return EDIT_ERR_UNSUPPORTED. The
 * library never calls cudaMalloc, cudaFree or any allocating routine here.
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture. All calls share the one array and it keeps the last call's
 * contents (every value a call reads is written earlier in the same call), so
 * calls whose kernels may overlap on the GPU (different streams without
 * ordering) race on it: order them on one stream. */
#define EDIT_NOALLOC_SCRATCH_BYTES (4u << 20)

EDIT_API int edit_linear_attention_noalloc(const void *q, const void *k, const void *v, int B, int N, int M, int C,
                                           int heads, int dtype, float attn_eps, void *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* EDIT_ATTN_H_ */

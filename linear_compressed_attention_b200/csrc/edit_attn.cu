// C ABI of the EDiT linear compressed attention library (include/edit_attn.h):
// argument validation, the workspace plan, TMA tensor-map encoding and the
// launch sequence of one EDiT layer / one MM-EDiT hybrid layer.
//
// Step order of one EDiT layer (bf16; fp32 uses the CUDA-core GEMM instead of
// the tensor-core one):
//   1. KVp = X [Wk; Wv]^T + [bk; bv]                      tensor-core GEMM
//   2. K = ReLU(DW_k(Kp)), V = DW_v(Vp)                    depthwise stride 2
//   3. [S_h | z_h] = sum_j K_jh^T [V_jh | 1]               split + fixed-order combine
//   4. Wqw1 = Wq W1, bq' = Wq b1 + bq                      weight folding (see below)
//   5. U = Conv3x3(X) (+ GroupNorm partial sums)           implicit-GEMM on tensor cores
//   6. G = LeakyReLU(GN(U))                                fixed-order stats, elementwise
//   7. Q = ReLU([X | G] [Wq | Wqw1]^T + bq')               tensor-core GEMM, K = C + Cr
//   8. y = (Q_h S_h) / (Q_h z_h + eps)                     tensor-core GEMM per head
// Step 4/7: the 1x1 conv of eq. (Q^EDiT) feeds only Linear_Q, so
// Linear_Q(X + Conv1x1(G)) = X Wq^T + G (Wq W1)^T + (Wq b1 + bq): the same
// FLOPs as the two GEMMs in a row, without writing and re-reading R.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "sdpa_tc.cuh"
#include "simt_kernels.cuh"
#include "tc_conv.cuh"
#include "tc_gemm.cuh"

using namespace edit;

namespace {

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

#define EDIT_TRY_CHECK(expr)          \
  do {                                \
    const int rc_ = (expr);           \
    if (rc_ != EDIT_OK) return rc_;   \
  } while (0)

enum Swz { SWZ_NONE = 0, SWZ_64 = 64, SWZ_128 = 128 };

bool encode(CUtensorMap* m, int rank, const void* base, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
            const cuuint32_t* box, int swz = SWZ_128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUtensorMapSwizzle sw = swz == SWZ_128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swz == SWZ_64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Apply output: out [img][R][C] bf16, unswizzled box d x 32 x 1 (one head of
// 32 rows per store).
bool map_out_heads(CUtensorMap* m, const void* base, long C, long R, long imgs, int d) {
  cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)R, (cuuint64_t)imgs};
  cuuint64_t st[2] = {(cuuint64_t)C * 2, (cuuint64_t)R * C * 2};
  cuuint32_t box[3] = {(cuuint32_t)d, 32, 1};
  return encode(m, 3, base, dims, st, box, SWZ_NONE);
}

// A operand: [imgs][rows][K] bf16, row stride ld elements, box 64 x 128 x 1.
bool map_a(CUtensorMap* m, const void* base, long K, long rows, long imgs, long ld, long img_stride) {
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)imgs};
  cuuint64_t st[2] = {(cuuint64_t)ld * 2, (cuuint64_t)img_stride * 2};
  cuuint32_t box[3] = {64, 128, 1};
  return encode(m, 3, base, dims, st, box);
}

// B operand: [rows][K] bf16, row stride ld elements, box 64 x box_rows.
bool map_b(CUtensorMap* m, const void* base, long K, long rows, long ld, int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t st[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  return encode(m, 2, base, dims, st, box);
}

// Output of the staged epilogue: [rows][ncols] bf16 (row stride ld), box 64 x 32.
bool map_out2d(CUtensorMap* m, const void* base, long ncols, long rows, long ld) {
  cuuint64_t dims[2] = {(cuuint64_t)ncols, (cuuint64_t)rows};
  cuuint64_t st[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, 32};
  return encode(m, 2, base, dims, st, box);
}

// Conv output U [B][H][W][Cr] bf16; one warp's 32 tile rows as a box
// 64 x bw x bh x 1 with bw = min(TW, 32), bh = 32 / bw.
bool map_out_grid(CUtensorMap* m, const void* base, int B, int H, int W, int Cr, int TW) {
  const int bw = TW < 32 ? TW : 32;
  cuuint64_t dims[4] = {(cuuint64_t)Cr, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t st[3] = {(cuuint64_t)Cr * 2, (cuuint64_t)W * Cr * 2, (cuuint64_t)H * W * Cr * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)bw, (cuuint32_t)(32 / bw), 1};
  return encode(m, 4, base, dims, st, box);
}

// Conv input patch for tap reuse: [B][H][W][C] bf16, box 64 x 130 x 3 x 1
// (3 image rows x 130 pixels: a 128-pixel tile row plus its halo).
bool map_patch(CUtensorMap* m, const void* base, int B, int H, int W, int C) {
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t st[3] = {(cuuint64_t)C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2};
  cuuint32_t box[4] = {64, 130, 3, 1};
  return encode(m, 4, base, dims, st, box);
}

// Conv input grid [B][H][W][C] bf16, box 64 x TW x TH x 1.
bool map_grid(CUtensorMap* m, const void* base, int B, int H, int W, int C, int TW, int TH) {
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t st[3] = {(cuuint64_t)C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)TW, (cuuint32_t)TH, 1};
  return encode(m, 4, base, dims, st, box);
}

// SM count of the current device, read once per device (148, the B200's,
// when no device is visible, so host-only queries still plan the same way).
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
  g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

// ------------------------------------------------------------ plan
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }


// Layers of at most this many tokens (B * H * W) run their K/V branch
// concurrently with the query branch (see run_edit).
constexpr long kForkMaxTokens = 32768;

// Most conv pair tiles ever split in the last wave (at most half of the
// co-resident pairs).
constexpr int kConvMaxSplit = 40;

struct Plan {
  // geometry
  int B, H, W, C, heads, Cr, G, d, Ho, Wo, M, NT;
  long HW;
  bool bf16;
  int es;  // bytes per element of activations/weights
  int TH, TW, tiles_h, tiles_w;
  int gn_P;       // GroupNorm partials per image
  int gn_slots = 0;  // bf16: GroupNorm column-sum slots per image (4 per conv tile, 32 rows each)
  int conv_pair_tiles = 0, conv_ksplit = 1;  // per-tap conv: pair tiles, k-parts per tile
  int gn_chunk;   // bf16: tokens per GroupNorm partial
  int kv_chunks;  // KV-state partials per (image, head)
  int NP, KP;     // apply operand padding: [S|z] rows (N) and K
  int bn_lin;     // tile N of the Linear GEMMs
  int npv = 0, nkpI = 0, nkpP = 0;  // MM-EDiT (bf16): [V | 1]^T rows per head, image / prompt keys padded to 128
  bool exact_eta = false;  // MM-EDiT: exact mixing weights (the apply keeps its normaliser in `den`)
  bool fork = false;   // K/V branch on the calling thread's side stream, concurrent with the query branch
  int Wop, Mp;    // bf16 KV state: padded compressed grid width and token count
  int kv_kb;      // bf16 KV state: 64-token k-blocks per chunk
  // query / key / value processing (edit_attn_variant; the EDiT layer is CF, SC, SC)
  int q_proc = EDIT_PROC_CF, k_proc = EDIT_PROC_SC, v_proc = EDIT_PROC_SC;
  bool compress = true;  // keys/values through the Spatial Compressor (M = ceil(H/2) ceil(W/2)), else M = N
  bool any_cf = true;    // some ConvFusion runs (c_red, gn_groups and their weights are used)
  bool oproj = false;    // output Linear after the attention
  // workspace offsets (bytes)
  size_t status, U, Gb, gnpart, gnstats, gnss, W1t, Wqw1, bfold, Q, KVp, K, V, KT, VTx, kvpart, Sz, SzT, QKVt,
      fixpart, VTi, VTp, den, Y, gncol, total;
};

int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Host-only shape/dtype checks and the workspace layout. Returns EDIT_OK or
// an error code; fills `pl` on success.
int make_plan(int B, int H, int W, int C, int heads, int NT, const edit_attn_weights* w, Plan& pl,
              const edit_attn_variant* var = nullptr) {
  if (!w) return EDIT_ERR_NULL;
  if (w->dtype != EDIT_F32 && w->dtype != EDIT_BF16) return EDIT_ERR_DTYPE;
  pl = Plan();
  if (var) {
    pl.q_proc = var->q_proc;
    pl.k_proc = var->k_proc;
    pl.v_proc = var->v_proc;
    const bool q_ok = pl.q_proc == EDIT_PROC_CF || pl.q_proc == EDIT_PROC_NONE;
    const bool kv_ok = (pl.k_proc == EDIT_PROC_SC && pl.v_proc == EDIT_PROC_SC) ||
                       (pl.k_proc == EDIT_PROC_CF && pl.v_proc == EDIT_PROC_NONE) ||
                       (pl.k_proc == EDIT_PROC_NONE && pl.v_proc == EDIT_PROC_NONE);
    if (!q_ok || !kv_ok) return EDIT_ERR_UNSUPPORTED;
    pl.compress = pl.k_proc == EDIT_PROC_SC;
    pl.any_cf = pl.q_proc == EDIT_PROC_CF || pl.k_proc == EDIT_PROC_CF;
    pl.oproj = var->o_w != nullptr;
  }
  if (B < 1 || H < 1 || W < 1 || C < 1 || heads < 1 || NT < 0) return EDIT_ERR_SHAPE;
  if (C % heads != 0) return EDIT_ERR_SHAPE;
  if (pl.any_cf && (w->c_red < 1 || w->gn_groups < 1 || w->c_red % w->gn_groups != 0)) return EDIT_ERR_SHAPE;
  if (static_cast<long>(H) * W > (1L << 28) || static_cast<long>(B) * H * W > (1L << 30) || C > 65536)
    return EDIT_ERR_SHAPE;
  pl.B = B;
  pl.H = H;
  pl.W = W;
  pl.C = C;
  pl.heads = heads;
  pl.Cr = pl.any_cf ? w->c_red : 0;
  pl.G = pl.any_cf ? w->gn_groups : 1;
  pl.d = C / heads;
  pl.Ho = pl.compress ? (H + 1) / 2 : H;
  pl.Wo = pl.compress ? (W + 1) / 2 : W;
  pl.M = pl.Ho * pl.Wo;
  pl.HW = static_cast<long>(H) * W;
  pl.NT = NT;
  pl.bf16 = w->dtype == EDIT_BF16;
  pl.es = pl.bf16 ? 2 : 4;
  if (pl.bf16) {
    // Tensor-core path constraints: 64-wide k-blocks over C, Linear tiles that
    // divide C, conv tile N = Cr (instantiated sizes), 16-byte head offsets.
    if (C % 128 != 0) return EDIT_ERR_UNSUPPORTED;
    if (pl.any_cf && !(pl.Cr == 64 || pl.Cr == 128 || pl.Cr == 256 || pl.Cr == 288 || pl.Cr == 384))
      return EDIT_ERR_UNSUPPORTED;
    if (!pl.compress && static_cast<long>(B) * (2 * C / 64) > 65535) return EDIT_ERR_UNSUPPORTED;
    if (pl.d % 8 != 0 || pl.d + 1 > 144) return EDIT_ERR_UNSUPPORTED;
    pl.bn_lin = (C % 256 == 0) ? 256 : (C % 192 == 0) ? 192 : 128;
    pl.TW = next_pow2(W) < 128 ? next_pow2(W) : 128;
    pl.TH = 128 / pl.TW;
    pl.tiles_h = (H + pl.TH - 1) / pl.TH;
    pl.tiles_w = (W + pl.TW - 1) / pl.TW;
    // per-tap conv (W < 128): when its pair tiles would fill at most half of the
    // CTA pairs, split every tile's 9C / 64 k-blocks over idle pairs
    pl.conv_pair_tiles = (B * pl.tiles_h * pl.tiles_w + 1) / 2;
    pl.conv_ksplit = 1;
    if (pl.TW < 128) {
      const int pairs = num_sms() / 2, nkb = 9 * C / 64;
      if (2 * pl.conv_pair_tiles <= pairs) {
        int k = pairs / pl.conv_pair_tiles;
        if (k > nkb / 9) k = nkb / 9;  // at least 9 k-blocks (one channel block of every tap) per part
        pl.conv_ksplit = k > 1 ? k : 1;
      }
    }
    pl.gn_chunk = 32;  // tokens per GroupNorm partial (many blocks: the pass is latency-bound otherwise)
    pl.gn_P = static_cast<int>((pl.HW + pl.gn_chunk - 1) / pl.gn_chunk);
    if (pl.gn_P < 2) pl.gn_P = 2;  // the fused GroupNorm runs at least two blocks
    if (!pl.any_cf) pl.gn_P = 0;
    // [S_h | z_h] has d + 1 columns; the apply GEMM is built for N = 48, 80, 144.
    pl.NP = (pl.d + 1 <= 48) ? 48 : (pl.d + 1 <= 80) ? 80 : 144;
    pl.KP = (pl.d + 63) / 64 * 64;
  } else {
    pl.gn_P = pl.any_cf ? static_cast<int>(pl.HW < 64 ? pl.HW : 64) : 0;
  }
  if (NT > 0 && !(pl.d == 32 || pl.d == 64 || pl.d == 72)) return EDIT_ERR_UNSUPPORTED;
  if (pl.bf16) {
    // Tensor-core KV state: tokens on a grid padded to 32 columns, split into
    // chunks of kv_kb 64-token blocks so that B * heads * chunks fills the GPU.
    // (without the compressor: the N tokens in one row padded to a multiple of 8)
    pl.Wop = pl.compress ? (pl.Wo + 31) / 32 * 32 : static_cast<int>((pl.HW + 7) / 8 * 8);
    pl.Mp = pl.compress ? pl.Ho * pl.Wop : pl.Wop;
    // The persistent kernel gives CTA i the tiles i, i + SMs, ...: pick the
    // chunk length that minimises (tiles per CTA) x (k-blocks per tile + 2,
    // the partial's store), i.e. no ragged extra wave of long tiles.
    const int total_kb = (pl.Mp + 63) / 64;
    const long bh = static_cast<long>(B) * heads;
    long best = -1;
    for (int kb = 4; kb <= (total_kb > 4 ? total_kb : 4); ++kb) {
      const long chunks = (total_kb + kb - 1) / kb;
      const long waves = (bh * chunks + num_sms() - 1) / num_sms();
      const long cost = waves * (kb + 2);
      if (best < 0 || cost < best) {
        best = cost;
        pl.kv_kb = kb;
      }
    }
    pl.kv_chunks = (total_kb + pl.kv_kb - 1) / pl.kv_kb;
  } else {
    pl.kv_chunks = pl.M / 256;
    if (pl.kv_chunks < 1) pl.kv_chunks = 1;
    if (pl.kv_chunks > 64) pl.kv_chunks = 64;
  }

  const size_t es = pl.es;
  const size_t tok = static_cast<size_t>(B) * pl.HW;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  pl.status = take(256);
  pl.U = take(tok * pl.Cr * es);
  pl.Gb = take(tok * pl.Cr * es);
  pl.gnpart = take(static_cast<size_t>(B) * pl.gn_P * pl.G * 2 * 4);
  pl.gnstats = take(static_cast<size_t>(B) * pl.G * 2 * 4);
  pl.gnss = take(static_cast<size_t>(B) * pl.Cr * 2 * 4);
  pl.W1t = take(static_cast<size_t>(pl.Cr) * C * es);  // (Cr = 0 when no ConvFusion runs)
  pl.Wqw1 = take(static_cast<size_t>(C) * pl.Cr * es);
  pl.bfold = take(static_cast<size_t>(C) * 4);
  pl.Q = take(tok * C * es);
  pl.KVp = take(tok * 2 * C * es);
  // token-major K, V: the fp32 path and MM-EDiT (prompt-row attention) read them
  const bool tokmajor = !pl.bf16 || NT > 0;
  pl.K = tokmajor ? take(static_cast<size_t>(B) * pl.M * C * es) : 0;
  pl.V = tokmajor ? take(static_cast<size_t>(B) * pl.M * C * es) : 0;
  pl.KT = pl.bf16 ? take(static_cast<size_t>(B) * C * pl.Mp * 2) : 0;
  pl.VTx = pl.bf16 ? take(static_cast<size_t>(B) * heads * pl.NP * pl.Mp * 2) : 0;
  pl.kvpart = take(static_cast<size_t>(B) * heads * pl.kv_chunks * pl.d * (pl.d + 1) * 4);
  pl.Sz = take(static_cast<size_t>(B) * heads * pl.d * (pl.d + 1) * 4);
  pl.SzT = pl.bf16 ? take(static_cast<size_t>(B) * heads * pl.NP * pl.KP * 2) : 0;
  pl.QKVt = NT > 0 ? take(static_cast<size_t>(B) * NT * 3 * C * es) : 0;
  // MM-EDiT: the linear part's normaliser Q z + eps per image row and head
  // (read by the image rows' exact mixing weights)
  pl.den = NT > 0 ? take(static_cast<size_t>(B) * pl.HW * heads * 4) : 0;
  // MM-EDiT softmax blocks (bf16): the image and prompt values as [V | 1]^T
  // operands, [B][heads][npv][keys padded to 128]
  pl.VTi = pl.VTp = 0;
  if (pl.bf16 && NT > 0) {
    pl.npv = pl.d + 1 <= 48 ? 48 : 80;
    pl.nkpI = (pl.M + 127) / 128 * 128;
    pl.nkpP = (NT + 127) / 128 * 128;
    pl.VTi = take(static_cast<size_t>(B) * heads * pl.npv * pl.nkpI * 2);
    pl.VTp = take(static_cast<size_t>(B) * heads * pl.npv * pl.nkpP * 2);
  }
  // fp32 halves of the conv tiles split in the last wave (tap-reuse conv only)
  pl.fixpart = (pl.bf16 && pl.TW == 128) ? take(static_cast<size_t>(kConvMaxSplit) * 4 * 128 * pl.Cr * 4) : 0;
  if (pl.bf16 && pl.TW < 128 && pl.conv_ksplit > 1)  // per-tap conv split over k: one fp32 partial per item
    pl.fixpart = take(static_cast<size_t>(pl.conv_pair_tiles) * pl.conv_ksplit * 2 * 128 * pl.Cr * 4);
  pl.Y = pl.oproj ? take(tok * C * es) : 0;  // attention output before the output Linear
  // GroupNorm column sums of U per 32-row slot of each conv tile, written by
  // the per-tap conv (bf16, W < 128): [B][gn_slots][Cr][2] fp32. The tap-reuse
  // conv (W >= 128) keeps a single TMEM accumulator, so work added to its
  // epilogue is not hidden; its layers take the cooperative GroupNorm.
  pl.gn_slots = (pl.bf16 && pl.any_cf && pl.TW < 128) ? pl.tiles_h * pl.tiles_w * 4 : 0;
  pl.gncol = take(static_cast<size_t>(B) * pl.gn_slots * pl.Cr * 2 * 4);
  // the key ConvFusion shares the query's ConvFusion buffers, so it stays serial
  pl.fork = pl.bf16 && pl.k_proc != EDIT_PROC_CF && static_cast<long>(B) * pl.HW <= kForkMaxTokens;
  pl.total = off;
  return EDIT_OK;
}

int check_ptrs(const void* const* ptrs, int n) {
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) return EDIT_ERR_NULL;
    if (!aligned(ptrs[i], 16)) return EDIT_ERR_ALIGN;
  }
  return EDIT_OK;
}

// The weights the plan's processing reads must be present and 16-byte aligned;
// the others are not touched and may be NULL.
int check_weights(const edit_attn_weights* w, const Plan& pl, const edit_attn_variant* var = nullptr) {
  const void* lin[] = {w->q_w, w->q_b, w->k_w, w->k_b, w->v_w, w->v_b};
  EDIT_TRY_CHECK(check_ptrs(lin, 6));
  if (pl.q_proc == EDIT_PROC_CF) {
    const void* cf[] = {w->cf3_w, w->cf3_b, w->gn_gamma, w->gn_beta, w->cf1_w, w->cf1_b};
    EDIT_TRY_CHECK(check_ptrs(cf, 6));
  }
  if (pl.compress) {
    const void* sc[] = {w->kdw_w, w->kdw_b, w->vdw_w, w->vdw_b};
    EDIT_TRY_CHECK(check_ptrs(sc, 4));
  }
  if (var && pl.k_proc == EDIT_PROC_CF) {
    const void* kcf[] = {var->kcf3_w, var->kcf3_b, var->kgn_gamma, var->kgn_beta, var->kcf1_w, var->kcf1_b};
    EDIT_TRY_CHECK(check_ptrs(kcf, 6));
  }
  if (var && pl.oproj) {
    const void* o[] = {var->o_w, var->o_b};
    EDIT_TRY_CHECK(check_ptrs(o, 2));
  }
  return EDIT_OK;
}

}  // namespace

namespace {

// ------------------------------------------------------------ measurement hooks
thread_local void* const* g_stage_events = nullptr;
thread_local int g_stage_n = 0;
thread_local uint64_t g_launches = 0;
// Wait drill (edit_attn_set_wait_drill): extra arrivals the fused GroupNorm's
// grid barrier waits for, and its wait limit while armed.
thread_local int g_drill_extra = 0;
thread_local uint64_t g_drill_limit_ns = 0;

void stage_mark(int i, cudaStream_t st) {
  if (g_stage_events && i < g_stage_n && g_stage_events[i])
    cudaEventRecord(static_cast<cudaEvent_t>(g_stage_events[i]), st);
}

// ------------------------------------------------------------ side stream
// The K/V branch (steps 1-3) and the query branch (steps 4-7) of a layer share
// no data. On small layers no kernel fills the GPU for long, so the K/V branch
// runs on a second stream, forked from the caller's stream after the status
// reset and joined back into it before the apply, and the two branches' fixed
// latencies (launch, pipeline fill, last wave) overlap. The stream and its
// four events belong to the caller (side_stream / side_events of the weights
// struct); without them every kernel runs on the caller's stream in order.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, fold = nullptr, kv = nullptr, join = nullptr;
};

SideStream side_of(void* stream, void* const* ev) {
  SideStream ss;
  if (!stream) return ss;
  ss.s = static_cast<cudaStream_t>(stream);
  ss.fork = static_cast<cudaEvent_t>(ev[0]);
  ss.fold = static_cast<cudaEvent_t>(ev[1]);
  ss.kv = static_cast<cudaEvent_t>(ev[2]);
  ss.join = static_cast<cudaEvent_t>(ev[3]);
  return ss;
}

// A side stream comes with all four events.
int check_side(void* stream, void* const* ev) {
  if (!stream) return EDIT_OK;
  for (int i = 0; i < EDIT_SIDE_EVENTS; ++i)
    if (!ev[i]) return EDIT_ERR_NULL;
  return EDIT_OK;
}

// ------------------------------------------------------------ launchers
// Every library kernel launches with programmatic stream serialization: it may
// start while the previous kernel drains and waits in pdl_wait() for that
// kernel's memory. The launch's own return code is kept for last_launch()
// (cudaGetLastError would also report, and clear, errors of the caller's
// earlier calls).
thread_local cudaError_t g_launch_err = cudaSuccess;

template <typename... KArgs, typename... Args>
void launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  g_launch_err = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

int last_launch() {
  ++g_launches;
  const cudaError_t e = g_launch_err;
  g_launch_err = cudaSuccess;
  return e == cudaSuccess ? EDIT_OK : EDIT_ERR_CUDA;
}

// Grid of gn_apply_leaky_bf16x8: B images (y), at most one wave of 8 blocks
// per SM over the images (x), each thread visiting several tokens.
dim3 gn_apply_grid(long HW, int B, int per_block) {
  long gx = (HW + per_block - 1) / per_block;
  long cap = static_cast<long>(num_sms()) * 8 / B;
  if (cap < 1) cap = 1;
  if (gx > cap) gx = cap;
  return dim3(static_cast<unsigned>(gx < 1 ? 1 : gx), static_cast<unsigned>(B), 1);
}

int grid_for(long total, int threads) {
  long g = (total + threads - 1) / threads;
  const long cap = static_cast<long>(num_sms()) * 16;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

template <int BN, int NSPLIT, int STAGES, int EPI, int STG = 0>
int launch_tc(const TcGemmParams& p, cudaStream_t st) {
  using Cfg = TcGemmCfg<BN, NSPLIT, STAGES, STG>;
  auto kern = tc_gemm_kernel<BN, NSPLIT, STAGES, EPI, STG>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
    return EDIT_ERR_CUDA;
  const int grid = p.num_tiles < num_sms() ? p.num_tiles : num_sms();
  if (grid < 1) return EDIT_OK;
  launch_pdl(kern, dim3(grid), dim3(192), Cfg::SMEM_BYTES, st, p);
  return last_launch();
}

// Co-resident 2-CTA clusters of a pair kernel on the current device (queried
// once per kernel instantiation and device, thread-safe).
template <typename Kern>
int pair_clusters(Kern kern, cudaLaunchConfig_t cfg, std::atomic<int>* cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = num_sms() / 2;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Pair kernel: clusters of 2 CTAs on neighbouring SMs, one persistent pair per
// co-resident cluster slot.
template <int BN, int NSPLIT, int STAGES, int EPI>
int launch_pair(const TcGemmParams& p, cudaStream_t st) {
  using Cfg = TcPairCfg<BN, NSPLIT, STAGES>;
  auto kern = tc_gemm_pair_kernel<BN, NSPLIT, STAGES, EPI>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
    return EDIT_ERR_CUDA;
  if (p.num_tiles < 1) return EDIT_OK;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(pair_threads(NSPLIT), 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  static std::atomic<int> cluster_cache[kMaxDevices];  // per instantiation and device
  const int max_clusters = pair_clusters(kern, cfg, cluster_cache);
  const int clusters = p.num_tiles < max_clusters ? p.num_tiles : max_clusters;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return EDIT_ERR_CUDA;
  return last_launch();
}

// Linear GEMM with 256 x 384 pair tiles (TMEM slot ring), same launch shape.
template <int STAGES, int STGBUF>
int launch_ring(const TcGemmParams& p, cudaStream_t st) {
  using Cfg = RingCfg<STAGES, STGBUF>;
  auto kern = tc_linear_ring_kernel<STAGES, STGBUF>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
    return EDIT_ERR_CUDA;
  if (p.num_tiles < 1) return EDIT_OK;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kRingThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  static std::atomic<int> cluster_cache[kMaxDevices];  // per instantiation and device
  const int max_clusters = pair_clusters(kern, cfg, cluster_cache);
  const int clusters = p.num_tiles < max_clusters ? p.num_tiles : max_clusters;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return EDIT_ERR_CUDA;
  return last_launch();
}

// Conv with tap reuse on CTA pairs (tiles of 128 pixels of one image row).
template <int BN, int NSPLIT, int NB>
int launch_conv_pair(TcGemmParams& p, cudaStream_t st, bool* split_out) {
  using Cfg = ConvPairCfg<BN, NSPLIT, NB>;
  auto kern = tc_conv_pair_kernel<BN, NSPLIT, NB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
    return EDIT_ERR_CUDA;
  if (p.num_tiles < 1) return EDIT_OK;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(conv_threads(NSPLIT), 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  static std::atomic<int> cluster_cache[kMaxDevices];  // per instantiation and device
  const int max_clusters = pair_clusters(kern, cfg, cluster_cache);
  // Last partial wave at most half full: split its tiles over the input-channel
  // blocks into two half items each, so every pair has work in that wave.
  const int T = p.num_tiles;
  const int R = T % max_clusters;
  p.split_first = T;
  p.split_count = 0;
  if (T > max_clusters && R > 0 && 2 * R <= max_clusters && R <= kConvMaxSplit && p.fix_part && p.kb_per_tap >= 2) {
    p.split_first = T - R;
    p.split_count = R;
    p.num_tiles = T + R;  // items
  }
  *split_out = p.split_count > 0;
  const int clusters = p.num_tiles < max_clusters ? p.num_tiles : max_clusters;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return EDIT_ERR_CUDA;
  return last_launch();
}

int gemm_conv_reuse(TcGemmParams& p, int cr, cudaStream_t st, bool* split) {
  p.num_n_tiles = 1;
  p.num_tiles = (p.num_m_tiles + 1) / 2;
  switch (cr) {
    case 64: return launch_conv_pair<64, 1, 8>(p, st, split);
    case 128: return launch_conv_pair<128, 1, 8>(p, st, split);
    case 256: return launch_conv_pair<256, 1, 5>(p, st, split);
    case 288: return launch_conv_pair<288, 2, 5>(p, st, split);
    case 384: return launch_conv_pair<384, 2, 3>(p, st, split);
  }
  return EDIT_ERR_UNSUPPORTED;
}

// Box rows of a B map = the MMA N of one instruction (half of it per CTA in a pair).
int conv_chunk(int cr) { return (cr == 288) ? 144 : (cr == 384) ? 192 : cr; }

// Linear GEMMs on CTA pairs: 256 x 256 pair tiles (one N = 256 MMA per
// k-step), or 256 x 384 tiles (three N = 128 chunks over a TMEM slot ring),
// which need 17% fewer operand bytes per MMA cycle. 384 is taken where the
// weight sources split on 192-row boundaries and it needs no more waves of
// pair tiles than 256 (measured: with equal waves, e.g. the K|V GEMM of 2 x
// 1,024 tokens, the 384 ring still finishes first, 24.8 -> 22.7 us).
constexpr int kPairBN = 256;
int ceil_div(long a, long b);
int linear_bn(long rows, int N, int n_split, const void* const* biases, int nbias) {
  if (!(n_split >= (1 << 30) || n_split % 192 == 0)) return kPairBN;
  for (int s = 0; s < nbias; ++s)  // the 384 epilogue reads bias vectors 16 bytes at a time
    if (reinterpret_cast<uintptr_t>(biases[s]) % 16 != 0) return kPairBN;
  const long m_pairs = (ceil_div(rows, 128) + 1) / 2;
  const long pairs = num_sms() / 2;
  const long w256 = (m_pairs * ceil_div(N, 256) + pairs - 1) / pairs;
  const long w384 = (m_pairs * ceil_div(N, 384) + pairs - 1) / pairs;
  return w384 <= w256 ? 384 : kPairBN;
}
// Weight-map box height (rows per CTA of a pair tile) for tile width bn.
int linear_box(int bn) { return bn / 2; }
int gemm_linear_pair(TcGemmParams& p, int bn, cudaStream_t st) {
  const int m_pairs = (p.num_m_tiles + 1) / 2;
  p.num_n_tiles = (p.N + bn - 1) / bn;
  p.num_tiles = m_pairs * p.num_n_tiles;
  if (bn == 384) return launch_ring<5, 1>(p, st);
  return launch_pair<kPairBN, 1, 5, EPI_LINEAR>(p, st);
}

// Small Linear GEMMs (weight folding) on single CTAs: 128 x 32 tiles, so the
// 1152 x 288 product spreads over 81 SMs.
int gemm_linear(const TcGemmParams& p, int bn, cudaStream_t st) {
  if (bn == 32) return launch_tc<32, 1, 8, EPI_LINEAR>(p, st);
  return EDIT_ERR_UNSUPPORTED;
}

// 3x3 conv on CTA pairs: 256 tokens x Cr pair tiles.
int gemm_conv(TcGemmParams& p, int cr, cudaStream_t st) {
  p.num_tiles = (p.num_m_tiles + 1) / 2 * (p.ksplit > 1 ? p.ksplit : 1);
  switch (cr) {
    case 64: return launch_pair<64, 1, 9, EPI_CONV>(p, st);
    case 128: return launch_pair<128, 1, 7, EPI_CONV>(p, st);
    case 256: return launch_pair<256, 1, 5, EPI_CONV>(p, st);
    case 288: return launch_pair<288, 2, 5, EPI_CONV>(p, st);
    case 384: return launch_pair<384, 2, 4, EPI_CONV>(p, st);
  }
  return EDIT_ERR_UNSUPPORTED;
}

// Apply: staging of 4 warps x 2 buffers x (32 rows x d bf16); d <= 40 / 72 / 136 for NP 48 / 80 / 144.
int gemm_apply(const TcGemmParams& p, int np, cudaStream_t st) {
  switch (np) {
    case 48: return launch_tc<48, 1, 8, EPI_APPLY, 8 * 32 * 40 * 2>(p, st);
    case 80: return launch_tc<80, 1, 6, EPI_APPLY, 8 * 32 * 72 * 2>(p, st);
    case 144: return launch_tc<144, 1, 4, EPI_APPLY, 8 * 32 * 136 * 2>(p, st);
  }
  return EDIT_ERR_UNSUPPORTED;
}

int gemm_kvstate(const TcGemmParams& p, int np, cudaStream_t st) {
  switch (np) {
    case 48: return launch_tc<48, 1, 8, EPI_KVSTATE>(p, st);
    case 80: return launch_tc<80, 1, 8, EPI_KVSTATE>(p, st);
    case 144: return launch_tc<144, 1, 6, EPI_KVSTATE>(p, st);
  }
  return EDIT_ERR_UNSUPPORTED;
}

int ceil_div(long a, long b) { return static_cast<int>((a + b - 1) / b); }

// Plain Linear on the tensor cores: out[rows][nsrc*C] = A[rows][K] [W0; W1; W2]^T + bias
// (optionally ReLU'd), output rows ldo elements apart.
int tc_linear(const void* a, long rows, int K, const void* const* wts, const void* const* biases, int nsrc, int C,
              void* out, long ldo, int relu, int* status, cudaStream_t st) {
  TcGemmParams p;
  std::memset(&p, 0, sizeof(p));
  if (!map_a(&p.a0, a, K, rows, 1, K, rows * K)) return EDIT_ERR_CUDA;
  p.a1 = p.a0;
  const int lbn = linear_bn(rows, nsrc * C, C, biases, nsrc);
  CUtensorMap* bm[3] = {&p.b0, &p.b1, &p.b2};
  for (int s = 0; s < 3; ++s)
    if (!map_b(bm[s], wts[s < nsrc ? s : 0], K, C, K, linear_box(lbn))) return EDIT_ERR_CUDA;
  p.bk = p.b0;
  p.R = static_cast<int>(rows);
  p.m_tiles_per_img = ceil_div(rows, 128);
  p.num_m_tiles = p.m_tiles_per_img;
  p.num_kb = K / 64;
  p.kb_split = p.num_kb;
  p.n_split = C;
  p.N = nsrc * C;
  p.out = out;
  p.ldo = ldo;
  if (!map_out2d(&p.out_map, out, p.N, rows, p.ldo)) return EDIT_ERR_CUDA;
  for (int s = 0; s < nsrc; ++s) p.bias[s] = biases[s];
  p.relu = relu;
  p.status = status;
  return gemm_linear_pair(p, lbn, st);
}

int simt_linear(const void* a, long rows, int K, const void* const* wts, const void* const* biases, int nsrc,
                int C, void* out, int ldo, int relu, cudaStream_t st) {
  SimtGemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.a0 = static_cast<const float*>(a);
  p.K0 = K;
  for (int s = 0; s < nsrc; ++s) {
    p.b[s] = static_cast<const float*>(wts[s]);
    p.bias[s] = static_cast<const float*>(biases[s]);
  }
  p.n_split = C;
  p.M = static_cast<int>(rows);
  p.N = nsrc * C;
  p.out = static_cast<float*>(out);
  p.ldo = ldo;
  p.relu = relu;
  launch_pdl(simt_gemm_f32, dim3(dim3(ceil_div(p.N, 64), ceil_div(p.M, 64))), dim3(256), 0, st, p);
  return last_launch();
}

#define EDIT_TRY(expr)        \
  do {                        \
    const int rc_ = (expr);   \
    if (rc_ != EDIT_OK) return rc_; \
  } while (0)

// One ConvFusion feature map: out = ReLU(Linear(X + Conv1x1(LeakyReLU(GN(Conv3x3(X)))))).
struct CfWeights {
  const void *cf3_w, *cf3_b, *gamma, *beta, *cf1_w, *cf1_b, *lin_w, *lin_b;
};
template <typename T>
int run_convfusion(const void* x, const Plan& pl, const CfWeights& cf, float gn_eps, float slope, void* out, long ldo,
                   int barrier_off, bool marks, uint8_t* ws, cudaStream_t st, bool fold = true,
                   cudaEvent_t fold_ready = nullptr);

// Steps 1-3: K, V and the per-head [S | z] (fp32) into the workspace. With the
// Spatial Compressor (the EDiT layer) K = ReLU(DW(Linear_K(X))), V = DW(Linear_V(X));
// without it the keys and values keep all N tokens: K = ReLU(Linear_K(X)) or the
// key's own ConvFusion feature map, V = Linear_V(X).
// Per-head partial [S | z] sums of the channel-major K, V operands (KT, VTx)
// over chunks of tokens: tensor-core GEMM Kᵀ [V | 1] into kvpart.
int kv_state_tc(const Plan& pl, uint8_t* ws, cudaStream_t st) {
  const __nv_bfloat16* KT = reinterpret_cast<const __nv_bfloat16*>(ws + pl.KT);
  const __nv_bfloat16* VTx = reinterpret_cast<const __nv_bfloat16*>(ws + pl.VTx);
  TcGemmParams p;
  std::memset(&p, 0, sizeof(p));
  {  // KT as [img * heads][d][Mp], box 64 x 128 x 1: the M = 128 tile reads one head's d rows, the rest is zero
    cuuint64_t dims[3] = {(cuuint64_t)pl.Mp, (cuuint64_t)pl.d, (cuuint64_t)pl.B * pl.heads};
    cuuint64_t st2[2] = {(cuuint64_t)pl.Mp * 2, (cuuint64_t)pl.d * pl.Mp * 2};
    cuuint32_t box[3] = {64, 128, 1};
    if (!encode(&p.a0, 3, KT, dims, st2, box)) return EDIT_ERR_CUDA;
  }
  p.a1 = p.a0;
  {  // VTx as [img * heads][d][Mp] (rows NP apart), box 64 x NP x 1: rows d.. read as zero, and the
     // kernel sets row d to ones (the [V | 1] operand: z as column d of the product)
    cuuint64_t dims[3] = {(cuuint64_t)pl.Mp, (cuuint64_t)pl.d, (cuuint64_t)pl.B * pl.heads};
    cuuint64_t st2[2] = {(cuuint64_t)pl.Mp * 2, (cuuint64_t)pl.NP * pl.Mp * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)pl.NP, 1};
    if (!encode(&p.b0, 3, VTx, dims, st2, box)) return EDIT_ERR_CUDA;
  }
  p.b1 = p.b2 = p.bk = p.b0;
  p.num_kb = (pl.Mp + 63) / 64;
  p.kb_split = p.num_kb;
  p.kb_per_chunk = pl.kv_kb;
  p.num_chunks = pl.kv_chunks;
  p.num_m_tiles = pl.kv_chunks;
  p.num_tiles = pl.B * pl.heads * pl.kv_chunks;
  p.num_n_tiles = 1;
  p.n_split = pl.NP;
  p.N = pl.NP;
  p.d = pl.d;
  p.heads = pl.heads;
  p.kv_part = reinterpret_cast<float*>(ws + pl.kvpart);
  p.status = reinterpret_cast<int*>(ws + pl.status);
  return gemm_kvstate(p, pl.NP, st);
}

// Depthwise stride-2 conv of the token-major K'|V' rows (an image of `rows`
// rows, the first `row_shift` of them a halo above the output rows) into the
// channel-major KT, VTx operands (and token-major K, V when the plan keeps
// them): output row i reads K'|V' rows 2i - 1 + row_shift .. 2i + 1 + row_shift.
int dwconv_tc(const Plan& pl, const edit_attn_weights* w, uint8_t* ws, int rows, int row_shift, cudaStream_t st) {
  __nv_bfloat16* KT = reinterpret_cast<__nv_bfloat16*>(ws + pl.KT);
  __nv_bfloat16* VTx = reinterpret_cast<__nv_bfloat16*>(ws + pl.VTx);
  DwTmaMaps mp;
  std::memset(&mp, 0, sizeof(mp));
  const long C2 = 2L * pl.C;
  cuuint64_t d_in[4] = {(cuuint64_t)C2, (cuuint64_t)pl.W, (cuuint64_t)rows, (cuuint64_t)pl.B};
  cuuint64_t s_in[3] = {(cuuint64_t)C2 * 2, (cuuint64_t)pl.W * C2 * 2, (cuuint64_t)rows * pl.W * C2 * 2};
  cuuint32_t b_in[4] = {64, 65, 3, 1};
  cuuint64_t d_kt[2] = {(cuuint64_t)pl.Mp, (cuuint64_t)pl.B * pl.C};
  cuuint64_t s_kt[1] = {(cuuint64_t)pl.Mp * 2};
  cuuint32_t b_kt[2] = {32, 64};
  cuuint64_t d_vt[3] = {(cuuint64_t)pl.Mp, (cuuint64_t)pl.NP, (cuuint64_t)pl.B * pl.heads};
  cuuint64_t s_vt[2] = {(cuuint64_t)pl.Mp * 2, (cuuint64_t)pl.NP * pl.Mp * 2};
  cuuint32_t b_vt[3] = {32, 8, 1};
  if (!encode(&mp.in, 4, ws + pl.KVp, d_in, s_in, b_in, SWZ_NONE) ||
      !encode(&mp.kt, 2, KT, d_kt, s_kt, b_kt, SWZ_64) || !encode(&mp.vtx, 3, VTx, d_vt, s_vt, b_vt, SWZ_64))
    return EDIT_ERR_CUDA;
  const int tokmajor = pl.K ? 1 : 0;
  if (tokmajor) {
    cuuint64_t d_t[4] = {(cuuint64_t)pl.C, (cuuint64_t)pl.Wo, (cuuint64_t)pl.Ho, (cuuint64_t)pl.B};
    cuuint64_t s_t[3] = {(cuuint64_t)pl.C * 2, (cuuint64_t)pl.Wo * pl.C * 2, (cuuint64_t)pl.Ho * pl.Wo * pl.C * 2};
    cuuint32_t b_t[4] = {64, 32, 1, 1};
    if (!encode(&mp.ktok, 4, ws + pl.K, d_t, s_t, b_t, SWZ_NONE) ||
        !encode(&mp.vtok, 4, ws + pl.V, d_t, s_t, b_t, SWZ_NONE))
      return EDIT_ERR_CUDA;
  }
  // The token-major staging block (MM-EDiT) is dynamic shared memory: without
  // it 7 blocks fit per SM instead of 6 (64K tokens: 84 -> 79 us). A layer
  // whose K/V branch runs beside the query branch keeps 6, leaving that
  // branch its share of the SMs (2 x 1K tokens: 0.088 ms with 6, 0.090 with 7).
  const size_t tok_bytes = (tokmajor || pl.fork) ? 32 * 64 * 2 : 0;
  launch_pdl(dwconv_s2_tma_kernel, dim3(dim3(pl.Wop / 32, pl.B * (2 * pl.C / 64), pl.Ho)), dim3(256), tok_bytes, st,
             mp, rows,
             pl.W, pl.C, pl.d, pl.heads, pl.Wop, static_cast<const __nv_bfloat16*>(w->kdw_w),
             static_cast<const __nv_bfloat16*>(w->kdw_b), static_cast<const __nv_bfloat16*>(w->vdw_w),
             static_cast<const __nv_bfloat16*>(w->vdw_b), tokmajor, row_shift, reinterpret_cast<int*>(ws + pl.status));
  return last_launch();
}

template <typename T>
int run_kv(const void* x, const Plan& pl, const edit_attn_weights* w, const edit_attn_variant* var, uint8_t* ws,
           cudaStream_t st, cudaEvent_t after_linear = nullptr) {
  int* status = reinterpret_cast<int*>(ws + pl.status);
  const long tok = static_cast<long>(pl.B) * pl.HW;
  const void* wts[3] = {w->k_w, w->v_w, w->k_w};
  const void* bs[3] = {w->k_b, w->v_b, nullptr};
  if (pl.k_proc == EDIT_PROC_CF) {
    // key = ConvFusion feature map with the key's weights (its GroupNorm uses
    // grid-barrier word 32 of the status block), value = Linear_V(X), side by
    // side in the token-major K'|V' rows (bf16) or into K and V (fp32)
    const CfWeights kcf = {var->kcf3_w, var->kcf3_b, var->kgn_gamma, var->kgn_beta,
                           var->kcf1_w, var->kcf1_b, w->k_w,         w->k_b};
    const long ldk = pl.bf16 ? 2L * pl.C : pl.C;
    EDIT_TRY(run_convfusion<T>(x, pl, kcf, w->gn_eps, w->leaky_slope, ws + (pl.bf16 ? pl.KVp : pl.K), ldk, 128,
                               false, ws, st));
    const void* vw[1] = {w->v_w};
    const void* vb[1] = {w->v_b};
    if (pl.bf16)
      EDIT_TRY(tc_linear(x, tok, pl.C, vw, vb, 1, pl.C, ws + pl.KVp + pl.C * 2, 2L * pl.C, 0, status, st));
    else
      EDIT_TRY(simt_linear(x, tok, pl.C, vw, vb, 1, pl.C, ws + pl.V, pl.C, 0, st));
  } else if (pl.bf16) {
    EDIT_TRY(tc_linear(x, tok, pl.C, wts, bs, 2, pl.C, ws + pl.KVp, 2L * pl.C, 0, status, st));
  } else if (pl.compress) {
    EDIT_TRY(simt_linear(x, tok, pl.C, wts, bs, 2, pl.C, ws + pl.KVp, 2 * pl.C, 0, st));
  } else {
    EDIT_TRY(simt_linear(x, tok, pl.C, wts, bs, 1, pl.C, ws + pl.K, pl.C, 1, st));
    EDIT_TRY(simt_linear(x, tok, pl.C, wts + 1, bs + 1, 1, pl.C, ws + pl.V, pl.C, 0, st));
  }
  stage_mark(1, st);
  if (after_linear && cudaEventRecord(after_linear, st) != cudaSuccess) return EDIT_ERR_CUDA;
  if (pl.bf16) {
    __nv_bfloat16* KT = reinterpret_cast<__nv_bfloat16*>(ws + pl.KT);
    __nv_bfloat16* VTx = reinterpret_cast<__nv_bfloat16*>(ws + pl.VTx);
    if (!pl.compress) {
      launch_pdl(kv_transpose_kernel, dim3(static_cast<unsigned>((pl.Mp + 63) / 64), pl.B * (2 * pl.C / 64)),
                 dim3(256), 0, st, reinterpret_cast<const __nv_bfloat16*>(ws + pl.KVp), static_cast<long>(pl.HW),
                 pl.C, pl.d, pl.heads, pl.NP, static_cast<long>(pl.Mp), KT, VTx);
      EDIT_TRY(last_launch());
    } else {
      EDIT_TRY(dwconv_tc(pl, w, ws, pl.H, 0, st));
    }
    stage_mark(2, st);
    EDIT_TRY(kv_state_tc(pl, ws, st));
  } else {
    if (pl.compress) {
      const long total = static_cast<long>(pl.B) * pl.M * (2 * pl.C);
      launch_pdl(dwconv_s2_kernel<T, 1>, dim3(grid_for(total, 256)), dim3(256), 0, st, 
          reinterpret_cast<const T*>(ws + pl.KVp), pl.B, pl.H, pl.W, pl.C, static_cast<const T*>(w->kdw_w),
          static_cast<const T*>(w->kdw_b), static_cast<const T*>(w->vdw_w), static_cast<const T*>(w->vdw_b),
          reinterpret_cast<T*>(ws + pl.K), reinterpret_cast<T*>(ws + pl.V));
      EDIT_TRY(last_launch());
    }
    stage_mark(2, st);
    const int nb = (pl.d + 3) / 4;
    int threads = (nb * nb + 31) / 32 * 32;
    if (threads < pl.d) threads = (pl.d + 31) / 32 * 32;
    const size_t smem = 2 * 32 * static_cast<size_t>(pl.d) * sizeof(float);
    launch_pdl(kv_state_partial_kernel<T>, dim3(dim3(pl.kv_chunks, pl.heads, pl.B)), dim3(threads), smem, st, 
        reinterpret_cast<const T*>(ws + pl.K), reinterpret_cast<const T*>(ws + pl.V), pl.M, pl.C, pl.heads,
        pl.kv_chunks, reinterpret_cast<float*>(ws + pl.kvpart));
    EDIT_TRY(last_launch());
  }
  {
    const int per_head = pl.d * (pl.d + 1);
    const long total = static_cast<long>(pl.B) * pl.heads * per_head;
    if (pl.bf16) {
      const long total_t = static_cast<long>(pl.B) * pl.heads * pl.NP * pl.KP;
      launch_pdl(kv_state_combine_pack_kernel, dim3(grid_for(total_t, 256)), dim3(256), 0, st,
                 reinterpret_cast<const float*>(ws + pl.kvpart), pl.kv_chunks, pl.d, pl.NP, pl.KP, total_t,
                 reinterpret_cast<float*>(ws + pl.Sz), reinterpret_cast<__nv_bfloat16*>(ws + pl.SzT));
    } else {
      launch_pdl(kv_state_combine_kernel, dim3(grid_for(total, 256)), dim3(256), 0, st,
                 reinterpret_cast<const float*>(ws + pl.kvpart), pl.kv_chunks, per_head, total,
                 reinterpret_cast<float*>(ws + pl.Sz));
    }
    EDIT_TRY(last_launch());
  }
  stage_mark(3, st);
  return EDIT_OK;
}

// Step 5 on the tensor cores: U = Conv3x3(X) + b for the plan's image grid
// (stage event 5 after the conv kernel when `marks`).
// gn_col: when set, the conv epilogue (whole tiles) and the fixup (tiles split
// over k) also write the GroupNorm column sums of U per 32-row slot of every
// tile, [B][gn_slots][Cr][2].
int conv3x3_tc(const void* x, const Plan& pl, const CfWeights& cf, uint8_t* ws, cudaStream_t st, bool marks,
               float* gn_col) {
  int* status = reinterpret_cast<int*>(ws + pl.status);
  const int C = pl.C, Cr = pl.Cr;
  TcGemmParams p;
  std::memset(&p, 0, sizeof(p));
  if (!map_grid(&p.a0, x, pl.B, pl.H, pl.W, C, pl.TW, pl.TH)) return EDIT_ERR_CUDA;
  p.a1 = p.a0;
  if (!map_b(&p.b0, cf.cf3_w, 9L * C, Cr, 9L * C, conv_chunk(Cr) / 2)) return EDIT_ERR_CUDA;
  p.b1 = p.b2 = p.bk = p.b0;
  p.num_kb = 9 * C / 64;
  p.kb_split = p.num_kb;
  p.kb_per_tap = C / 64;
  p.n_split = Cr;
  p.N = Cr;
  p.num_n_tiles = 1;
  p.H = pl.H;
  p.W = pl.W;
  p.TH = pl.TH;
  p.TW = pl.TW;
  p.tiles_h = pl.tiles_h;
  p.tiles_w = pl.tiles_w;
  p.num_m_tiles = pl.B * pl.tiles_h * pl.tiles_w;
  p.out = ws + pl.U;
  p.ldo = Cr;
  if (!map_out_grid(&p.out_map, ws + pl.U, pl.B, pl.H, pl.W, Cr, pl.TW)) return EDIT_ERR_CUDA;
  p.bias[0] = cf.cf3_b;
  p.status = status;
  p.gn_col = gn_col;
  if (pl.TW == 128) {  // tap reuse: one input patch per channel block feeds all 9 taps
    if (!map_patch(&p.a1, x, pl.B, pl.H, pl.W, C)) return EDIT_ERR_CUDA;
    p.fix_part = reinterpret_cast<float*>(ws + pl.fixpart);
    bool split = false;
    EDIT_TRY(gemm_conv_reuse(p, Cr, st, &split));
    if (marks) stage_mark(5, st);
    if (split) {  // the last wave's split tiles: two halves over the channel blocks
      const long nblk = static_cast<long>(p.split_count) * 2 * 4 * (Cr / 32);  // (tile, 32 rows, 8 quads)
      launch_pdl(conv_parts_fixup_kernel, dim3(grid_for(nblk * 256, 256)), dim3(256), 0, st, p.fix_part, 2,
                 p.split_first, p.split_count, pl.tiles_w, pl.tiles_h, pl.TH, pl.TW, pl.H, pl.W, Cr,
                 static_cast<const __nv_bfloat16*>(cf.cf3_b), p.num_m_tiles, reinterpret_cast<__nv_bfloat16*>(ws + pl.U),
                 gn_col);
      EDIT_TRY(last_launch());
    }
  } else {
    p.ksplit = pl.conv_ksplit;
    p.fix_part = reinterpret_cast<float*>(ws + pl.fixpart);
    EDIT_TRY(gemm_conv(p, Cr, st));
    if (marks) stage_mark(5, st);
    if (pl.conv_ksplit > 1) {  // every tile split over k
      const long nblk = static_cast<long>(pl.conv_pair_tiles) * 2 * 4 * (Cr / 32);  // (tile, 32 rows, 8 quads)
      launch_pdl(conv_parts_fixup_kernel, dim3(grid_for(nblk * 256, 256)), dim3(256), 0, st, p.fix_part, pl.conv_ksplit, 0,
                 pl.conv_pair_tiles, pl.tiles_w, pl.tiles_h, pl.TH, pl.TW, pl.H, pl.W, Cr,
                 static_cast<const __nv_bfloat16*>(cf.cf3_b), p.num_m_tiles, reinterpret_cast<__nv_bfloat16*>(ws + pl.U),
                 gn_col);
      EDIT_TRY(last_launch());
    }
  }
  return EDIT_OK;
}

// Step 7 on the tensor cores: out = ReLU([X | G] [Wl | Wl W1]^T + Wl b1 + bl)
// for `tok` token rows of x and g, with the folded weights of the plan's
// workspace (Wqw1, bfold); rows ldo elements apart.
int query_gemm_tc(const void* x, long tok, const Plan& pl, const CfWeights& cf, const void* g, uint8_t* ws, void* qout,
                  long ldo, cudaStream_t st) {
  int* status = reinterpret_cast<int*>(ws + pl.status);
  const int C = pl.C, Cr = pl.Cr;
  TcGemmParams p;
  std::memset(&p, 0, sizeof(p));
  if (!map_a(&p.a0, x, C, tok, 1, C, tok * C)) return EDIT_ERR_CUDA;
  if (!map_a(&p.a1, g, Cr, tok, 1, Cr, tok * Cr)) return EDIT_ERR_CUDA;
  const void* qb = ws + pl.bfold;
  const int lbn = linear_bn(tok, C, 1 << 30, &qb, 1);
  if (!map_b(&p.b0, cf.lin_w, C, C, C, linear_box(lbn))) return EDIT_ERR_CUDA;
  if (!map_b(&p.bk, ws + pl.Wqw1, Cr, C, Cr, linear_box(lbn))) return EDIT_ERR_CUDA;
  p.b1 = p.b2 = p.b0;
  p.R = static_cast<int>(tok);
  p.m_tiles_per_img = ceil_div(tok, 128);
  p.num_m_tiles = p.m_tiles_per_img;
  p.kb_split = C / 64;
  p.num_kb = C / 64 + ceil_div(Cr, 64);
  p.n_split = 1 << 30;  // one weight source; rows past C read as zeros
  p.N = C;
  p.out = qout;
  p.ldo = ldo;
  if (!map_out2d(&p.out_map, qout, C, tok, ldo)) return EDIT_ERR_CUDA;
  p.bias[0] = ws + pl.bfold;
  p.bias_f32 = 1;
  p.relu = 1;
  p.status = status;
  return gemm_linear_pair(p, lbn, st);
}

// Cooperative launch of the fused GroupNorm (bf16): as many blocks as are
// co-resident (at most gn_P, the partial buffer's capacity), 512 threads.
// The grid barrier counter is the status-block word at byte barrier_off (64 for
// the query's ConvFusion, 128 for the key's; clear of the status word and the
// wait-site words 1-7), which every call zeroes before its first launch. The
// barrier expects one arrival per block and gives up after EDIT_WAIT_TIMEOUT_NS,
// unless this thread armed the wait drill (edit_attn_set_wait_drill).
int launch_gn_fused(const Plan& pl, const CfWeights& cf, float gn_eps, float slope, int barrier_off, uint8_t* ws,
                    cudaStream_t st) {
  // two blocks per SM at most: more blocks only add partials to combine
  int nblk = 2 * num_sms();
  if (nblk > pl.gn_P) nblk = pl.gn_P;
  if (nblk > GN_FUSED_MAXB) nblk = GN_FUSED_MAXB;
  const size_t smem = (512 * 4 + static_cast<size_t>(pl.Cr) * 4) * sizeof(float);
  // (a per-device function attribute; setting it on every launch keeps it
  // right for whichever device and thread launches)
  if (cudaFuncSetAttribute(gn_fused_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024) !=
      cudaSuccess)
    return EDIT_ERR_CUDA;
  const unsigned int expect = static_cast<unsigned int>(nblk + (g_drill_extra > 0 ? g_drill_extra : 0));
  const uint64_t limit_ns = g_drill_extra > 0 ? g_drill_limit_ns : EDIT_WAIT_TIMEOUT_NS;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gn_fused_bf16_kernel, 512, smem) != cudaSuccess ||
      per_sm * num_sms() < nblk)
    return EDIT_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(nblk, 1, 1);
  cfg.blockDim = dim3(512, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, gn_fused_bf16_kernel, reinterpret_cast<const __nv_bfloat16*>(ws + pl.U), pl.B,
                         static_cast<long>(pl.HW), pl.Cr, pl.G, gn_eps,
                         static_cast<const __nv_bfloat16*>(cf.gamma), static_cast<const __nv_bfloat16*>(cf.beta),
                         slope, reinterpret_cast<float*>(ws + pl.gnpart),
                         reinterpret_cast<unsigned int*>(ws + pl.status + barrier_off), reinterpret_cast<float*>(ws + pl.gnstats),
                         reinterpret_cast<float*>(ws + pl.gnss), reinterpret_cast<__nv_bfloat16*>(ws + pl.Gb),
                         reinterpret_cast<int*>(ws + pl.status), expect, limit_ns) != cudaSuccess)
    return EDIT_ERR_CUDA;
  return last_launch();
}

// Step 4 for one ConvFusion feature map: the weight folding
// Wlw1 = Wl W1 and bl' = Wl b1 + bl (Wl, bl: the Linear after the residual).
// It reads only weights, so it may run on another stream than the steps that
// follow (the caller orders it before the query GEMM).
template <typename T>
int run_fold(const Plan& pl, const CfWeights& cf, uint8_t* ws, cudaStream_t st) {
  int* status = reinterpret_cast<int*>(ws + pl.status);
  const int C = pl.C, Cr = pl.Cr;
  // 4. weight folding
  launch_pdl(fold_prep_kernel<T>, dim3(ceil_div(Cr, 32) * ceil_div(C, 32) + ceil_div(C, 8)), dim3(256), 0, st,
             static_cast<const T*>(cf.cf1_w), C, Cr, reinterpret_cast<T*>(ws + pl.W1t), static_cast<const T*>(cf.lin_w),
             static_cast<const T*>(cf.lin_b), static_cast<const T*>(cf.cf1_b), reinterpret_cast<float*>(ws + pl.bfold));
  EDIT_TRY(last_launch());
  if (pl.bf16) {
    TcGemmParams p;
    std::memset(&p, 0, sizeof(p));
    if (!map_a(&p.a0, cf.lin_w, C, C, 1, C, static_cast<long>(C) * C)) return EDIT_ERR_CUDA;
    p.a1 = p.a0;
    if (!map_b(&p.b0, ws + pl.W1t, C, Cr, C, 32)) return EDIT_ERR_CUDA;
    p.b1 = p.b2 = p.bk = p.b0;
    p.R = C;
    p.m_tiles_per_img = ceil_div(C, 128);
    p.num_m_tiles = p.m_tiles_per_img;
    p.num_kb = C / 64;
    p.kb_split = p.num_kb;
    p.n_split = Cr;
    p.N = Cr;
    p.num_n_tiles = ceil_div(Cr, 32);
    p.num_tiles = p.m_tiles_per_img * p.num_n_tiles;
    p.out = ws + pl.Wqw1;
    p.ldo = Cr;
    p.status = status;
    EDIT_TRY(gemm_linear(p, 32, st));
  } else {
    SimtGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.a0 = static_cast<const float*>(cf.lin_w);
    p.K0 = C;
    p.b[0] = reinterpret_cast<const float*>(ws + pl.W1t);
    p.n_split = Cr;
    p.M = C;
    p.N = Cr;
    p.out = reinterpret_cast<float*>(ws + pl.Wqw1);
    p.ldo = Cr;
    launch_pdl(simt_gemm_f32, dim3(dim3(ceil_div(Cr, 64), ceil_div(C, 64))), dim3(256), 0, st, p);
    EDIT_TRY(last_launch());
  }

  return EDIT_OK;
}

// Steps 4-7 for one ConvFusion feature map (the query's in the EDiT layer):
// out = ReLU([X | G] [Wl | Wl W1]^T + Wl b1 + bl), rows ldo elements apart,
// with G = LeakyReLU(GN(Conv3x3(X))) and Wl, bl the Linear after the residual.
// Stage events 4-7 are recorded when `marks` is set. With `fold` false the
// folded weights come from run_fold on another stream, which records
// `fold_ready` after it: the query GEMM waits for that event.
template <typename T>
int run_convfusion(const void* x, const Plan& pl, const CfWeights& cf, float gn_eps, float slope, void* qout, long ldo,
                   int barrier_off, bool marks, uint8_t* ws, cudaStream_t st, bool fold, cudaEvent_t fold_ready) {
  auto mark = [&](int i) {
    if (marks) stage_mark(i, st);
  };
  const long tok = static_cast<long>(pl.B) * pl.HW;
  const int C = pl.C, Cr = pl.Cr;
  if (fold) EDIT_TRY(run_fold<T>(pl, cf, ws, st));
  mark(4);
  // 5. U = Conv3x3(X) (+ GroupNorm partials)
  float* gnpart = reinterpret_cast<float*>(ws + pl.gnpart);
  bool gn_fused = false;
  // GroupNorm partials: (P, cols) of the layout gn_finalize_kernel reads
  int gn_parts = pl.gn_P, gn_cols = 1;
  float* gn_src = gnpart;
  if (pl.bf16) {
    // The per-tap conv (W < 128) writes the GroupNorm column sums of U per
    // 32-row slot of each of its tiles, so no pass over U forms the statistics
    // and no grid-wide barrier is needed; wider layers run the cooperative
    // GroupNorm (statistics, bounded grid barrier, apply in one grid). With the
    // wait drill armed the cooperative kernel always runs: its barrier is the
    // wait the drill drives out.
    const bool colsum = pl.gn_slots > 0 && g_drill_extra <= 0;
    EDIT_TRY(conv3x3_tc(x, pl, cf, ws, st, marks, colsum ? reinterpret_cast<float*>(ws + pl.gncol) : nullptr));
    if (!colsum && (Cr / pl.G) >= 8 && Cr / 8 <= 512) {
      // 6. G = LeakyReLU(GN(U)) in one cooperative grid
      const int r = launch_gn_fused(pl, cf, gn_eps, slope, barrier_off, ws, st);
      if (r != EDIT_OK && r != EDIT_ERR_UNSUPPORTED) return r;
      gn_fused = r == EDIT_OK;
    }
    if (!gn_fused) {
      if (!colsum) {
        launch_pdl(gn_partial_kernel<__nv_bfloat16>, dim3(dim3(pl.gn_P, pl.B)), dim3(256), 0, st,
                   reinterpret_cast<const __nv_bfloat16*>(ws + pl.U), static_cast<int>(pl.HW), Cr, pl.G, pl.gn_P,
                   gnpart);
        EDIT_TRY(last_launch());
      } else {
        gn_parts = pl.gn_slots;
        gn_cols = Cr / pl.G;
        gn_src = reinterpret_cast<float*>(ws + pl.gncol);
      }
    }
  } else {
    SimtGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.a0 = static_cast<const float*>(x);
    p.K0 = 9 * C;
    p.conv = 1;
    p.B = pl.B;
    p.H = pl.H;
    p.W = pl.W;
    p.Cin = C;
    p.b[0] = static_cast<const float*>(cf.cf3_w);
    p.bias[0] = static_cast<const float*>(cf.cf3_b);
    p.n_split = Cr;
    p.M = static_cast<int>(tok);
    p.N = Cr;
    p.out = reinterpret_cast<float*>(ws + pl.U);
    p.ldo = Cr;
    launch_pdl(simt_gemm_f32, dim3(dim3(ceil_div(Cr, 64), ceil_div(tok, 64))), dim3(256), 0, st, p);
    EDIT_TRY(last_launch());
    mark(5);
    launch_pdl(gn_partial_kernel<float>, dim3(dim3(pl.gn_P, pl.B)), dim3(256), 0, st, reinterpret_cast<const float*>(ws + pl.U),
                                                                  static_cast<int>(pl.HW), Cr, pl.G, pl.gn_P, gnpart);
    EDIT_TRY(last_launch());
  }
  // 6. G = LeakyReLU(GN(U))
  if (!gn_fused) {
    launch_pdl(gn_finalize_kernel<T>, dim3(dim3(pl.G, pl.B)), dim3(gn_cols > 1 ? 1024 : 256), 0, st, gn_src, gn_parts,
               gn_cols, pl.G, Cr,
               pl.HW * (Cr / pl.G), gn_eps,
                                                static_cast<const T*>(cf.gamma), static_cast<const T*>(cf.beta),
                                                reinterpret_cast<float*>(ws + pl.gnstats),
                                                reinterpret_cast<float*>(ws + pl.gnss));
    EDIT_TRY(last_launch());
    if (pl.bf16) {
      const int nvec = Cr / 8;
      const int per_block = 256 / nvec > 0 ? 256 / nvec : 1;
      const int threads = per_block * nvec;
      launch_pdl(gn_apply_leaky_bf16x8, gn_apply_grid(pl.HW, pl.B, per_block), dim3(threads), 0, st,
                 reinterpret_cast<const __nv_bfloat16*>(ws + pl.U), reinterpret_cast<const float*>(ws + pl.gnss), pl.HW,
                 Cr, slope, reinterpret_cast<__nv_bfloat16*>(ws + pl.Gb));
    } else {
      const long total = tok * Cr;
      launch_pdl(gn_apply_leaky_kernel<float>, dim3(grid_for(total, 256)), dim3(256), 0, st, 
          reinterpret_cast<const float*>(ws + pl.U), reinterpret_cast<const float*>(ws + pl.gnss), pl.HW, Cr,
          slope, reinterpret_cast<float*>(ws + pl.Gb), total);
    }
    EDIT_TRY(last_launch());
  }
  mark(6);
  // 7. Q
  if (fold_ready && cudaStreamWaitEvent(st, fold_ready, 0) != cudaSuccess) return EDIT_ERR_CUDA;
  if (pl.bf16) {
    EDIT_TRY(query_gemm_tc(x, tok, pl, cf, ws + pl.Gb, ws, qout, ldo, st));
  } else {
    SimtGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.a0 = static_cast<const float*>(x);
    p.a1 = reinterpret_cast<const float*>(ws + pl.Gb);
    p.K0 = C;
    p.K1 = Cr;
    p.b[0] = static_cast<const float*>(cf.lin_w);
    p.bk = reinterpret_cast<const float*>(ws + pl.Wqw1);
    p.n_split = C;
    p.M = static_cast<int>(tok);
    p.N = C;
    p.out = static_cast<float*>(qout);
    p.ldo = static_cast<int>(ldo);
    p.bias[0] = reinterpret_cast<const float*>(ws + pl.bfold);
    p.relu = 1;
    launch_pdl(simt_gemm_f32, dim3(dim3(ceil_div(C, 64), ceil_div(tok, 64))), dim3(256), 0, st, p);
    EDIT_TRY(last_launch());
  }
  mark(7);
  return EDIT_OK;
}

// Steps 4-7: the query. ConvFusion (the EDiT layer) or, in the variant
// without it, Q = ReLU(X Wq^T + bq).
CfWeights query_cf(const edit_attn_weights* w) {
  return CfWeights{w->cf3_w, w->cf3_b, w->gn_gamma, w->gn_beta, w->cf1_w, w->cf1_b, w->q_w, w->q_b};
}

template <typename T>
int run_query(const void* x, const Plan& pl, const edit_attn_weights* w, uint8_t* ws, cudaStream_t st,
              bool fold = true, cudaEvent_t fold_ready = nullptr) {
  if (pl.q_proc == EDIT_PROC_CF)
    return run_convfusion<T>(x, pl, query_cf(w), w->gn_eps, w->leaky_slope, ws + pl.Q, pl.C, 64, true, ws, st, fold,
                             fold_ready);
  const long tok = static_cast<long>(pl.B) * pl.HW;
  const void* qw[1] = {w->q_w};
  const void* qb[1] = {w->q_b};
  if (pl.bf16)
    EDIT_TRY(tc_linear(x, tok, pl.C, qw, qb, 1, pl.C, ws + pl.Q, pl.C, 1, reinterpret_cast<int*>(ws + pl.status), st));
  else
    EDIT_TRY(simt_linear(x, tok, pl.C, qw, qb, 1, pl.C, ws + pl.Q, pl.C, 1, st));
  stage_mark(7, st);
  return EDIT_OK;
}

// Step 8: out = per-head (Q_h S_h) / (Q_h z_h + eps).
template <typename T>
int run_apply(const Plan& pl, const edit_attn_weights* w, uint8_t* ws, void* out, cudaStream_t st) {
  int* status = reinterpret_cast<int*>(ws + pl.status);
  if (pl.bf16) {
    TcGemmParams p;
    std::memset(&p, 0, sizeof(p));
    {  // Q as [img][row][head][d], box 64 x 1 x 128 x 1: a head's d columns (the rest reads as zero)
      cuuint64_t dims[4] = {(cuuint64_t)pl.d, (cuuint64_t)pl.heads, (cuuint64_t)pl.HW, (cuuint64_t)pl.B};
      cuuint64_t st3[3] = {(cuuint64_t)pl.d * 2, (cuuint64_t)pl.C * 2, (cuuint64_t)pl.HW * pl.C * 2};
      cuuint32_t box[4] = {64, 1, 128, 1};
      if (!encode(&p.a0, 4, ws + pl.Q, dims, st3, box)) return EDIT_ERR_CUDA;
    }
    p.a1 = p.a0;
    if (!map_b(&p.b0, ws + pl.SzT, pl.KP, static_cast<long>(pl.B) * pl.heads * pl.NP, pl.KP, pl.NP))
      return EDIT_ERR_CUDA;
    p.b1 = p.b2 = p.bk = p.b0;
    p.R = static_cast<int>(pl.HW);
    p.m_tiles_per_img = ceil_div(pl.HW, 128);
    p.num_m_tiles = pl.B * p.m_tiles_per_img;
    p.num_kb = pl.KP / 64;
    p.kb_split = p.num_kb;
    p.n_split = pl.heads * pl.NP;
    p.N = pl.C;
    p.num_n_tiles = pl.heads;
    p.num_tiles = pl.B * p.m_tiles_per_img * pl.heads;
    p.d = pl.d;
    p.heads = pl.heads;
    p.eps = w->attn_eps;
    p.out = out;
    p.ldo = pl.C;
    if (!map_out_heads(&p.out_map, out, pl.C, pl.HW, pl.B, pl.d)) return EDIT_ERR_CUDA;
    p.status = status;
    p.den_out = pl.exact_eta ? reinterpret_cast<float*>(ws + pl.den) : nullptr;
    return gemm_apply(p, pl.NP, st);
  }
  const size_t smem = static_cast<size_t>(pl.d) * (pl.d + 1) * sizeof(float);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(apply_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return EDIT_ERR_CUDA;
  launch_pdl(apply_simt_kernel<T>, dim3(dim3(ceil_div(pl.HW, 128), pl.heads, pl.B)), dim3(128), smem, st, 
      reinterpret_cast<const T*>(ws + pl.Q), reinterpret_cast<const float*>(ws + pl.Sz), static_cast<int>(pl.HW),
      pl.C, pl.heads, w->attn_eps, static_cast<T*>(out),
      pl.exact_eta ? reinterpret_cast<float*>(ws + pl.den) : static_cast<float*>(nullptr));
  return last_launch();
}

template <int D>
int launch_sdpa_simt(const SdpaParams& p, int B, cudaStream_t st) {
  const size_t smem = (128 * D + 128 * (D + 1)) * sizeof(float);
  auto kern = sdpa_blend_kernel<float, D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return EDIT_ERR_CUDA;
  launch_pdl(kern, dim3(dim3(ceil_div(p.Nq, 128), p.heads, B)), dim3(128), smem, st, p);
  return last_launch();
}

// fp32 softmax blocks on the CUDA cores.
int sdpa_simt(const SdpaParams& p, int B, cudaStream_t st) {
  switch (p.d) {
    case 32: return launch_sdpa_simt<32>(p, B, st);
    case 64: return launch_sdpa_simt<64>(p, B, st);
    case 72: return launch_sdpa_simt<72>(p, B, st);
  }
  return EDIT_ERR_UNSUPPORTED;
}

// One key set of a tensor-core softmax launch: K token-major (row stride ld
// elements, n keys per image) and its [V | 1]^T operand (keys padded to nkp).
struct SdpaSet {
  const void* k;
  long ld;
  int n;
  const void* vt;
  int nkp;
};

// Token-major rows seen per head: [rows][heads][d] bf16, box 64 x 1 x 128
// (columns past d, and rows past the end, read as zero).
bool map_head_rows(CUtensorMap* m, const void* base, int d, int heads, long rows, long ld) {
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t st[2] = {(cuuint64_t)d * 2, (cuuint64_t)ld * 2};
  cuuint32_t box[3] = {64, 1, 128};
  return encode(m, 3, base, dims, st, box);
}

// bf16 softmax blocks on the tensor cores (sdpa_tc_kernel): one persistent
// CTA per SM at most (512 TMEM columns, ~200 KB of shared memory each).
template <int D>
int launch_sdpa_tc(const void* q, long ldq, int Nq, const SdpaSet& s1, const SdpaSet* s2, SdpaTcParams p,
                   const Plan& pl, cudaStream_t st) {
  using Cfg = SdpaTcCfg<D>;
  CUtensorMap mq, mk1, mv1, mk2, mv2;
  const long B = pl.B, heads = pl.heads;
  if (!map_head_rows(&mq, q, D, pl.heads, B * Nq, ldq) || !map_head_rows(&mk1, s1.k, D, pl.heads, B * s1.n, s1.ld) ||
      !map_b(&mv1, s1.vt, s1.nkp, B * heads * Cfg::NPV, s1.nkp, Cfg::NPV))
    return EDIT_ERR_CUDA;
  if (s2) {
    if (!map_head_rows(&mk2, s2->k, D, pl.heads, B * s2->n, s2->ld) ||
        !map_b(&mv2, s2->vt, s2->nkp, B * heads * Cfg::NPV, s2->nkp, Cfg::NPV))
      return EDIT_ERR_CUDA;
  } else {
    mk2 = mk1;
    mv2 = mv1;
  }
  p.Nq = Nq;
  p.heads = pl.heads;
  p.nimg = pl.B;
  p.n1 = s1.n;
  p.n2 = s2 ? s2->n : 0;
  auto kern = s2 ? sdpa_tc_kernel<D, 2> : sdpa_tc_kernel<D, 1>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
    return EDIT_ERR_CUDA;
  const long items = B * heads * ceil_div(Nq, 128);
  const int grid = static_cast<int>(items < num_sms() ? items : num_sms());
  launch_pdl(kern, dim3(grid), dim3(320), Cfg::SMEM_BYTES, st, mq, mk1, mv1, mk2, mv2, p);
  return last_launch();
}

int sdpa_tc(const void* q, long ldq, int Nq, const SdpaSet& s1, const SdpaSet* s2, const SdpaTcParams& p,
            const Plan& pl, cudaStream_t st) {
  switch (pl.d) {
    case 32: return launch_sdpa_tc<32>(q, ldq, Nq, s1, s2, p, pl, st);
    case 64: return launch_sdpa_tc<64>(q, ldq, Nq, s1, s2, p, pl, st);
    case 72: return launch_sdpa_tc<72>(q, ldq, Nq, s1, s2, p, pl, st);
  }
  return EDIT_ERR_UNSUPPORTED;
}

// [V | 1]^T of one key set (vt_ones_kernel), keys padded to nkp.
int vt_ones(const void* v, long ldv, int n, int nkp, const Plan& pl, void* vt, cudaStream_t st) {
  const dim3 grid(nkp / 64, pl.heads, pl.B);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  auto* out = static_cast<__nv_bfloat16*>(vt);
  switch (pl.d) {
    case 32: launch_pdl(vt_ones_kernel<32, 48>, grid, dim3(256), 0, st, vb, ldv, n, nkp, pl.heads, out); break;
    case 64: launch_pdl(vt_ones_kernel<64, 80>, grid, dim3(256), 0, st, vb, ldv, n, nkp, pl.heads, out); break;
    case 72: launch_pdl(vt_ones_kernel<72, 80>, grid, dim3(256), 0, st, vb, ldv, n, nkp, pl.heads, out); break;
    default: return EDIT_ERR_UNSUPPORTED;
  }
  return last_launch();
}

// MM-EDiT, prompt side: the prompt projections [Q_P | K_P | V_P] (stage 9).
template <typename T>
int mm_project(const void* x_txt, const Plan& pl, const mmedit_weights* w, uint8_t* ws, cudaStream_t st) {
  int* status = reinterpret_cast<int*>(ws + pl.status);
  const long trow = static_cast<long>(pl.B) * pl.NT;
  const void* wts[3] = {w->tq_w, w->tk_w, w->tv_w};
  const void* bs[3] = {w->tq_b, w->tk_b, w->tv_b};
  if (pl.bf16) {
    EDIT_TRY(tc_linear(x_txt, trow, pl.C, wts, bs, 3, pl.C, ws + pl.QKVt, 3L * pl.C, 0, status, st));
    // [V | 1]^T operands of the softmax blocks: prompt values, then the image's
    // compressed values (token-major V, written by the K/V branch)
    const T* qkv = reinterpret_cast<const T*>(ws + pl.QKVt);
    EDIT_TRY(vt_ones(qkv + 2 * pl.C, 3L * pl.C, pl.NT, pl.nkpP, pl, ws + pl.VTp, st));
    EDIT_TRY(vt_ones(ws + pl.V, pl.C, pl.M, pl.nkpI, pl, ws + pl.VTi, st));
  } else {
    EDIT_TRY(simt_linear(x_txt, trow, pl.C, wts, bs, 3, pl.C, ws + pl.QKVt, 3 * pl.C, 0, st));
  }
  stage_mark(9, st);
  return EDIT_OK;
}

double mm_eta(const Plan& pl) { return static_cast<double>(pl.HW) / static_cast<double>(pl.HW + pl.NT); }

// Image rows: eta * y + (1 - eta) * A(Q_I, K_P, V_P), blended into out_img,
// which holds y (stage 10).
template <typename T>
int mm_image_rows(const Plan& pl, uint8_t* ws, void* out_img, cudaStream_t st) {
  const double eta = mm_eta(pl);
  const T* qkv = reinterpret_cast<const T*>(ws + pl.QKVt);
  if (pl.bf16) {
    SdpaTcParams p;
    std::memset(&p, 0, sizeof(p));
    p.w0 = static_cast<float>(eta);
    p.w1 = static_cast<float>(1.0 - eta);
    p.blend_in = 1;
    p.out = out_img;
    p.ldo = pl.C;
    p.status = reinterpret_cast<int*>(ws + pl.status);
    p.exact = pl.exact_eta ? 1 : 0;
    p.den = reinterpret_cast<const float*>(ws + pl.den);
    const SdpaSet prompt = {qkv + pl.C, 3L * pl.C, pl.NT, ws + pl.VTp, pl.nkpP};
    EDIT_TRY(sdpa_tc(ws + pl.Q, pl.C, static_cast<int>(pl.HW), prompt, nullptr, p, pl, st));
  } else {
    SdpaParams a;
    std::memset(&a, 0, sizeof(a));
    a.q = ws + pl.Q;
    a.ldq = pl.C;
    a.k1 = qkv + pl.C;
    a.v1 = qkv + 2 * pl.C;
    a.ld1 = 3L * pl.C;
    a.n1 = pl.NT;
    a.out = out_img;
    a.ldo = pl.C;
    a.Nq = static_cast<int>(pl.HW);
    a.heads = pl.heads;
    a.d = pl.d;
    a.w0 = static_cast<float>(eta);
    a.w1 = static_cast<float>(1.0 - eta);
    a.blend_in = 1;
    a.exact = pl.exact_eta ? 1 : 0;
    a.den = reinterpret_cast<const float*>(ws + pl.den);
    EDIT_TRY(sdpa_simt(a, pl.B, st));
  }
  stage_mark(10, st);
  return EDIT_OK;
}

// Prompt rows: eta * A(Q_P, K_I, V_I) + (1 - eta) * A(Q_P, K_P, V_P) (stage 11).
template <typename T>
int mm_prompt_rows(const Plan& pl, uint8_t* ws, void* out_txt, cudaStream_t st) {
  const double eta = mm_eta(pl);
  const T* qkv = reinterpret_cast<const T*>(ws + pl.QKVt);
  if (pl.bf16) {
    SdpaTcParams p;
    std::memset(&p, 0, sizeof(p));
    p.w1 = static_cast<float>(eta);
    p.w2 = static_cast<float>(1.0 - eta);
    p.out = out_txt;
    p.ldo = pl.C;
    p.status = reinterpret_cast<int*>(ws + pl.status);
    p.exact = pl.exact_eta ? 1 : 0;
    const SdpaSet image = {ws + pl.K, pl.C, pl.M, ws + pl.VTi, pl.nkpI};
    const SdpaSet prompt = {qkv + pl.C, 3L * pl.C, pl.NT, ws + pl.VTp, pl.nkpP};
    EDIT_TRY(sdpa_tc(qkv, 3L * pl.C, pl.NT, image, &prompt, p, pl, st));
  } else {
    SdpaParams t;
    std::memset(&t, 0, sizeof(t));
    t.q = qkv;
    t.ldq = 3L * pl.C;
    t.k1 = ws + pl.K;
    t.v1 = ws + pl.V;
    t.ld1 = pl.C;
    t.n1 = pl.M;
    t.k2 = qkv + pl.C;
    t.v2 = qkv + 2 * pl.C;
    t.ld2 = 3L * pl.C;
    t.n2 = pl.NT;
    t.out = out_txt;
    t.ldo = pl.C;
    t.Nq = pl.NT;
    t.heads = pl.heads;
    t.d = pl.d;
    t.w1 = static_cast<float>(eta);
    t.w2 = static_cast<float>(1.0 - eta);
    t.exact = pl.exact_eta ? 1 : 0;
    EDIT_TRY(sdpa_simt(t, pl.B, st));
  }
  stage_mark(11, st);
  return EDIT_OK;
}

// MM-EDiT prompt-side work that run_edit may put on the side stream after the
// K/V branch (it needs only K_I, V_I and the prompt tokens): the projections
// and the prompt rows. `done` tells the caller whether it ran there.
struct MmPrompt {
  const void* x_txt;
  const mmedit_weights* w;
  void* out_txt;
  bool done;
};

// One layer: steps 1-8, then (variants with an output Linear) out = Y Wo^T + bo
// from the attention output Y kept in the workspace (stage event 9).
template <typename T>
int run_edit(const void* x, const Plan& pl, const edit_attn_weights* w, uint8_t* ws, void* out, cudaStream_t st,
             const SideStream& side, const edit_attn_variant* var = nullptr, MmPrompt* mm = nullptr) {
  if (cudaMemsetAsync(ws + pl.status, 0, 256, st) != cudaSuccess) return EDIT_ERR_CUDA;
  stage_mark(0, st);
  // Side stream (bf16; stage events time the steps one after the other, so
  // they keep one stream): the query's weight folding, which reads only
  // weights, and for small layers the whole K/V branch. Small layers fork at
  // the start (side: folding, then K/V; main: conv, GroupNorm, query); larger
  // ones fork after the K|V GEMM, so the folding fills SMs the memory-bound
  // depthwise conv leaves idle instead of delaying the GEMM's CTAs. The key
  // ConvFusion shares the folding buffers, so that variant stays serial.
  const bool side_fold = pl.bf16 && pl.q_proc == EDIT_PROC_CF && pl.k_proc != EDIT_PROC_CF;
  const SideStream* ss = (!g_stage_events && (pl.fork || side_fold) && side.s) ? &side : nullptr;
  const bool fold_on_side = ss && side_fold;
  int rkv = EDIT_OK, rq = EDIT_OK, rs = EDIT_OK;
  if (ss && pl.fork) {
    if (cudaEventRecord(ss->fork, st) != cudaSuccess) return EDIT_ERR_CUDA;
  } else if (ss) {
    rkv = run_kv<T>(x, pl, w, var, ws, st, ss->fork);
    if (rkv != EDIT_OK) return rkv;  // nothing was forked yet
  }
  if (ss) {
    if (cudaStreamWaitEvent(ss->s, ss->fork, 0) != cudaSuccess) return EDIT_ERR_CUDA;
    if (fold_on_side) {
      rs = run_fold<T>(pl, query_cf(w), ws, ss->s);
      if (cudaEventRecord(ss->fold, ss->s) != cudaSuccess && rs == EDIT_OK) rs = EDIT_ERR_CUDA;
    }
    if (pl.fork && rs == EDIT_OK) rs = run_kv<T>(x, pl, w, var, ws, ss->s);
    if (cudaEventRecord(ss->kv, ss->s) != cudaSuccess && rs == EDIT_OK) rs = EDIT_ERR_CUDA;
    // MM-EDiT: the prompt projections and prompt rows follow the K/V branch there
    if (pl.fork && mm && pl.NT > 0 && rs == EDIT_OK) {
      rs = mm_project<T>(mm->x_txt, pl, mm->w, ws, ss->s);
      if (rs == EDIT_OK) rs = mm_prompt_rows<T>(pl, ws, mm->out_txt, ss->s);
      mm->done = true;
    }
    if (cudaEventRecord(ss->join, ss->s) != cudaSuccess && rs == EDIT_OK) rs = EDIT_ERR_CUDA;
  } else {
    rkv = run_kv<T>(x, pl, w, var, ws, st);
  }
  if (rkv == EDIT_OK && rs == EDIT_OK)
    rq = run_query<T>(x, pl, w, ws, st, !fold_on_side, fold_on_side ? ss->fold : nullptr);
  int ra = EDIT_OK;
  if (rkv == EDIT_OK && rs == EDIT_OK && rq == EDIT_OK) {
    // (without the fork the side stream holds only the folding, already awaited)
    if (ss && pl.fork && cudaStreamWaitEvent(st, ss->kv, 0) != cudaSuccess) ra = EDIT_ERR_CUDA;
    if (ra == EDIT_OK) ra = run_apply<T>(pl, w, ws, pl.oproj ? static_cast<void*>(ws + pl.Y) : out, st);
  }
  if (ss && cudaStreamWaitEvent(st, ss->join, 0) != cudaSuccess)
    return EDIT_ERR_CUDA;  // (joined even when a step failed: nothing is left running unordered)
  EDIT_TRY(rkv);
  EDIT_TRY(rs);
  EDIT_TRY(rq);
  EDIT_TRY(ra);
  stage_mark(8, st);
  if (pl.oproj) {
    const long tok = static_cast<long>(pl.B) * pl.HW;
    const void* ow[1] = {var->o_w};
    const void* ob[1] = {var->o_b};
    if (pl.bf16)
      EDIT_TRY(tc_linear(ws + pl.Y, tok, pl.C, ow, ob, 1, pl.C, out, pl.C, 0, reinterpret_cast<int*>(ws + pl.status), st));
    else
      EDIT_TRY(simt_linear(ws + pl.Y, tok, pl.C, ow, ob, 1, pl.C, out, pl.C, 0, st));
    stage_mark(9, st);
  }
  return EDIT_OK;
}

template <typename T>
int run_mm(const void* x_img, const void* x_txt, const Plan& pl, const mmedit_weights* w, uint8_t* ws,
           void* out_img, void* out_txt, cudaStream_t st) {
  MmPrompt mm = {x_txt, w, out_txt, false};
  EDIT_TRY(run_edit<T>(x_img, pl, &w->img, ws, out_img, st, side_of(w->side_stream, w->side_events), nullptr, &mm));
  if (pl.NT == 0) return EDIT_OK;  // eta = 1: the image rows are the EDiT layer
  if (!mm.done) EDIT_TRY(mm_project<T>(x_txt, pl, w, ws, st));
  EDIT_TRY(mm_image_rows<T>(pl, ws, out_img, st));
  if (!mm.done) EDIT_TRY(mm_prompt_rows<T>(pl, ws, out_txt, st));
  return EDIT_OK;
}

// ------------------------------------------------------------ row bands
// One image split into horizontal bands of rows, one per rank. Layout of a
// band's workspace: the plan `pe` of the band with its halo rows as one image
// (conv3x3, U, G, GroupNorm partials, weight folding, K'|V' of the band and its
// upper halo row), then the plan `pq` of the band's own rows (compressed K, V,
// KV state, Q, the apply operand), whose offsets are shifted past pe's.
struct BandPlan {
  Plan pe, pq;
  int H, row0, rows, top, bot;
  size_t rec_bytes, sz_off, total;
};

// The record a band contributes to the two global reductions: fp64 GroupNorm
// sums [groups][2] at byte 0, fp32 [S | z] [heads][d][d + 1] at sz_off.
size_t band_record_layout(int groups, int heads, int d, size_t* sz_off) {
  *sz_off = align_up(static_cast<size_t>(groups) * 2 * sizeof(double), 256);
  return align_up(*sz_off + static_cast<size_t>(heads) * d * (d + 1) * sizeof(float), 256);
}

int make_band_plan(int W, int C, int heads, const edit_band* band, const edit_attn_weights* w, BandPlan& bp) {
  if (!band || !w) return EDIT_ERR_NULL;
  if (w->dtype != EDIT_F32 && w->dtype != EDIT_BF16) return EDIT_ERR_DTYPE;
  if (w->dtype != EDIT_BF16) return EDIT_ERR_UNSUPPORTED;
  const int H = band->H, r0 = band->row0, rows = band->rows;
  if (H < 1 || rows < 1 || r0 < 0 || r0 > H - rows) return EDIT_ERR_SHAPE;
  // band boundaries on even rows: no stride-2 key/value token straddles two bands
  if (r0 % 2 != 0 || (r0 + rows != H && (r0 + rows) % 2 != 0)) return EDIT_ERR_SHAPE;
  bp.H = H;
  bp.row0 = r0;
  bp.rows = rows;
  bp.top = r0 > 0 ? 1 : 0;
  bp.bot = r0 + rows < H ? 1 : 0;
  EDIT_TRY_CHECK(make_plan(1, rows + bp.top + bp.bot, W, C, heads, 0, w, bp.pe));
  EDIT_TRY_CHECK(make_plan(1, rows, W, C, heads, 0, w, bp.pq));
  const size_t sh = bp.pe.total;
  Plan& q = bp.pq;
  q.status = bp.pe.status;
  q.KT += sh;
  q.VTx += sh;
  q.kvpart += sh;
  q.Sz += sh;
  q.SzT += sh;
  q.Q += sh;
  bp.total = bp.pe.total + q.total;
  bp.rec_bytes = band_record_layout(bp.pe.G, heads, bp.pe.d, &bp.sz_off);
  return EDIT_OK;
}

// Band step 1: its rows' compressed K, V and partial [S | z]; U of the band
// with its halo rows and the band rows' GroupNorm sums. Writes the record.
int run_band_partials(const void* x, const BandPlan& bp, const edit_attn_weights* w, uint8_t* ws, uint8_t* rec,
                      cudaStream_t st) {
  const Plan& pe = bp.pe;
  const Plan& pq = bp.pq;
  int* status = reinterpret_cast<int*>(ws + pe.status);
  if (cudaMemsetAsync(ws + pe.status, 0, 256, st) != cudaSuccess) return EDIT_ERR_CUDA;
  const int W = pe.W, C = pe.C, Cr = pe.Cr;
  // K'|V' of the band's rows and its upper halo row; the depthwise conv reads
  // them with that halo as row 0 (output row i: rows 2i - 1 + top .. 2i + 1 + top)
  const long tokkv = static_cast<long>(bp.rows + bp.top) * W;
  const void* wts[2] = {w->k_w, w->v_w};
  const void* bs[2] = {w->k_b, w->v_b};
  EDIT_TRY(tc_linear(x, tokkv, C, wts, bs, 2, C, ws + pe.KVp, 2L * C, 0, status, st));
  Plan pk = pq;  // the K'|V' rows live in pe's buffer
  pk.KVp = pe.KVp;
  EDIT_TRY(dwconv_tc(pk, w, ws, bp.rows + bp.top, bp.top, st));
  EDIT_TRY(kv_state_tc(pq, ws, st));
  const int per_head = pq.d * (pq.d + 1);
  const long total = static_cast<long>(pq.heads) * per_head;
  launch_pdl(kv_state_combine_kernel, dim3(grid_for(total, 256)), dim3(256), 0, st,
             reinterpret_cast<const float*>(ws + pq.kvpart), pq.kv_chunks, per_head, total,
             reinterpret_cast<float*>(rec + bp.sz_off));
  EDIT_TRY(last_launch());
  // U of the band with its halo rows (the halo rows' own outputs are not used)
  EDIT_TRY(conv3x3_tc(x, pe, query_cf(w), ws, st, false, nullptr));
  const __nv_bfloat16* Ub = reinterpret_cast<const __nv_bfloat16*>(ws + pe.U) + static_cast<long>(bp.top) * W * Cr;
  float* gnpart = reinterpret_cast<float*>(ws + pe.gnpart);
  launch_pdl(gn_partial_kernel<__nv_bfloat16>, dim3(dim3(pq.gn_P, 1)), dim3(256), 0, st, Ub,
             static_cast<int>(pq.HW), Cr, pe.G, pq.gn_P, gnpart);
  EDIT_TRY(last_launch());
  launch_pdl(gn_band_sums_kernel, dim3(pe.G), dim3(256), 0, st, static_cast<const float*>(gnpart), pq.gn_P, pe.G,
             reinterpret_cast<double*>(rec));
  return last_launch();
}

// Band step 2: the global GroupNorm statistics and [S | z] from every band's
// record (summed in band order), then G, the query and the attention output of
// the band's rows.
int run_band_finish(const void* x, const BandPlan& bp, const edit_attn_weights* w, uint8_t* ws, const uint8_t* recs,
                    int nrec, void* out, cudaStream_t st) {
  const Plan& pe = bp.pe;
  const Plan& pq = bp.pq;
  const int W = pe.W, C = pe.C, Cr = pe.Cr;
  const long count = static_cast<long>(bp.H) * W * (Cr / pe.G);
  launch_pdl(gn_band_finalize_kernel, dim3(pe.G), dim3(64), 0, st, recs, nrec, static_cast<long>(bp.rec_bytes), pe.G,
             Cr, count, w->gn_eps, static_cast<const __nv_bfloat16*>(w->gn_gamma),
             static_cast<const __nv_bfloat16*>(w->gn_beta), reinterpret_cast<float*>(ws + pe.gnstats),
             reinterpret_cast<float*>(ws + pe.gnss));
  EDIT_TRY(last_launch());
  const long tok = pq.HW;
  {
    const int nvec = Cr / 8;
    const int per_block = 256 / nvec > 0 ? 256 / nvec : 1;
    launch_pdl(gn_apply_leaky_bf16x8, gn_apply_grid(tok, 1, per_block), dim3(per_block * nvec), 0, st,
               reinterpret_cast<const __nv_bfloat16*>(ws + pe.U) + static_cast<long>(bp.top) * W * Cr,
               reinterpret_cast<const float*>(ws + pe.gnss), tok, Cr, w->leaky_slope,
               reinterpret_cast<__nv_bfloat16*>(ws + pe.Gb));
    EDIT_TRY(last_launch());
  }
  const CfWeights cf = query_cf(w);
  EDIT_TRY(run_fold<__nv_bfloat16>(pe, cf, ws, st));
  const void* xb = static_cast<const __nv_bfloat16*>(x) + static_cast<long>(bp.top) * W * C;
  EDIT_TRY(query_gemm_tc(xb, tok, pe, cf, ws + pe.Gb, ws, ws + pq.Q, C, st));
  const long total_t = static_cast<long>(pq.heads) * pq.NP * pq.KP;
  launch_pdl(sz_band_combine_pack_kernel, dim3(grid_for(total_t, 256)), dim3(256), 0, st, recs, nrec,
             static_cast<long>(bp.rec_bytes), static_cast<long>(bp.sz_off), pq.d, pq.NP, pq.KP, total_t,
             reinterpret_cast<float*>(ws + pq.Sz), reinterpret_cast<__nv_bfloat16*>(ws + pq.SzT));
  EDIT_TRY(last_launch());
  return run_apply<__nv_bfloat16>(pq, w, ws, out, st);
}

int band_checks(const void* x, const edit_attn_weights* w, const BandPlan& bp) {
  if (!x) return EDIT_ERR_NULL;
  EDIT_TRY_CHECK(check_weights(w, bp.pe));
  if (!aligned(x, 16)) return EDIT_ERR_ALIGN;
  if (!w->workspace) return EDIT_ERR_NULL;
  if (!aligned(w->workspace, 256)) return EDIT_ERR_ALIGN;
  if (w->workspace_bytes < bp.total) return EDIT_ERR_WORKSPACE;
  return EDIT_OK;
}

// ------------------------------------------------------------ DiT block
// The block around the attention: LayerNorm modulation, the EDiT layer with
// its output Linear, gated residuals, cross-attention over the caption tokens
// and the tanh-GELU MLP. Workspace: the EDiT layer's (plan `pa`, its variant
// with the output Linear) at offset 0, then the block's token buffers.
struct DitPlan {
  Plan pa;
  int NT, hidden, nkp;
  size_t h1, x1, q, kv, vt, att, c, x2, h2, f, m, total;
};

edit_attn_variant dit_attn_variant(const edit_dit_block_weights* w) {
  edit_attn_variant v;
  std::memset(&v, 0, sizeof(v));
  v.q_proc = EDIT_PROC_CF;
  v.k_proc = EDIT_PROC_SC;
  v.v_proc = EDIT_PROC_SC;
  v.o_w = w->o_w;
  v.o_b = w->o_b;
  return v;
}

int make_dit_plan(int B, int H, int W, int NT, int C, int heads, const edit_dit_block_weights* w, DitPlan& dp) {
  if (!w) return EDIT_ERR_NULL;
  const edit_attn_variant var = dit_attn_variant(w);
  EDIT_TRY_CHECK(make_plan(B, H, W, C, heads, 0, &w->attn, dp.pa, &var));
  const Plan& pa = dp.pa;
  if (NT < 1 || w->hidden < 1) return EDIT_ERR_SHAPE;
  if (!(pa.d == 32 || pa.d == 64 || pa.d == 72)) return EDIT_ERR_UNSUPPORTED;
  if (pa.bf16 && w->hidden % 128 != 0) return EDIT_ERR_UNSUPPORTED;
  if (!pa.bf16 && (C % 8 != 0 || w->hidden % 4 != 0)) return EDIT_ERR_UNSUPPORTED;
  if (C > 2048) return EDIT_ERR_UNSUPPORTED;  // the residual / LayerNorm kernel keeps a row in registers
  dp.NT = NT;
  dp.hidden = w->hidden;
  dp.nkp = (NT + 127) / 128 * 128;
  const size_t es = pa.es, tok = static_cast<size_t>(B) * pa.HW;
  size_t off = pa.total;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  dp.h1 = take(tok * C * es);
  dp.x1 = take(tok * C * es);
  dp.q = take(tok * C * es);
  dp.kv = take(static_cast<size_t>(B) * NT * 2 * C * es);
  dp.vt = pa.bf16 ? take(static_cast<size_t>(B) * heads * (pa.d + 1 <= 48 ? 48 : 80) * dp.nkp * 2) : 0;
  dp.att = take(tok * C * es);
  dp.c = take(tok * C * es);
  dp.x2 = take(tok * C * es);
  dp.h2 = take(tok * C * es);
  dp.f = take(tok * w->hidden * es);
  dp.m = take(tok * C * es);
  dp.total = off;
  return EDIT_OK;
}

template <typename T>
int dit_residual_ln(const Plan& pl, const void* base, const void* delta, const void* sst, const void* t6, int kg,
                    int ks, int kh, float eps, void* r_out, void* h_out, cudaStream_t st) {
  const long rows = static_cast<long>(pl.B) * pl.HW;
  launch_pdl(dit_residual_ln_kernel<T>, dim3(grid_for(rows * 32, 256)), dim3(256), 0, st,
             static_cast<const T*>(base), static_cast<const T*>(delta), static_cast<const T*>(sst),
             static_cast<const T*>(t6), kg, ks, kh, static_cast<long>(pl.HW), rows, pl.C, eps, static_cast<T*>(r_out),
             static_cast<T*>(h_out));
  return last_launch();
}

// out[rows][n] = act(a[rows][K] w^T + b), rows ldo elements apart
template <typename T>
int linear_any(const Plan& pl, const void* a, long rows, int K, const void* w, const void* b, int n, void* out,
               long ldo, int act, int* status, cudaStream_t st) {
  const void* ws1[1] = {w};
  const void* bs1[1] = {b};
  if (pl.bf16) return tc_linear(a, rows, K, ws1, bs1, 1, n, out, ldo, act, status, st);
  return simt_linear(a, rows, K, ws1, bs1, 1, n, out, static_cast<int>(ldo), act, st);
}

template <typename T>
int run_dit(const void* x, const void* y, const void* t6, const DitPlan& dp, const edit_dit_block_weights* w,
            uint8_t* ws, void* out, cudaStream_t st) {
  const Plan& pa = dp.pa;
  const int C = pa.C;
  const long tok = static_cast<long>(pa.B) * pa.HW, trow = static_cast<long>(pa.B) * dp.NT;
  int* status = reinterpret_cast<int*>(ws + pa.status);
  // h1 = LN(x) (1 + scale_a) + shift_a
  EDIT_TRY(dit_residual_ln<T>(pa, x, nullptr, w->sst, t6, -1, 1, 0, w->ln_eps, nullptr, ws + dp.h1, st));
  // a = EDiT(h1) o_w^T + o_b (resets the status block)
  edit_attn_weights aw = w->attn;
  aw.workspace = ws;
  aw.workspace_bytes = dp.pa.total;
  const edit_attn_variant var = dit_attn_variant(w);
  EDIT_TRY(run_edit<T>(ws + dp.h1, pa, &aw, ws, ws + dp.att, st, side_of(w->side_stream, w->side_events), &var));
  // x1 = x + gate_a a
  EDIT_TRY(dit_residual_ln<T>(pa, x, ws + dp.att, w->sst, t6, 2, 0, 0, w->ln_eps, ws + dp.x1, nullptr, st));
  // cross-attention over the caption tokens
  EDIT_TRY(linear_any<T>(pa, ws + dp.x1, tok, C, w->cq_w, w->cq_b, C, ws + dp.q, C, ACT_NONE, status, st));
  {
    const void* kvw[2] = {w->ck_w, w->cv_w};
    const void* kvb[2] = {w->ck_b, w->cv_b};
    if (pa.bf16)
      EDIT_TRY(tc_linear(y, trow, C, kvw, kvb, 2, C, ws + dp.kv, 2L * C, 0, status, st));
    else
      EDIT_TRY(simt_linear(y, trow, C, kvw, kvb, 2, C, ws + dp.kv, 2 * C, 0, st));
  }
  const T* kv = reinterpret_cast<const T*>(ws + dp.kv);
  if (pa.bf16) {
    EDIT_TRY(vt_ones(kv + C, 2L * C, dp.NT, dp.nkp, pa, ws + dp.vt, st));
    SdpaTcParams p;
    std::memset(&p, 0, sizeof(p));
    p.w1 = 1.f;
    p.out = ws + dp.att;
    p.ldo = C;
    p.status = status;
    const SdpaSet cap = {kv, 2L * C, dp.NT, ws + dp.vt, dp.nkp};
    EDIT_TRY(sdpa_tc(ws + dp.q, C, static_cast<int>(pa.HW), cap, nullptr, p, pa, st));
  } else {
    SdpaParams a;
    std::memset(&a, 0, sizeof(a));
    a.q = ws + dp.q;
    a.ldq = C;
    a.k1 = kv;
    a.v1 = kv + C;
    a.ld1 = 2L * C;
    a.n1 = dp.NT;
    a.out = ws + dp.att;
    a.ldo = C;
    a.Nq = static_cast<int>(pa.HW);
    a.heads = pa.heads;
    a.d = pa.d;
    a.w1 = 1.f;
    EDIT_TRY(sdpa_simt(a, pa.B, st));
  }
  EDIT_TRY(linear_any<T>(pa, ws + dp.att, tok, C, w->co_w, w->co_b, C, ws + dp.c, C, ACT_NONE, status, st));
  // x2 = x1 + c; h2 = LN(x2) (1 + scale_f) + shift_f
  EDIT_TRY(dit_residual_ln<T>(pa, ws + dp.x1, ws + dp.c, w->sst, t6, -1, 4, 3, w->ln_eps, ws + dp.x2, ws + dp.h2, st));
  // MLP: f = GELU(h2 fc1^T + b1), m = f fc2^T + b2; out = x2 + gate_f m
  EDIT_TRY(linear_any<T>(pa, ws + dp.h2, tok, C, w->fc1_w, w->fc1_b, dp.hidden, ws + dp.f, dp.hidden, ACT_GELU,
                         status, st));
  EDIT_TRY(linear_any<T>(pa, ws + dp.f, tok, dp.hidden, w->fc2_w, w->fc2_b, C, ws + dp.m, C, ACT_NONE, status, st));
  return dit_residual_ln<T>(pa, ws + dp.x2, ws + dp.m, w->sst, t6, 5, 0, 0, w->ln_eps, out, nullptr, st);
}

int dit_checks(const void* x, const void* y, const void* t6, const void* out, const edit_dit_block_weights* w,
               const DitPlan& dp) {
  if (!x || !y || !t6 || !out || !w->workspace) return EDIT_ERR_NULL;
  const edit_attn_variant var = dit_attn_variant(w);
  EDIT_TRY_CHECK(check_weights(&w->attn, dp.pa, &var));
  const void* blk[] = {w->sst, w->cq_w, w->cq_b, w->ck_w, w->ck_b, w->cv_w, w->cv_b, w->co_w, w->co_b,
                       w->fc1_w, w->fc1_b, w->fc2_w, w->fc2_b};
  EDIT_TRY_CHECK(check_ptrs(blk, 13));
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(t6, 16) || !aligned(out, 16)) return EDIT_ERR_ALIGN;
  if (!aligned(w->workspace, 256)) return EDIT_ERR_ALIGN;
  if (w->workspace_bytes < dp.total) return EDIT_ERR_WORKSPACE;
  return check_side(w->side_stream, w->side_events);
}

int common_checks(const void* x, const void* out, const edit_attn_weights* w, void* ws, size_t ws_bytes,
                  const Plan& pl, const edit_attn_variant* var = nullptr) {
  if (!x || !out || !ws) return EDIT_ERR_NULL;
  EDIT_TRY(check_weights(w, pl, var));
  if (!aligned(x, 16) || !aligned(out, 16)) return EDIT_ERR_ALIGN;
  if (!aligned(ws, 256)) return EDIT_ERR_ALIGN;
  if (ws_bytes < pl.total) return EDIT_ERR_WORKSPACE;
  return EDIT_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

size_t edit_attn_workspace_bytes(int B, int H, int W, int C, int heads, const edit_attn_weights* w) {
  Plan pl;
  return make_plan(B, H, W, C, heads, 0, w, pl) == EDIT_OK ? pl.total : 0;
}

int edit_attn_forward(const void* x, int B, int H, int W, int C, int heads, const edit_attn_weights* w, void* out,
                      void* stream) {
  Plan pl;
  EDIT_TRY(make_plan(B, H, W, C, heads, 0, w, pl));
  EDIT_TRY(common_checks(x, out, w, w->workspace, w->workspace_bytes, pl));
  EDIT_TRY(check_side(w->side_stream, w->side_events));
  uint8_t* ws = static_cast<uint8_t*>(w->workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const SideStream side = side_of(w->side_stream, w->side_events);
  return pl.bf16 ? run_edit<__nv_bfloat16>(x, pl, w, ws, out, st, side)
                 : run_edit<float>(x, pl, w, ws, out, st, side);
}

size_t edit_attn_variant_workspace_bytes(int B, int H, int W, int C, int heads, const edit_attn_weights* w,
                                         const edit_attn_variant* var) {
  if (!var) return 0;
  Plan pl;
  return make_plan(B, H, W, C, heads, 0, w, pl, var) == EDIT_OK ? pl.total : 0;
}

int edit_attn_variant_forward(const void* x, int B, int H, int W, int C, int heads, const edit_attn_weights* w,
                              const edit_attn_variant* var, void* out, void* stream) {
  if (!var) return EDIT_ERR_NULL;
  Plan pl;
  EDIT_TRY(make_plan(B, H, W, C, heads, 0, w, pl, var));
  EDIT_TRY(common_checks(x, out, w, w->workspace, w->workspace_bytes, pl, var));
  EDIT_TRY(check_side(w->side_stream, w->side_events));
  uint8_t* ws = static_cast<uint8_t*>(w->workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const SideStream side = side_of(w->side_stream, w->side_events);
  return pl.bf16 ? run_edit<__nv_bfloat16>(x, pl, w, ws, out, st, side, var)
                 : run_edit<float>(x, pl, w, ws, out, st, side, var);
}

size_t mmedit_workspace_bytes(int B, int H, int W, int N_T, int C, int heads, const mmedit_weights* w) {
  if (!w) return 0;
  Plan pl;
  return make_plan(B, H, W, C, heads, N_T, &w->img, pl) == EDIT_OK ? pl.total : 0;
}

int mmedit_hybrid_forward(const void* x_img, const void* x_txt, int B, int H, int W, int N_T, int C, int heads,
                          const mmedit_weights* w, void* out_img, void* out_txt, void* stream) {
  if (!w) return EDIT_ERR_NULL;
  Plan pl;
  EDIT_TRY(make_plan(B, H, W, C, heads, N_T, &w->img, pl));
  EDIT_TRY(common_checks(x_img, out_img, &w->img, w->workspace, w->workspace_bytes, pl));
  EDIT_TRY(check_side(w->side_stream, w->side_events));
  if (N_T > 0) {
    if (!x_txt || !out_txt) return EDIT_ERR_NULL;
    if (!aligned(x_txt, 16) || !aligned(out_txt, 16)) return EDIT_ERR_ALIGN;
    const void* tp[] = {w->tq_w, w->tq_b, w->tk_w, w->tk_b, w->tv_w, w->tv_b};
    for (const void* p : tp) {
      if (!p) return EDIT_ERR_NULL;
      if (!aligned(p, 16)) return EDIT_ERR_ALIGN;
    }
  }
  if (w->eta_mode != EDIT_ETA_RATIO && w->eta_mode != EDIT_ETA_EXACT) return EDIT_ERR_UNSUPPORTED;
  pl.exact_eta = w->eta_mode == EDIT_ETA_EXACT && N_T > 0;
  uint8_t* ws = static_cast<uint8_t*>(w->workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return pl.bf16 ? run_mm<__nv_bfloat16>(x_img, x_txt, pl, w, ws, out_img, out_txt, st)
                 : run_mm<float>(x_img, x_txt, pl, w, ws, out_img, out_txt, st);
}

int edit_attn_read_status(const void* workspace, void* stream, int* status) {
  if (!workspace || !status) return EDIT_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(status, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return EDIT_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return EDIT_ERR_CUDA;
  return EDIT_OK;
}

size_t edit_attn_band_workspace_bytes(int W, int C, int heads, const edit_band* band, const edit_attn_weights* w) {
  BandPlan bp;
  return make_band_plan(W, C, heads, band, w, bp) == EDIT_OK ? bp.total : 0;
}

size_t edit_attn_band_record_bytes(int C, int heads, const edit_attn_weights* w) {
  if (!w || heads < 1 || C % heads != 0 || w->gn_groups < 1) return 0;
  size_t sz_off = 0;
  return band_record_layout(w->gn_groups, heads, C / heads, &sz_off);
}

int edit_attn_band_partials(const void* x_ext, int W, int C, int heads, const edit_band* band,
                            const edit_attn_weights* w, void* record, void* stream) {
  BandPlan bp;
  EDIT_TRY(make_band_plan(W, C, heads, band, w, bp));
  EDIT_TRY(band_checks(x_ext, w, bp));
  if (!record) return EDIT_ERR_NULL;
  if (!aligned(record, 256)) return EDIT_ERR_ALIGN;
  return run_band_partials(x_ext, bp, w, static_cast<uint8_t*>(w->workspace), static_cast<uint8_t*>(record),
                           static_cast<cudaStream_t>(stream));
}

int edit_attn_band_finish(const void* x_ext, int W, int C, int heads, const edit_band* band,
                          const edit_attn_weights* w, const void* records, int nrecords, void* out, void* stream) {
  BandPlan bp;
  EDIT_TRY(make_band_plan(W, C, heads, band, w, bp));
  EDIT_TRY(band_checks(x_ext, w, bp));
  if (!records || !out) return EDIT_ERR_NULL;
  if (nrecords < 1 || nrecords > (bp.H + 1) / 2) return EDIT_ERR_SHAPE;
  if (!aligned(records, 256) || !aligned(out, 16)) return EDIT_ERR_ALIGN;
  return run_band_finish(x_ext, bp, w, static_cast<uint8_t*>(w->workspace), static_cast<const uint8_t*>(records),
                         nrecords, out, static_cast<cudaStream_t>(stream));
}

size_t edit_dit_block_workspace_bytes(int B, int H, int W, int N_T, int C, int heads,
                                      const edit_dit_block_weights* w) {
  DitPlan dp;
  return make_dit_plan(B, H, W, N_T, C, heads, w, dp) == EDIT_OK ? dp.total : 0;
}

int edit_dit_block_forward(const void* x, const void* y, const void* t6, int B, int H, int W, int N_T, int C,
                           int heads, const edit_dit_block_weights* w, void* out, void* stream) {
  DitPlan dp;
  EDIT_TRY(make_dit_plan(B, H, W, N_T, C, heads, w, dp));
  EDIT_TRY(dit_checks(x, y, t6, out, w, dp));
  uint8_t* ws = static_cast<uint8_t*>(w->workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dp.pa.bf16 ? run_dit<__nv_bfloat16>(x, y, t6, dp, w, ws, out, st)
                    : run_dit<float>(x, y, t6, dp, w, ws, out, st);
}

const char* edit_status_string(int status) {
  switch (status) {
    case EDIT_OK: return "ok";
    case EDIT_ERR_NULL: return "null pointer";
    case EDIT_ERR_SHAPE: return "bad shape";
    case EDIT_ERR_ALIGN: return "misaligned pointer";
    case EDIT_ERR_DTYPE: return "unsupported dtype";
    case EDIT_ERR_WORKSPACE: return "workspace too small";
    case EDIT_ERR_CUDA: return "CUDA error";
    case EDIT_ERR_TIMEOUT: return "device wait timed out";
    case EDIT_ERR_UNSUPPORTED: return "shape not supported by the kernels";
    case EDIT_ERR_SCRATCH: return "request exceeds the library's fixed scratch";
  }
  return "unknown status";
}

int edit_attn_workspace_layout(int B, int H, int W, int C, int heads, const edit_attn_weights* w,
                               edit_ws_layout* layout) {
  return edit_attn_variant_workspace_layout(B, H, W, C, heads, w, nullptr, layout);
}

int edit_attn_variant_workspace_layout(int B, int H, int W, int C, int heads, const edit_attn_weights* w,
                                       const edit_attn_variant* var, edit_ws_layout* layout) {
  if (!layout) return EDIT_ERR_NULL;
  Plan pl;
  EDIT_TRY(make_plan(B, H, W, C, heads, 0, w, pl, var));
  layout->status = static_cast<int64_t>(pl.status);
  layout->U = static_cast<int64_t>(pl.U);
  layout->G = static_cast<int64_t>(pl.Gb);
  layout->Q = static_cast<int64_t>(pl.Q);
  layout->KVp = static_cast<int64_t>(pl.KVp);
  layout->K = static_cast<int64_t>(pl.K);
  layout->V = static_cast<int64_t>(pl.V);
  layout->gn_stats = static_cast<int64_t>(pl.gnstats);
  layout->Sz = static_cast<int64_t>(pl.Sz);
  layout->KT = pl.KT ? static_cast<int64_t>(pl.KT) : -1;
  layout->VTx = pl.VTx ? static_cast<int64_t>(pl.VTx) : -1;
  layout->K = pl.K ? static_cast<int64_t>(pl.K) : -1;
  layout->V = pl.V ? static_cast<int64_t>(pl.V) : -1;
  layout->Mp = pl.bf16 ? pl.Mp : pl.M;
  layout->Wop = pl.bf16 ? pl.Wop : pl.Wo;
  layout->NP = pl.bf16 ? pl.NP : 0;
  return EDIT_OK;
}

int edit_attn_set_stage_events(void* const* events, int n) {
  if (n < 0) return EDIT_ERR_SHAPE;
  g_stage_events = events;
  g_stage_n = events ? n : 0;
  return EDIT_OK;
}

uint64_t edit_attn_kernel_launches(void) { return g_launches; }

int edit_attn_set_wait_drill(int gn_extra_arrivals, uint64_t limit_ns) {
  if (gn_extra_arrivals < 0 || gn_extra_arrivals > 1024) return EDIT_ERR_SHAPE;
  if (gn_extra_arrivals > 0 && (limit_ns < 1000ull || limit_ns > EDIT_WAIT_TIMEOUT_NS)) return EDIT_ERR_SHAPE;
  g_drill_extra = gn_extra_arrivals;
  g_drill_limit_ns = gn_extra_arrivals > 0 ? limit_ns : 0;
  return EDIT_OK;
}

}  // extern "C"

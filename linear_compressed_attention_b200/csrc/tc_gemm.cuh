// tcgen05 / TMEM / TMA GEMM for the dense contractions of the EDiT layer.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]      (bf16 in, fp32 accumulate in TMEM)
//
// Three epilogues share one main loop:
//  EPI_LINEAR  Linear projections (section "Spatial Compressor", eq. phi_SC;
//              the Linear of eq. Q^EDiT): + bias, optional ReLU, bf16 store.
//  EPI_CONV    ConvFusion 3x3 conv as an implicit GEMM over the token grid
//              (K = 9 * C_in, one shifted TMA box per tap; the box's
//              out-of-grid rows/columns are zero-filled by TMA, which is
//              exactly the conv's zero padding): + bias, bf16 store of U.
//  EPI_APPLY   Linear attention apply, eq. (y_i): per head h, [num | den] =
//              Q_h [S_h | z_h] and y = num / (den + eps) fused into the store.
//  EPI_KVSTATE Linear attention state, eq. (y_i): per (image, head, chunk of
//              compressed tokens) tile, D = K_h^T [V_h | 1 | 0] with the
//              tokens as the reduction dimension (both operands stored
//              channel-major, so K-major for the MMA); rows a < d, columns
//              c <= d of D are a partial [S_h | z_h], written in fp32 for a
//              fixed-order combine.
//
// Block: 192 threads. Warp 0 = TMA producer (one lane), warp 1 = TMEM owner
// and MMA issuer (one lane), warps 2..5 = epilogue (tcgen05.ld of the warp's
// lane quarter, one tile row per thread). Persistent over tiles; STAGES-deep
// shared-memory ring guarded by full/empty mbarriers; one or two TMEM
// accumulators so the epilogue of tile t overlaps the main loop of t+1.
// No cluster, no multicast.
#pragma once

#include "common.cuh"

namespace edit {

enum { EPI_LINEAR = 0, EPI_CONV = 1, EPI_APPLY = 2, EPI_KVSTATE = 3 };

struct TcGemmParams {
  // A sources (3D maps [img][rows][K], box 64 x 128 x 1): a0 gives the first
  // kb_split k-blocks, a1 the rest. EPI_CONV: a0 is the 4D grid map
  // [B][H][W][C] with box 64 x TW x TH x 1.
  CUtensorMap a0, a1;
  // B sources (2D maps [rows][K], box 64 x NCHUNK): b[s] holds output columns
  // [s*n_split, (s+1)*n_split) for the first kb_split k-blocks; bk holds the
  // rest of K (single N source only). EPI_APPLY: b0 = [img*heads*BN][KP].
  CUtensorMap b0, b1, b2, bk;
  // Output map for the staged (TMA store) epilogue of the pair kernel:
  // EPI_LINEAR: 2D [rows][N] box 64 x 32; EPI_CONV: 4D [img][H][W][Cr] box
  // 64 x min(TW,32) x (32/min(TW,32)) x 1. Both 128-byte swizzled.
  CUtensorMap out_map;
  int R;            // rows per image (A)
  int m_tiles_per_img;
  int num_m_tiles;  // real 128-row tiles (the pair kernel may add one empty tile)
  int num_kb;       // 64-wide k-blocks
  int kb_split;
  int n_split;
  int N;            // output columns (EPI_LINEAR masks columns >= N)
  int num_n_tiles;
  int num_tiles;
  // implicit-conv geometry (EPI_CONV)
  int H, W, TH, TW, tiles_h, tiles_w, kb_per_tap;
  // apply / KV-state geometry (EPI_APPLY, EPI_KVSTATE)
  int d, heads;
  float eps;
  int kb_per_chunk, num_chunks;
  // tap-reuse conv: pair tiles [split_first, split_first + split_count) run as
  // two half items over the input-channel blocks, writing fp32 partials to
  // fix_part [(split tile * 2 + half) * 2 + rank][N / 4][128][4] (summed with
  // the bias afterwards)
  int split_first, split_count;
  float* fix_part;
  // per-tap conv (pair kernel, EPI_CONV): ksplit > 1 splits every tile's
  // k-blocks into ksplit parts; item it = tile it / ksplit, part it % ksplit,
  // whose fp32 partial goes to fix_part [item][rank][N / 4][128][4]
  int ksplit;
  float* kv_part;       // EPI_KVSTATE: [img][heads][num_chunks][d][d+1]
  // epilogue
  void* out;        // bf16, row (img*R + r) at out + row*ldo (+ column offset)
  long ldo;
  const void* bias[3];
  int bias_f32;
  int relu;  // epilogue activation: ACT_NONE, ACT_RELU or ACT_GELU
  int* status;
  float* den_out;  // EPI_APPLY: when set, den + eps per row and head, [img][R][heads] fp32
  // EPI_CONV: when set, the GroupNorm column sums of the stored U (bf16 values):
  // gn_col[img][tile * 4 + row / 32][N][2] = (sum, sum of squares) over rows
  // 32 (row / 32) .. + 31 of the image's 128-pixel tile `tile` (pixels outside
  // the image add nothing). Tiles split over k get theirs from the fixup kernel.
  float* gn_col;

};

template <int BN, int NSPLIT, int STAGES, int STG = 0>
struct TcGemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int NCHUNK = BN / NSPLIT;
  static_assert(BN % NSPLIT == 0 && NCHUNK % 16 == 0 && NCHUNK <= 256, "bad MMA N");
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static_assert(B_BYTES % 1024 == 0 && (NCHUNK * 128) % 1024 == 0, "1024-byte operand alignment");
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC = (2 * BN <= 512) ? 2 : 1;
  static constexpr int TMEM_COLS = (ACC * BN <= 32) ? 32 : (ACC * BN <= 64) ? 64 : (ACC * BN <= 128) ? 128
                                   : (ACC * BN <= 256) ? 256 : 512;
  static_assert(ACC * BN <= 512, "TMEM");
  static constexpr int STG_BYTES = STG;  // epilogue staging (EPI_APPLY)
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * ACC) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STG_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, NCHUNK);
};




struct TileCoord {
  int m_tile, n_tile, img, r0, h0, w0;
  int kb0, nkb;  // k-block range of this tile
};

template <int EPI>
__device__ __forceinline__ TileCoord decode_m(const TcGemmParams& p, TileCoord t);

template <int EPI>
__device__ __forceinline__ TileCoord decode_tile(const TcGemmParams& p, int tile) {
  TileCoord t;
  t.kb0 = 0;
  t.nkb = p.num_kb;
  if (EPI == EPI_KVSTATE) {  // tile = (img * heads + head) * num_chunks + chunk
    const int chunk = tile % p.num_chunks;
    const int ih = tile / p.num_chunks;
    t.img = ih / p.heads;
    t.n_tile = ih - t.img * p.heads;
    t.m_tile = chunk;
    t.kb0 = chunk * p.kb_per_chunk;
    t.nkb = min(p.kb_per_chunk, p.num_kb - t.kb0);
    t.r0 = t.h0 = t.w0 = 0;
    return t;
  }
  t.m_tile = tile / p.num_n_tiles;
  t.n_tile = tile - t.m_tile * p.num_n_tiles;
  return decode_m<EPI>(p, t);
}

// Pair tile pt of the 2-CTA kernel: CTA `rank` takes 128-row tile 2*mp + rank.
template <int EPI>
__device__ __forceinline__ TileCoord decode_pair_tile(const TcGemmParams& p, int pt, int rank) {
  TileCoord t;
  t.kb0 = 0;
  t.nkb = p.num_kb;
  if (EPI == EPI_CONV && p.ksplit > 1) {
    const int part = pt % p.ksplit;
    pt /= p.ksplit;
    t.kb0 = static_cast<int>(static_cast<long>(part) * p.num_kb / p.ksplit);
    t.nkb = static_cast<int>(static_cast<long>(part + 1) * p.num_kb / p.ksplit) - t.kb0;
  }
  const int mp = pt / p.num_n_tiles;
  t.n_tile = pt - mp * p.num_n_tiles;
  t.m_tile = 2 * mp + rank;
  return decode_m<EPI>(p, t);
}

template <int EPI>
__device__ __forceinline__ TileCoord decode_m(const TcGemmParams& p, TileCoord t) {
  if (EPI == EPI_CONV) {
    const int per_img = p.tiles_h * p.tiles_w;
    t.img = t.m_tile / per_img;
    const int u = t.m_tile - t.img * per_img;
    t.h0 = (u / p.tiles_w) * p.TH;
    t.w0 = (u % p.tiles_w) * p.TW;
    t.r0 = 0;
  } else {
    t.img = t.m_tile / p.m_tiles_per_img;
    t.r0 = (t.m_tile - t.img * p.m_tiles_per_img) * 128;
    t.h0 = t.w0 = 0;
  }
  return t;
}

__device__ __forceinline__ void store_bf16x16(__nv_bfloat16* dst, const float (&v)[16], int nvalid) {
  uint4 o0, o1;
  o0.x = pack_bf16x2(v[0], v[1]);
  o0.y = pack_bf16x2(v[2], v[3]);
  o0.z = pack_bf16x2(v[4], v[5]);
  o0.w = pack_bf16x2(v[6], v[7]);
  o1.x = pack_bf16x2(v[8], v[9]);
  o1.y = pack_bf16x2(v[10], v[11]);
  o1.z = pack_bf16x2(v[12], v[13]);
  o1.w = pack_bf16x2(v[14], v[15]);
  uint4* d = reinterpret_cast<uint4*>(dst);
  if (nvalid >= 8) d[0] = o0;
  if (nvalid >= 16) d[1] = o1;
}

// Epilogue of one tile for the thread owning TMEM lane (row) r = q*32 + lane:
// read the accumulator columns, apply the step's output function, store.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile(const TcGemmParams& p, const TileCoord& tc, uint32_t t_row, int q,
                                              int lane) {
  const int r = q * 32 + lane;
  long row;
  bool valid;
  if (EPI == EPI_CONV) {
    const int hh = tc.h0 + r / p.TW, ww = tc.w0 + r % p.TW;
    valid = tc.m_tile < p.num_m_tiles && hh < p.H && ww < p.W;
    row = (static_cast<long>(tc.img) * p.H + hh) * p.W + ww;
  } else {
    valid = tc.m_tile < p.num_m_tiles && tc.r0 + r < p.R;
    row = static_cast<long>(tc.img) * p.R + tc.r0 + r;
  }
  if (EPI == EPI_KVSTATE) {
    const int dd = p.d;
    float* prow = p.kv_part +
                  ((static_cast<long>(tc.img * p.heads + tc.n_tile) * p.num_chunks + tc.m_tile) * dd + r) * (dd + 1);
#pragma unroll 1
    for (int c = 0; c < (dd + 16) / 16; ++c) {
      float v[16];
      tmem_ld16(t_row + c * 16, v);
      if (r < dd) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c * 16 + i <= dd) prow[c * 16 + i] = v[i];
      }
    }
  } else if (EPI == EPI_APPLY) {
    // columns 0..d-1: numerator; column d: denominator
    float v[16];
    tmem_ld16(t_row + (p.d / 16) * 16, v);
    float den = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i == p.d % 16) den = v[i];
    const float inv = 1.f / (den + p.eps);
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.ldo + tc.n_tile * p.d;
#pragma unroll 1
    for (int c = 0; c < (p.d + 15) / 16; ++c) {
      tmem_ld16(t_row + c * 16, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] *= inv;
      if (valid) store_bf16x16(orow + c * 16, v, p.d - c * 16);
    }
  } else {
    const int n0 = tc.n_tile * BN;
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.ldo + n0;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 64) {
      float v[64];
      if (c0 + 64 <= BN || BN >= 256) {
        tmem_ld64(t_row + c0, v);  // (BN >= 256: columns past BN are still inside the 512-column allocation)
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (c0 + 16 * j < BN) tmem_ld16(t_row + c0 + 16 * j, *reinterpret_cast<float(*)[16]>(&v[16 * j]));
      }
#pragma unroll
      for (int g16 = 0; g16 < 4; ++g16) {
        const int col = c0 + 16 * g16;
        const int n = n0 + col;
        if (col >= BN) continue;
        const int src = n / p.n_split;
        const void* bias = (src < 3 && n < p.N) ? p.bias[src] : nullptr;
        if (bias) {
          const int j0 = n - src * p.n_split;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            v[16 * g16 + i] += p.bias_f32 ? reinterpret_cast<const float*>(bias)[j0 + i]
                                          : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(bias)[j0 + i]);
        }
        if (p.relu == ACT_RELU) {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[16 * g16 + i] = fmaxf(v[16 * g16 + i], 0.f);
        } else if (p.relu == ACT_GELU) {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[16 * g16 + i] = gelu_tanh(v[16 * g16 + i]);
        }
        if (valid && n < p.N) store_bf16x16(orow + col, *reinterpret_cast<const float(*)[16]>(&v[16 * g16]), 16);
      }
    }
  }
}

// Apply epilogue with staged TMA stores: per warp, 32 rows x d outputs of one
// head in a dense [32][d] bf16 block (2 buffers, 32*d*2 bytes each), written
// by one 3D tensor store into out [img][R][C] at column head * d.
template <int BN>
__device__ __forceinline__ void epilogue_apply_staged(const TcGemmParams& p, const TileCoord& tc, uint32_t t_row,
                                                      int q, int lane, uint8_t* stg, int& sbuf) {
  const int d = p.d;
  float v[64];
  float dv[16];
  tmem_ld16(t_row + (d / 16) * 16, dv);  // the denominator column d
  float den = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (i == d % 16) den = dv[i];
  const float inv = 1.f / (den + p.eps);
  if (p.den_out) {
    const int row = tc.r0 + q * 32 + lane;
    if (tc.m_tile < p.num_m_tiles && row < p.R)
      p.den_out[(static_cast<long>(tc.img) * p.R + row) * p.heads + tc.n_tile] = den + p.eps;
  }
  if (lane == 0) bulk_wait_read<1>();
  __syncwarp();
  uint8_t* buf = stg + sbuf * (32 * d * 2);
  uint4* rowp = reinterpret_cast<uint4*>(buf + lane * d * 2);
#pragma unroll 1
  for (int c0 = 0; c0 < d; c0 += 64) {
    tmem_ld64(t_row + c0, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (c0 + 8 * j < d) {
        uint4 o;
        o.x = pack_bf16x2(v[8 * j + 0] * inv, v[8 * j + 1] * inv);
        o.y = pack_bf16x2(v[8 * j + 2] * inv, v[8 * j + 3] * inv);
        o.z = pack_bf16x2(v[8 * j + 4] * inv, v[8 * j + 5] * inv);
        o.w = pack_bf16x2(v[8 * j + 6] * inv, v[8 * j + 7] * inv);
        rowp[c0 / 8 + j] = o;
      }
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && tc.m_tile < p.num_m_tiles && tc.r0 + q * 32 < p.R) {
    tma_store_3d(&p.out_map, buf, tc.n_tile * d, tc.r0 + q * 32, tc.img);
    bulk_commit();
  }
  sbuf ^= 1;
}

// A and B loads of k-block kb of a (1-CTA) tile into one pipeline stage.
template <int BN, int NSPLIT, int EPI, bool PAIR>
__device__ __forceinline__ void load_stage(const TcGemmParams& p, const TileCoord& tc, int kb, uint8_t* dA,
                                           uint8_t* dB, uint64_t* bar, int rank) {
  constexpr int NCHUNK = BN / NSPLIT;
  constexpr int BROWS = PAIR ? NCHUNK / 2 : NCHUNK;  // B rows of one chunk in this CTA
  const uint32_t bar_addr = PAIR ? mapa_shared(smem_u32(bar), 0) : smem_u32(bar);  // pair: leader's barrier
  // ---- A: 128 rows of this CTA's tile
  if (EPI == EPI_CONV) {
    const int tap = kb / p.kb_per_tap;
    const int c0 = (kb - tap * p.kb_per_tap) * 64;
    const int kh = tap / 3, kw = tap - 3 * (tap / 3);
    if (PAIR)
      tma2_load_4d(&p.a0, bar_addr, dA, c0, tc.w0 + kw - 1, tc.h0 + kh - 1, tc.img);
    else
      tma_load_4d(&p.a0, bar, dA, c0, tc.w0 + kw - 1, tc.h0 + kh - 1, tc.img);
  } else if (EPI == EPI_APPLY) {
    // Q as [img][row][head][d]: the head's d columns only (columns past d read as zero)
    tma_load_4d(&p.a0, bar, dA, kb * 64, tc.n_tile, tc.r0, tc.img);
  } else {
    const CUtensorMap* am = &p.a0;
    int x = kb * 64, y = tc.r0, z = tc.img;
    if (EPI == EPI_KVSTATE) {
      // KT as [img * heads][d][Mp]: the head's d channel rows only (rows past d read as zero)
      x = (tc.kb0 + kb) * 64;
      y = 0;
      z = tc.img * p.heads + tc.n_tile;
    } else if (kb >= p.kb_split) {
      am = &p.a1;
      x = (kb - p.kb_split) * 64;
    }
    if (PAIR)
      tma2_load_3d(am, bar_addr, dA, x, y, z);
    else
      tma_load_3d(am, bar, dA, x, y, z);
  }
  // ---- B: NSPLIT chunks of NCHUNK output columns (this CTA's half in a pair)
#pragma unroll
  for (int s = 0; s < NSPLIT; ++s) {
    const CUtensorMap* bm;
    int x, y;
    if (EPI == EPI_KVSTATE) {
      // VTx as [img * heads][d][Mp]: the head's d value rows; the rest of the box
      // reads as zero and the MMA issuer writes the ones row
      uint8_t* d = dB + s * BROWS * 128;
      tma_load_3d(&p.b0, bar, d, (tc.kb0 + kb) * 64, 0, tc.img * p.heads + tc.n_tile);
      continue;
    } else if (EPI == EPI_APPLY) {
      bm = &p.b0;
      x = kb * 64;
      y = (tc.img * p.heads + tc.n_tile) * BN + s * NCHUNK;
    } else {
      const int n = tc.n_tile * BN + s * NCHUNK + (PAIR ? rank * BROWS : 0);
      if (kb >= p.kb_split) {
        bm = &p.bk;
        x = (kb - p.kb_split) * 64;
        y = n;
      } else {
        const int src = n / p.n_split;
        bm = src == 0 ? &p.b0 : (src == 1 ? &p.b1 : &p.b2);
        x = kb * 64;
        y = n - src * p.n_split;
      }
    }
    uint8_t* d = dB + s * BROWS * 128;
    if (PAIR)
      tma2_load_2d(bm, bar_addr, d, x, y);
    else
      tma_load_2d(bm, bar, d, x, y);
  }
}

template <int BN, int NSPLIT, int STAGES, int EPI, int STG = 0>
__global__ void __launch_bounds__(192, 1) tc_gemm_kernel(const __grid_constant__ TcGemmParams p) {
  using Cfg = TcGemmCfg<BN, NSPLIT, STAGES, STG>;
  constexpr int NCHUNK = Cfg::NCHUNK, ACC = Cfg::ACC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* stg_base = sB + STAGES * Cfg::B_BYTES;  // 1024-byte aligned
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(stg_base + Cfg::STG_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;
  uint64_t* tempty_bar = tfull_bar + ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + ACC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < ACC; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a0);
    tma_prefetch_desc(&p.b0);
  }
  if (warp == 1) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // inputs of this grid are ready past this point

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && !*abort_flag; tile += gridDim.x) {
        const TileCoord tc = decode_tile<EPI>(p, tile);
        for (int kb = 0; kb < tc.nkb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.status)) break;
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::STAGE_BYTES);
          load_stage<BN, NSPLIT, EPI, false>(p, tc, kb, sA + stage * Cfg::A_BYTES, sB + stage * Cfg::B_BYTES,
                                             &full_bar[stage], 0);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // On abort, give copies and MMAs already issued time to land before
      // the block releases its shared memory and TMEM.
      if (*abort_flag) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && !*abort_flag; tile += gridDim.x) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const int nkb = decode_tile<EPI>(p, tile).nkb;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (EPI == EPI_KVSTATE) {  // [V | 1]: row d of the B tile (64 keys, 128 bytes) is all ones
            const uint32_t one2 = 0x3F803F80u;  // two bf16 1.0
            uint4* r1 = reinterpret_cast<uint4*>(sB + stage * Cfg::B_BYTES + p.d * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j) r1[j] = make_uint4(one2, one2, one2, one2);
            fence_proxy_async_smem();
          }
          const uint32_t a_addr = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t adesc = sdesc_kmajor_sw128(a_addr + k * 32);
#pragma unroll
            for (int s = 0; s < NSPLIT; ++s) {
              const uint64_t bdesc = sdesc_kmajor_sw128(b_addr + s * NCHUNK * 128 + k * 32);
              umma_bf16(d_tmem + s * NCHUNK, adesc, bdesc, Cfg::IDESC, (kb | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        if (++acc == ACC) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* stg = stg_base + q * (STG / 4);
    int sbuf = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      if (!warp_wait(&tfull_bar[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const TileCoord tc = decode_tile<EPI>(p, tile);
      const uint32_t t_row = tmem_base + acc * BN + (static_cast<uint32_t>(q * 32) << 16);
      if (EPI == EPI_APPLY && STG > 0)
        epilogue_apply_staged<BN>(p, tc, t_row, q, lane, stg, sbuf);
      else
        epilogue_tile<BN, EPI>(p, tc, t_row, q, lane);
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      if (++acc == ACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (STG > 0) {
      if (lane == 0) bulk_wait_read<0>();  // staged stores have read shared memory before it is released
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ===================================================================== pairs
// Two-SM version (cta_group::2, cluster of 2): pair tile = 256 rows (128 per
// CTA) x BN columns. Each CTA loads its own 128 A rows and half of each B
// chunk into its own shared memory; TMA completion is counted on the
// leader's (rank 0) full barrier; the leader's single thread issues the
// M = 256 MMAs and multicasts each commit to both CTAs' barriers; each CTA's
// epilogue drains its own TMEM rows and arrives on the leader's TMEM-empty
// barrier (256 arrivals). Per CTA, shared-memory operand traffic per MMA
// column is half that of the 1-CTA kernel.
template <int BN, int NSPLIT, int STAGES>
struct TcPairCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int NCHUNK = BN / NSPLIT;  // MMA N
  static constexpr int BROWS = NCHUNK / 2;    // B rows per chunk per CTA
  static_assert(BN % NSPLIT == 0 && NCHUNK % 16 == 0 && NCHUNK <= 256 && (BROWS * 128) % 1024 == 0, "pair N");
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = NSPLIT * BROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // per CTA
  static constexpr int ACC = (2 * BN <= 512) ? 2 : 1;
  static constexpr int TMEM_COLS = (ACC * BN <= 128) ? 128 : (ACC * BN <= 256) ? 256 : 512;
  static_assert(ACC * BN <= 512, "TMEM");
  static constexpr int STG_BYTES = 4 * 2 * 4096;  // 4 epilogue warps x 2 buffers x (32 rows x 128 B)
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * ACC) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STG_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static constexpr uint32_t IDESC = idesc_bf16_f32(256, NCHUNK);
};

// Staged epilogue (EPI_LINEAR / EPI_CONV): per 64-column chunk, one 64-wide
// TMEM load, bias / ReLU in registers, a 128B-swizzled
// 32 x 128-byte staging block per warp (double-buffered), and one TMA tensor
// store of the block, so global writes leave the SM as full lines.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile_staged(const TcGemmParams& p, const TileCoord& tc, uint32_t t_row,
                                                     int q, int lane, uint8_t* stg, int& sbuf) {
  const bool real = tc.m_tile < p.num_m_tiles;
  const int n0 = tc.n_tile * BN;
  // EPI_CONV with gn_col: bit i = row q*32 + i of the tile is a pixel of the image
  uint32_t inside = 0;
  if (EPI == EPI_CONV && p.gn_col != nullptr) {
    const int r = q * 32 + lane;
    inside = __ballot_sync(0xffffffffu, real && tc.h0 + r / p.TW < p.H && tc.w0 + r % p.TW < p.W);
  }
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 64) {
    float v[64];
    tmem_ld64(t_row + c0, v);
#pragma unroll
    for (int g16 = 0; g16 < 4; ++g16) {
      const int col = c0 + 16 * g16;
      const int n = n0 + col;
      const int src = n / p.n_split;
      const void* bias = (col < BN && src < 3 && n < p.N) ? p.bias[src] : nullptr;
      if (bias) {
        const int j0 = n - src * p.n_split;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[16 * g16 + i] += p.bias_f32 ? reinterpret_cast<const float*>(bias)[j0 + i]
                                        : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(bias)[j0 + i]);
      }
    }
    if (p.relu == ACT_RELU) {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = fmaxf(v[i], 0.f);
    } else if (p.relu == ACT_GELU) {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = gelu_tanh(v[i]);
    }
    // stage this warp's 32 rows x 64 columns (bf16) in 128B-swizzled order
    if (lane == 0) bulk_wait_read<1>();  // the store that last read this buffer is done
    __syncwarp();
    uint8_t* buf = stg + sbuf * 4096;
    uint4* rowp = reinterpret_cast<uint4*>(buf + lane * 128);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint4 o;
      o.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
      o.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
      o.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
      o.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
      rowp[j ^ (lane & 7)] = o;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (EPI == EPI_CONV && p.gn_col != nullptr && real) {
      // column sums of the staged bf16 values over this warp's 32 rows: lane l
      // takes columns c0 + 2l, c0 + 2l + 1 (one 32-bit word per row; the 128-byte
      // swizzle puts the eight lanes of a 16-byte chunk on distinct banks)
      float s0 = 0.f, q0 = 0.f, s1 = 0.f, q1 = 0.f;
      const uint8_t* colp = buf + ((lane & 3) << 2);
#pragma unroll 8
      for (int i = 0; i < 32; ++i) {
        if ((inside >> i) & 1u) {
          const uint32_t wd = *reinterpret_cast<const uint32_t*>(colp + i * 128 + (((lane >> 2) ^ (i & 7)) << 4));
          const float a = __uint_as_float(wd << 16), b = __uint_as_float(wd & 0xffff0000u);
          s0 += a;
          q0 = fmaf(a, a, q0);
          s1 += b;
          q1 = fmaf(b, b, q1);
        }
      }
      const int col = n0 + c0 + 2 * lane;
      if (col < p.N) {
        const int per_img = p.tiles_h * p.tiles_w;
        const long slot = (static_cast<long>(tc.img) * per_img + (tc.m_tile - tc.img * per_img)) * 4 + q;
        *reinterpret_cast<float4*>(p.gn_col + (slot * p.N + col) * 2) = make_float4(s0, q0, s1, q1);
      }
    }
    if (lane == 0 && real) {
      if (EPI == EPI_CONV) {
        const int r0w = q * 32;
        const int ws = tc.w0 + r0w % p.TW, hs = tc.h0 + r0w / p.TW;
        if (ws < p.W && hs < p.H) tma_store_4d(&p.out_map, buf, n0 + c0, ws, hs, tc.img);
      } else {
        if (tc.r0 + q * 32 < p.R) tma_store_2d(&p.out_map, buf, n0 + c0, tc.img * p.R + tc.r0 + q * 32);
      }
      bulk_commit();
    }
    sbuf ^= 1;
  }
}

// One MMA-issuing thread per output chunk (warp 1: chunk 0, warps 6..: chunks
// 1..): a tcgen05.mma costs its issuing thread tens of cycles, so one thread
// cannot keep several short MMAs per k-step back to back. Every issuer waits
// on the same full barriers; empty and TMEM-full barriers take NSPLIT commits.
constexpr int pair_threads(int nsplit) { return 192 + 32 * (nsplit - 1); }

template <int BN, int NSPLIT, int STAGES, int EPI>
__global__ void __launch_bounds__(pair_threads(NSPLIT), 1) tc_gemm_pair_kernel(const __grid_constant__ TcGemmParams p) {
  using Cfg = TcPairCfg<BN, NSPLIT, STAGES>;
  constexpr int NCHUNK = Cfg::NCHUNK, ACC = Cfg::ACC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* stg_base = sB + STAGES * Cfg::B_BYTES;  // 1024-byte aligned
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(stg_base + Cfg::STG_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;
  uint64_t* tempty_bar = tfull_bar + ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + ACC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], NSPLIT);
    }
    for (int a = 0; a < ACC; ++a) {
      mbar_init(&tfull_bar[a], NSPLIT);
      mbar_init(&tempty_bar[a], 256);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a0);
    tma_prefetch_desc(&p.b0);
  }
  if (warp == 1) tmem_alloc2(tmem_slot, Cfg::TMEM_COLS);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // inputs of this grid are ready past this point

  if (warp == 0) {
    // ------------------------------------------------------------ producers (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int pt = pair; pt < p.num_tiles && !*abort_flag; pt += npairs) {
        const TileCoord tc = decode_pair_tile<EPI>(p, pt, rank);
        for (int kb = 0; kb < tc.nkb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.status)) break;
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * Cfg::STAGE_BYTES);
          load_stage<BN, NSPLIT, EPI, true>(p, tc, tc.kb0 + kb, sA + stage * Cfg::A_BYTES,
                                            sB + stage * Cfg::B_BYTES, &full_bar[stage], rank);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp >= 6) {
    // ------------------------------------------------------------ MMA issuers (leader), one per chunk
    if (leader && lane == 0) {
      const int sc = warp == 1 ? 0 : warp - 5;  // output chunk of this thread
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int pt = pair; pt < p.num_tiles && !*abort_flag; pt += npairs) {
        int to = 0;
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, abort_flag, p.status, &to)) {
          if (to) record_wait_site(p.status, 2, pt, -1, acc, acc_phase ^ 1);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN + sc * NCHUNK;
        const int nkb = decode_pair_tile<EPI>(p, pt, 0).nkb;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          int to = 0;
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.status, &to)) {
            if (to) record_wait_site(p.status, 3, pt, kb, stage, phase);
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors of k-step k are the k = 0 ones plus 32 bytes (2 in the address field) per step
          const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sA + stage * Cfg::A_BYTES));
          const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + stage * Cfg::B_BYTES) + sc * Cfg::BROWS * 128);
          const uint32_t first = kb != 0 ? 1u : 0u;
#pragma unroll
          for (int k = 0; k < 4; ++k) umma2_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, Cfg::IDESC, k ? 1u : first);
          umma2_commit_mc(&empty_bar[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma2_commit_mc(&tfull_bar[acc], 0x3);
        if (++acc == ACC) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
    uint8_t* stg = stg_base + q * 8192;
    int sbuf = 0;
    int acc = 0, ntile_done = 0;
    uint32_t acc_phase = 0;
    for (int pt = pair; pt < p.num_tiles; pt += npairs) {
      int to = 0;
      if (!warp_wait(&tfull_bar[acc], acc_phase, abort_flag, p.status, &to)) {
        if (lane == 0 && to) record_wait_site(p.status, 20 + rank * 10 + (warp & 3), pt, ntile_done, acc, acc_phase);
        break;
      }
      tc_fence_after();
      const TileCoord tc = decode_pair_tile<EPI>(p, pt, rank);
      const uint32_t t_row = tmem_base + acc * BN + (static_cast<uint32_t>(q * 32) << 16);
      if (EPI == EPI_CONV && p.ksplit > 1) {
        // fp32 partial of this k-part, column-quad major ([N / 4][128 rows][4]): a warp's
        // 16-byte stores of one column quad land on 512 contiguous bytes
        float* pbase = p.fix_part + (static_cast<long>(pt) * 2 + rank) * 128 * p.N + (q * 32 + lane) * 4;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 64) {
          float v[64];
          tmem_ld64(t_row + c0, v);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + 4 * j < BN)
              *reinterpret_cast<float4*>(pbase + static_cast<long>(c0 / 4 + j) * 512) =
                  make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      } else {
        epilogue_tile_staged<BN, EPI>(p, tc, t_row, q, lane, stg, sbuf);
      }
      tc_fence_before();
      mbar_arrive_relaxed_cluster(tempty_leader0 + acc * 8);  // TMEM reads done (wait::ld)
      ++ntile_done;
      if (++acc == ACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_read<0>();  // staged stores have read shared memory before it is released
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, Cfg::TMEM_COLS);
  }
}


// ----------------------------------------------------------------------------
// Linear projections on CTA pairs with 256 x 384 pair tiles (the Linear layers
// of section "Spatial Compressor" and the query Linear of eq. Q^EDiT).
//
// A 384-column tile halves the weight bytes each CTA ingests per MMA cycle
// against 256 columns (40 KB per k-block for 768 MMA cycles instead of 32 KB
// for 512), which is what bounds the 256-column kernel. A tile is three
// 128-column MMA chunks, each issued by its own thread (warps 1, 6, 7 of the
// leader). TMEM (512 columns) is a ring of four 128-column slots: chunk
// g = 3 * (local tile index) + c lives in slot g % 4, so the drain of one
// tile's chunks overlaps the next tile's main loop.
//
// Weight rows: CTA rank r loads the 192 contiguous rows n0 + 192 r ... of the
// tile as one TMA box; chunk c multiplies rows 64 c .. 64 c + 63 of both CTAs'
// boxes, so accumulator column j of chunk c is output column n0 + 64 c + j
// (j < 64) or n0 + 192 + 64 c + (j - 64) (j >= 64).
template <int STAGES, int STGBUF>
struct RingCfg {
  static constexpr int BN = 384, NCH = 3, NCHUNK = 128, BROWS = 192, SLOTS = 4;
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = BROWS * 64 * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // per CTA
  static constexpr int STG_BYTES = 4 * STGBUF * 4096;    // 4 epilogue warps x STGBUF x (32 rows x 128 B)
  static constexpr int BIAS_BYTES = 4 * BN * 4;          // per epilogue warp: the tile's bias in fp32
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * SLOTS) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STG_BYTES + BIAS_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert((BROWS / NCH) * 128 % 1024 == 0, "chunk offset keeps the 1024-byte swizzle atom");
  static constexpr uint32_t IDESC = idesc_bf16_f32(256, NCHUNK);
};
constexpr int kRingThreads = 256;

// Bias of output columns [n0, n0 + 384) in fp32, 12 per lane (columns
// 4 (32 i + lane) .. + 3, i < 3); zero past N or without a bias. One weight
// source per 4 columns (n_split is a multiple of 64); the bias vectors are
// 16-byte aligned (checked by the host).
__device__ __forceinline__ void ring_bias_fetch(const TcGemmParams& p, int n0, int lane, float4 (&b)[3]) {
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int n = n0 + 4 * (32 * i + lane);
    b[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n < p.N) {
      const int src = n / p.n_split;
      const void* bias = src < 3 ? p.bias[src] : nullptr;
      if (bias) {
        const int j0 = n - src * p.n_split;
        if (p.bias_f32) {
          b[i] = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(bias) + j0));
        } else {
          const uint2 t = __ldg(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(bias) + j0));
          b[i] = make_float4(__uint_as_float(t.x << 16), __uint_as_float(t.x & 0xffff0000u),
                             __uint_as_float(t.y << 16), __uint_as_float(t.y & 0xffff0000u));
        }
      }
    }
  }
}

// Bias (from the warp's shared copy, 64 values at bsm), optional ReLU, bf16
// staging and one TMA store for 32 rows x 64 output columns [n, n + 64).
template <int STGBUF>
__device__ __forceinline__ void ring_store64(const TcGemmParams& p, const TileCoord& tc, float (&v)[64], int n,
                                             const float* bsm, int q, int lane, uint8_t* stg, int& sbuf) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float4 t = reinterpret_cast<const float4*>(bsm)[i];
    v[4 * i] += t.x;
    v[4 * i + 1] += t.y;
    v[4 * i + 2] += t.z;
    v[4 * i + 3] += t.w;
  }
  if (p.relu == ACT_RELU) {
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = fmaxf(v[i], 0.f);
  } else if (p.relu == ACT_GELU) {
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = gelu_tanh(v[i]);
  }
  if (lane == 0) bulk_wait_read<STGBUF - 1>();  // the store that last read this buffer is done
  __syncwarp();
  uint8_t* buf = stg + sbuf * 4096;
  uint4* rowp = reinterpret_cast<uint4*>(buf + lane * 128);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint4 o;
    o.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
    o.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
    o.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
    o.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
    rowp[j ^ (lane & 7)] = o;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && tc.m_tile < p.num_m_tiles && tc.r0 + q * 32 < p.R && n < p.N) {
    tma_store_2d(&p.out_map, buf, n, tc.img * p.R + tc.r0 + q * 32);
    bulk_commit();
  }
  if (++sbuf == STGBUF) sbuf = 0;
}

template <int STAGES, int STGBUF>
__global__ void __launch_bounds__(kRingThreads, 1) tc_linear_ring_kernel(const __grid_constant__ TcGemmParams p) {
  using Cfg = RingCfg<STAGES, STGBUF>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* stg_base = sB + STAGES * Cfg::B_BYTES;  // 1024-byte aligned
  float* bias_base = reinterpret_cast<float*>(stg_base + Cfg::STG_BYTES);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(stg_base + Cfg::STG_BYTES + Cfg::BIAS_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;
  uint64_t* tempty_bar = tfull_bar + Cfg::SLOTS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + Cfg::SLOTS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], Cfg::NCH);  // one commit per chunk issuer
    }
    for (int a = 0; a < Cfg::SLOTS; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 8);  // one arrival per epilogue warp of both CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a0);
    tma_prefetch_desc(&p.b0);
  }
  if (warp == 1) tmem_alloc2(tmem_slot, 512);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // inputs of this grid are ready past this point

  if (warp == 0) {
    // ------------------------------------------------------------ producers (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t full0 = mapa_shared(smem_u32(&full_bar[0]), 0);  // the leader's barriers
      const int last_src = (p.N - 1) / p.n_split;
      for (int pt = pair; pt < p.num_tiles && !*abort_flag; pt += npairs) {
        const TileCoord tc = decode_pair_tile<EPI_LINEAR>(p, pt, rank);
        const int nb = tc.n_tile * Cfg::BN + rank * Cfg::BROWS;  // first weight row of this CTA
        int src = nb / p.n_split;
        if (src > last_src) src = last_src;  // rows past N: out of the map, zero-filled
        const CUtensorMap* bmap = src == 0 ? &p.b0 : (src == 1 ? &p.b1 : &p.b2);
        const int yb = nb - src * p.n_split;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          int to = 0;
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.status, &to)) {
            if (to) record_wait_site(p.status, 10 + warp, pt, kb, stage, phase ^ 1);
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * Cfg::STAGE_BYTES);
          const uint32_t bar = full0 + stage * 8;
          if (kb < p.kb_split) {
            tma2_load_3d(&p.a0, bar, sA + stage * Cfg::A_BYTES, kb * 64, tc.r0, tc.img);
            tma2_load_2d(bmap, bar, sB + stage * Cfg::B_BYTES, kb * 64, yb);
          } else {
            tma2_load_3d(&p.a1, bar, sA + stage * Cfg::A_BYTES, (kb - p.kb_split) * 64, tc.r0, tc.img);
            tma2_load_2d(&p.bk, bar, sB + stage * Cfg::B_BYTES, (kb - p.kb_split) * 64, nb);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {  // let loads already issued land before the CTA can exit
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp >= 6) {
    // ------------------------------------------------------------ MMA issuers (leader), one per chunk
    if (leader && lane == 0) {
      const int c = warp == 1 ? 0 : warp - 5;
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int pt = pair; pt < p.num_tiles && !*abort_flag; pt += npairs, ++it) {
        const int g = Cfg::NCH * it + c;
        const int slot = g & 3;
        const uint32_t use = static_cast<uint32_t>(g >> 2) & 1u;
        int to = 0;
        if (!mbar_wait(&tempty_bar[slot], use ^ 1u, abort_flag, p.status, &to)) {
          if (to) record_wait_site(p.status, 2, pt, c, slot, use ^ 1u);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + slot * Cfg::NCHUNK;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          int to = 0;
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.status, &to)) {
            if (to) record_wait_site(p.status, 3, pt, kb, stage, phase);
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors of k-step k are the k = 0 ones plus 32 bytes (2 in the address field) per step
          const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sA + stage * Cfg::A_BYTES));
          const uint64_t bdesc =
              sdesc_kmajor_sw128(smem_u32(sB + stage * Cfg::B_BYTES) + c * (Cfg::BROWS / Cfg::NCH) * 128);
          const uint32_t first = kb != 0 ? 1u : 0u;
#pragma unroll
          for (int k = 0; k < 4; ++k) umma2_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, Cfg::IDESC, k ? 1u : first);
          umma2_commit_mc(&empty_bar[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma2_commit_mc(&tfull_bar[slot], 0x3);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs), warps 2..5
    const int q = warp & 3;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
    uint8_t* stg = stg_base + q * STGBUF * 4096;
    float* bsm = bias_base + q * Cfg::BN;
    int sbuf = 0;
    int it = 0;
    bool ok = true;
    for (int pt = pair; pt < p.num_tiles && ok; pt += npairs, ++it) {
      const TileCoord tc = decode_pair_tile<EPI_LINEAR>(p, pt, rank);
      const int n0 = tc.n_tile * Cfg::BN;
      float4 bias4[3];  // fetched before the wait for the tile's first chunk, which hides the latency
      ring_bias_fetch(p, n0, lane, bias4);
#pragma unroll 1
      for (int c = 0; c < Cfg::NCH; ++c) {
        const int g = Cfg::NCH * it + c;
        const int slot = g & 3;
        const uint32_t use = static_cast<uint32_t>(g >> 2) & 1u;
        int to = 0;
        if (!warp_wait(&tfull_bar[slot], use, abort_flag, p.status, &to)) {
          if (lane == 0 && to) record_wait_site(p.status, 20 + rank * 10 + q, pt, c, slot, use);
          ok = false;
          break;
        }
        tc_fence_after();
        if (c == 0) {  // the previous tile's reads of bsm are complete (program order + the wait's warp sync)
#pragma unroll
          for (int i = 0; i < 3; ++i) reinterpret_cast<float4*>(bsm)[32 * i + lane] = bias4[i];
          __syncwarp();
        }
        const uint32_t t_row = tmem_base + slot * Cfg::NCHUNK + (static_cast<uint32_t>(q * 32) << 16);
        float v0[64], v1[64];
        tmem_ld64(t_row, v0);
        tmem_ld64(t_row + 64, v1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed_cluster(tempty_leader0 + slot * 8);  // slot free for chunk g + 4
        ring_store64<STGBUF>(p, tc, v0, n0 + 64 * c, bsm + 64 * c, q, lane, stg, sbuf);
        ring_store64<STGBUF>(p, tc, v1, n0 + Cfg::BROWS + 64 * c, bsm + Cfg::BROWS + 64 * c, q, lane, stg, sbuf);
      }
    }
    if (lane == 0) bulk_wait_read<0>();  // staged stores have read shared memory before it is released
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, 512);
  }
}

}  // namespace edit

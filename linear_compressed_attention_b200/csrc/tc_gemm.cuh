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
//              exactly the conv's zero padding): + bias, bf16 store of U and
//              per-tile GroupNorm partial sums.
//  EPI_APPLY   Linear attention apply, eq. (y_i): per head h, [num | den] =
//              Q_h [S_h | z_h] and y = num / (den + eps) fused into the store.
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

enum { EPI_LINEAR = 0, EPI_CONV = 1, EPI_APPLY = 2 };

struct TcGemmParams {
  // A sources (3D maps [img][rows][K], box 64 x 128 x 1): a0 gives the first
  // kb_split k-blocks, a1 the rest. EPI_CONV: a0 is the 4D grid map
  // [B][H][W][C] with box 64 x TW x TH x 1.
  CUtensorMap a0, a1;
  // B sources (2D maps [rows][K], box 64 x NCHUNK): b[s] holds output columns
  // [s*n_split, (s+1)*n_split) for the first kb_split k-blocks; bk holds the
  // rest of K (single N source only). EPI_APPLY: b0 = [img*heads*BN][KP].
  CUtensorMap b0, b1, b2, bk;
  int R;            // rows per image (A)
  int m_tiles_per_img;
  int num_kb;       // 64-wide k-blocks
  int kb_split;
  int n_split;
  int N;            // output columns (EPI_LINEAR masks columns >= N)
  int num_n_tiles;
  int num_tiles;
  // implicit-conv geometry (EPI_CONV)
  int H, W, TH, TW, tiles_h, tiles_w, kb_per_tap;
  // apply geometry (EPI_APPLY)
  int d, heads;
  float eps;
  // epilogue
  void* out;        // bf16, row (img*R + r) at out + row*ldo (+ column offset)
  long ldo;
  const void* bias[3];
  int bias_f32;
  int relu;
  float* gn_partials;  // EPI_CONV: [img][tiles_per_img][4][groups][2]
  int groups, cpg;
  int* status;
};

template <int BN, int NSPLIT, int STAGES>
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
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * ACC) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, NCHUNK);
};

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

struct TileCoord {
  int m_tile, n_tile, img, r0, h0, w0;
};

template <int EPI>
__device__ __forceinline__ TileCoord decode_tile(const TcGemmParams& p, int tile) {
  TileCoord t;
  t.m_tile = tile / p.num_n_tiles;
  t.n_tile = tile - t.m_tile * p.num_n_tiles;
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

template <int BN, int NSPLIT, int STAGES, int EPI>
__global__ void __launch_bounds__(192, 1) tc_gemm_kernel(const __grid_constant__ TcGemmParams p) {
  using Cfg = TcGemmCfg<BN, NSPLIT, STAGES>;
  constexpr int BM = Cfg::BM, NCHUNK = Cfg::NCHUNK, ACC = Cfg::ACC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::B_BYTES);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && !*abort_flag; tile += gridDim.x) {
        const TileCoord tc = decode_tile<EPI>(p, tile);
        const CUtensorMap* bmap = &p.b0;
        int brow0;
        if (EPI == EPI_APPLY) {
          brow0 = (tc.img * p.heads + tc.n_tile) * BN;
        } else {
          const int n0 = tc.n_tile * BN;
          const int src = n0 / p.n_split;
          bmap = src == 0 ? &p.b0 : (src == 1 ? &p.b1 : &p.b2);
          brow0 = n0 - src * p.n_split;
        }
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.status)) break;
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::STAGE_BYTES);
          uint8_t* dA = sA + stage * Cfg::A_BYTES;
          uint8_t* dB = sB + stage * Cfg::B_BYTES;
          if (EPI == EPI_CONV) {
            const int tap = kb / p.kb_per_tap;
            const int c0 = (kb - tap * p.kb_per_tap) * 64;
            const int kh = tap / 3, kw = tap - 3 * (tap / 3);
            tma_load_4d(&p.a0, &full_bar[stage], dA, c0, tc.w0 + kw - 1, tc.h0 + kh - 1, tc.img);
          } else if (EPI == EPI_APPLY) {
            tma_load_3d(&p.a0, &full_bar[stage], dA, tc.n_tile * p.d + kb * 64, tc.r0, tc.img);
          } else if (kb < p.kb_split) {
            tma_load_3d(&p.a0, &full_bar[stage], dA, kb * 64, tc.r0, tc.img);
          } else {
            tma_load_3d(&p.a1, &full_bar[stage], dA, (kb - p.kb_split) * 64, tc.r0, tc.img);
          }
#pragma unroll
          for (int s = 0; s < NSPLIT; ++s) {
            if (kb < p.kb_split)
              tma_load_2d(bmap, &full_bar[stage], dB + s * NCHUNK * 128, kb * 64, brow0 + s * NCHUNK);
            else
              tma_load_2d(&p.bk, &full_bar[stage], dB + s * NCHUNK * 128, (kb - p.kb_split) * 64,
                          brow0 + s * NCHUNK);
          }
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
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
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
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      if (!warp_wait(&tfull_bar[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const TileCoord tc = decode_tile<EPI>(p, tile);
      long row;
      bool valid;
      if (EPI == EPI_CONV) {
        const int hh = tc.h0 + r / p.TW, ww = tc.w0 + r % p.TW;
        valid = hh < p.H && ww < p.W;
        row = (static_cast<long>(tc.img) * p.H + hh) * p.W + ww;
      } else {
        valid = tc.r0 + r < p.R;
        row = static_cast<long>(tc.img) * p.R + tc.r0 + r;
      }
      const uint32_t t_row = tmem_base + acc * BN + (static_cast<uint32_t>(q * 32) << 16);
      if (EPI == EPI_APPLY) {
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
        const int src = n0 / p.n_split;
        const void* bias = p.bias[src];
        const int bias_off = n0 - src * p.n_split;
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.ldo + n0;
        float s1 = 0.f, s2 = 0.f;  // GroupNorm running sums of the current group
        int g_cur = 0;
        float* gpart = nullptr;
        if (EPI == EPI_CONV) {
          const int per_img = p.tiles_h * p.tiles_w;
          const int t_in_img = tc.m_tile - tc.img * per_img;
          gpart = p.gn_partials + ((static_cast<long>(tc.img) * per_img + t_in_img) * 4 + q) * p.groups * 2;
        }
#pragma unroll 1
        for (int c = 0; c < BN / 16; ++c) {
          float v[16];
          tmem_ld16(t_row + c * 16, v);
          if (bias) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int j = bias_off + c * 16 + i;
              v[i] += p.bias_f32 ? reinterpret_cast<const float*>(bias)[j]
                                 : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(bias)[j]);
            }
          }
          if (p.relu) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = fmaxf(v[i], 0.f);
          }
          if (EPI == EPI_CONV) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int g = (c * 16 + i) / p.cpg;  // warp-uniform
              if (g != g_cur) {
                const float t1 = warp_sum(s1), t2 = warp_sum(s2);
                if (lane == 0) {
                  gpart[g_cur * 2] = t1;
                  gpart[g_cur * 2 + 1] = t2;
                }
                s1 = s2 = 0.f;
                g_cur = g;
              }
              const float x = valid ? v[i] : 0.f;
              s1 += x;
              s2 += x * x;
            }
          }
          if (valid && n0 + c * 16 < p.N) store_bf16x16(orow + c * 16, v, 16);
        }
        if (EPI == EPI_CONV) {
          const float t1 = warp_sum(s1), t2 = warp_sum(s2);
          if (lane == 0) {
            gpart[g_cur * 2] = t1;
            gpart[g_cur * 2 + 1] = t2;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      if (++acc == ACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace edit

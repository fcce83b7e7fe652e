// ConvFusion 3x3 conv (eq. Q^EDiT, first Conv) as an implicit GEMM on CTA
// pairs with tap reuse: for each 64-channel block the CTA loads the input
// patch of its 128-token tile once (3 image rows x 130 pixels, zero-filled
// outside the grid by TMA) and feeds all 9 taps from it, each tap being the
// same 128 x 64 operand shifted by kh * 130 + kw rows inside the patch (a
// descriptor start offset; the swizzle follows the absolute address). Only the weights
// stream per tap. Requires tiles of 128 consecutive pixels of one image row
// (TW = 128, TH = 1, i.e. W >= 128). The epilogue only adds the bias and
// stores U through 128B-swizzled shared-memory blocks and TMA tensor stores
// (GroupNorm statistics are a separate pass over U), so the non-overlapped
// epilogue of the single TMEM accumulator stays short.
//
// Roles: warp 0 producer (both CTAs), warp 1 TMEM owner and (leader) MMA
// issuer of output chunk 0, warps 2..5 epilogue (bias + staged U store), and
// with NSPLIT > 1 warps 6.. issue the MMAs of chunks 1.. (leader). One issuing
// thread per accumulator chunk: a tcgen05.mma costs its issuing thread tens of
// cycles, more than an N = 144 MMA leaves between issues when one thread
// feeds two accumulators. Every issuer waits on the same operand barriers
// and commits to the shared empty / TMEM-full barriers (NSPLIT arrivals).
#pragma once

#include "tc_gemm.cuh"

namespace edit {

template <int BN, int NSPLIT, int NB>
struct ConvPairCfg {
  static constexpr int NCHUNK = BN / NSPLIT;
  static constexpr int BROWS = NCHUNK / 2;
  static_assert(BN % NSPLIT == 0 && NCHUNK % 16 == 0 && NCHUNK <= 256 && (BROWS * 128) % 1024 == 0, "pair N");
  static constexpr int PATCH_W = 130, PATCH_H = 3;
  static constexpr int PATCH_TX = 64 * PATCH_W * PATCH_H * 2;           // bytes one patch load brings
  static constexpr int PATCH_BYTES = (PATCH_TX + 1023) / 1024 * 1024;  // buffer size
  static constexpr int B_BYTES = NSPLIT * BROWS * 128;                 // per CTA per tap
  static constexpr int ACC = (2 * BN <= 512) ? 2 : 1;
  static constexpr int TMEM_COLS = (ACC * BN <= 128) ? 128 : (ACC * BN <= 256) ? 256 : 512;
  static constexpr int STG_BYTES = 4 * 2 * 4096;  // 4 epilogue warps x 2 buffers x (32 rows x 128 B)
  static constexpr int BAR_BYTES = (2 * 2 + 2 * NB + 2 * ACC) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + 2 * PATCH_BYTES + NB * B_BYTES + STG_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static constexpr uint32_t IDESC = idesc_bf16_f32(256, NCHUNK);
};

// Work item `it`: a whole pair tile, or (for the last partial wave) one half of
// a pair tile's input-channel blocks.
struct ConvItem {
  int pt, cb0, cb1, half;  // half = -1: whole tile
};
__device__ __forceinline__ ConvItem conv_item(const TcGemmParams& p, int it, int ncb) {
  ConvItem c;
  if (it < p.split_first) {
    c.pt = it;
    c.cb0 = 0;
    c.cb1 = ncb;
    c.half = -1;
  } else {
    const int k = it - p.split_first;
    c.pt = p.split_first + k / 2;
    c.half = k & 1;
    c.cb0 = c.half ? ncb / 2 : 0;
    c.cb1 = c.half ? ncb : ncb / 2;
  }
  return c;
}

constexpr int conv_threads(int nsplit) { return 192 + 32 * (nsplit - 1); }

template <int BN, int NSPLIT, int NB>
__global__ void __launch_bounds__(conv_threads(NSPLIT), 1) tc_conv_pair_kernel(const __grid_constant__ TcGemmParams p) {
  using Cfg = ConvPairCfg<BN, NSPLIT, NB>;
  constexpr int NCHUNK = Cfg::NCHUNK, ACC = Cfg::ACC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                              // 2 patch buffers
  uint8_t* sB = smem + 2 * Cfg::PATCH_BYTES;       // NB weight stages
  uint64_t* a_full = reinterpret_cast<uint64_t*>(sB + NB * Cfg::B_BYTES + Cfg::STG_BYTES);
  uint64_t* a_empty = a_full + 2;
  uint64_t* b_full = a_empty + 2;
  uint64_t* b_empty = b_full + NB;
  uint64_t* tfull_bar = b_empty + NB;
  uint64_t* tempty_bar = tfull_bar + ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + ACC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int ncb = p.kb_per_tap;  // 64-channel blocks of the input
  const int C = ncb * 64;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], NSPLIT);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], NSPLIT);
    }
    for (int a = 0; a < ACC; ++a) {
      mbar_init(&tfull_bar[a], NSPLIT);
      mbar_init(&tempty_bar[a], 256);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a1);
    tma_prefetch_desc(&p.b0);
  }
  if (warp == 1) tmem_alloc2(tmem_slot, Cfg::TMEM_COLS);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // inputs of this grid are ready past this point

  if (warp == 0) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      int ai = 0, bi = 0;
      uint32_t aph = 0, bph = 0;
      bool ok = true;
      for (int it = pair; it < p.num_tiles && ok && !*abort_flag; it += npairs) {
        const ConvItem ci = conv_item(p, it, ncb);
        const TileCoord tc = decode_pair_tile<EPI_CONV>(p, ci.pt, rank);
        for (int cb = ci.cb0; cb < ci.cb1 && ok; ++cb) {
          if (!mbar_wait(&a_empty[ai], aph ^ 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&a_full[ai], 2 * Cfg::PATCH_TX);
          tma2_load_4d(&p.a1, mapa_shared(smem_u32(&a_full[ai]), 0), sA + ai * Cfg::PATCH_BYTES, cb * 64,
                       tc.w0 - 1, tc.h0 - 1, tc.img);
          if (++ai == 2) {
            ai = 0;
            aph ^= 1;
          }
          for (int tap = 0; tap < 9; ++tap) {
            if (!mbar_wait(&b_empty[bi], bph ^ 1, abort_flag, p.status)) {
              ok = false;
              break;
            }
            if (leader) mbar_arrive_expect_tx(&b_full[bi], 2 * Cfg::B_BYTES);
            const uint32_t bar = mapa_shared(smem_u32(&b_full[bi]), 0);
#pragma unroll
            for (int s = 0; s < NSPLIT; ++s)
              tma2_load_2d(&p.b0, bar, sB + bi * Cfg::B_BYTES + s * Cfg::BROWS * 128, tap * C + cb * 64,
                           tc.n_tile * BN + s * NCHUNK + rank * Cfg::BROWS);
            if (++bi == NB) {
              bi = 0;
              bph ^= 1;
            }
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
      int ai = 0, bi = 0, acc = 0;
      uint32_t aph = 0, bph = 0, acc_phase = 0;
      bool ok = true;
      for (int it = pair; it < p.num_tiles && ok && !*abort_flag; it += npairs) {
        const ConvItem ci = conv_item(p, it, ncb);
        int to = 0;
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, abort_flag, p.status, &to)) {
          if (to) record_wait_site(p.status, 2, ci.pt, -1, acc, acc_phase ^ 1);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN + sc * NCHUNK;
        for (int cb = ci.cb0; cb < ci.cb1 && ok; ++cb) {
          if (!mbar_wait(&a_full[ai], aph, abort_flag, p.status, &to)) {
            if (to) record_wait_site(p.status, 4, ci.pt, cb, ai, aph);
            ok = false;
            break;
          }
          const uint32_t patch = smem_u32(sA + ai * Cfg::PATCH_BYTES);
          for (int tap = 0; tap < 9; ++tap) {
            if (!mbar_wait(&b_full[bi], bph, abort_flag, p.status, &to)) {
              if (to) record_wait_site(p.status, 3, ci.pt, cb, bi, bph);
              ok = false;
              break;
            }
            tc_fence_after();
            // descriptors of k-step k are the k = 0 ones plus 32 bytes (2 in the address field) per step
            const int off = (tap / 3) * Cfg::PATCH_W + tap % 3;  // first patch row of this tap's operand
            const uint64_t adesc = sdesc_kmajor_sw128(patch + off * 128);
            const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + bi * Cfg::B_BYTES) + sc * Cfg::BROWS * 128);
            const uint32_t first = (cb != ci.cb0 || tap != 0) ? 1u : 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) umma2_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, Cfg::IDESC, k ? 1u : first);
            umma2_commit_mc(&b_empty[bi], 0x3);
            if (++bi == NB) {
              bi = 0;
              bph ^= 1;
            }
          }
          if (!ok) break;
          umma2_commit_mc(&a_empty[ai], 0x3);
          if (++ai == 2) {
            ai = 0;
            aph ^= 1;
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
    uint8_t* stg = sB + NB * Cfg::B_BYTES + q * 8192;  // 1024-byte aligned staging of this warp
    int sbuf = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int it = pair; it < p.num_tiles; it += npairs) {
      if (!warp_wait(&tfull_bar[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const ConvItem ci = conv_item(p, it, ncb);
      const TileCoord tc = decode_pair_tile<EPI_CONV>(p, ci.pt, rank);
      const uint32_t t_row = tmem_base + acc * BN + (static_cast<uint32_t>(q * 32) << 16);
      if (ci.half < 0) {
        epilogue_tile_staged<BN, EPI_CONV>(p, tc, t_row, q, lane, stg, sbuf);
      } else {  // fp32 partial of this half, column-quad major ([N / 4][128 rows][4]):
                // a warp's 16-byte stores of one column quad land on 512 contiguous bytes
        float* pbase = p.fix_part + ((static_cast<long>(ci.pt - p.split_first) * 2 + ci.half) * 2 + rank) * 128 * p.N +
                       (q * 32 + lane) * 4;
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
      }
      tc_fence_before();
      mbar_arrive_relaxed_cluster(tempty_leader0 + acc * 8);  // TMEM reads done (wait::ld)
      if (++acc == ACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_read<0>();  // staged stores have read shared memory before it is released
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace edit

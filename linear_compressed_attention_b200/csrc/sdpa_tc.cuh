// Softmax attention blocks of MM-EDiT (section "MM-EDiT", eq. (A^Hybrid)) on
// the 5th-generation tensor cores (tcgen05, accumulators in TMEM, operands
// staged by TMA), bf16 in, fp32 accumulate:
//
//   out = [w0 * out] + sum_s w_s * softmax(q K_s^T / sqrt(d)) V_s
//
// over one or two key sets s, each normalised over its own keys.
//
// Work item: 128 query rows of one (image, head). A persistent CTA takes items
// i, i + gridDim.x, ... and streams every key set of an item through one
// pipeline in tiles of 128 keys; the tile sequence runs on across items.
//   warp 0   TMA producer: the item's Q tile (once), then per key tile the K
//            rows (token-major, K-major operand) and the V^T rows (channel-
//            major with a ones row, K-major operand) into a STAGES-deep ring.
//   warp 1   TMEM owner and MMA issuer: S_g = Q K_g^T (M = 128, N = 128) into
//            one of two TMEM S buffers; then, for the previous tile,
//            O_g = P_g [V_g | 1]^T (M = 128, N = NPV) into one of two TMEM O
//            buffers. Column d of O is the row sum of P (the ones row of V^T),
//            so numerator and denominator come from the same bf16 P.
//   warps 2-9 softmax, two threads per query row (its TMEM lane), one per
//            64-key half of the tile: the half's row max, exchanged with the
//            partner through shared memory; P = 2^(S c - m) rounded to bf16 and
//            written to shared memory as the K-major A operand of the second
//            product (128-byte swizzle); then, for half of the accumulator
//            columns, the running accumulator R = R 2^(m_prev - m) + O of the
//            previous tile (deferred by one tile so that the next tile's
//            exponentials overlap the product), R / l at the end of a key set,
//            and the blended output row at the end of the item.
// Keys past the set's end (the zero-filled or next-image rows of a tile) get
// P = 0. Every wait is bounded (EDIT_ERR_TIMEOUT in the status word).
#pragma once

#include "common.cuh"

namespace edit {

struct SdpaTcParams {
  int Nq, heads, nimg;
  int n1, n2;          // keys of the two sets (n2 = 0: one set)
  float w0, w1, w2;    // out = [w0 * out] + w1 A_1 + w2 A_2
  int blend_in;
  void* out;
  long ldo;
  int* status;
  // exact mixing weights instead of w0..w2: one key set with blend_in mixes
  // with the linear part, whose normaliser (Q z + eps) is den [img][row][head];
  // two key sets mix by their softmax normalisers (one softmax over both)
  int exact;
  const float* den;
};

template <int D>
struct SdpaTcCfg {
  static_assert(D == 32 || D == 64 || D == 72, "head width");
  static constexpr int NBX = (D + 63) / 64;          // 64-column boxes of a Q / K row
  static constexpr int KS = (D + 15) / 16;           // k-steps of q . k
  static constexpr int NPV = (D + 1 <= 48) ? 48 : 80;  // [V | 1] rows: MMA N of the second product
  static constexpr int STAGES = (D == 72) ? 2 : 3;
  static constexpr int QB = (D == 72) ? 1 : 2;       // Q tile buffers
  static constexpr int QBOX = 128 * 128;             // one 128-row x 128-byte box
  static constexpr int Q_BYTES = QB * NBX * QBOX;
  static constexpr int K_BYTES = STAGES * NBX * QBOX;
  static constexpr int VBOX = NPV * 128;             // NPV rows x 64 keys
  static constexpr int V_BYTES = STAGES * 2 * VBOX;
  static constexpr int P_BYTES = 2 * 2 * QBOX;       // two P buffers of 128 rows x 128 keys
  static constexpr int XCH_BYTES = (2 * 2 * 128 + 128) * 4;  // row-max exchange (2 tiles x 2 halves), l exchange
  static constexpr int BAR_BYTES = (2 * QB + 2 * STAGES + 10) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + Q_BYTES + K_BYTES + V_BYTES + P_BYTES + XCH_BYTES + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(128, NPV);
  static constexpr int TMEM_COLS = 512;  // S buffers at 0, 128; O buffers at 256, 384
  static constexpr int OC = (D + 16) / 16;    // 16-column chunks of [O | l] (d + 1 columns)
  static constexpr int OC0 = (OC + 1) / 2;    // chunks of the first softmax half
  static constexpr int OCH = OC0;             // most chunks a half holds
};

// 2^x with the SFU's approximate exponential (flushes denormals; P is rounded
// to bf16 right after, far coarser than its error).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 32 lanes x N consecutive fp32 columns (N = 32 or 64), waited for.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[N]);
template <>
__device__ __forceinline__ void tmem_ld_cols<64>(uint32_t taddr, float (&v)[64]) {
  tmem_ld64(taddr, v);
}
template <>
__device__ __forceinline__ void tmem_ld_cols<32>(uint32_t taddr, float (&v)[32]) {
  float a[16], b[16];
  tmem_ld16(taddr, a);
  tmem_ld16(taddr + 16, b);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = a[i];
    v[16 + i] = b[i];
  }
}

// NSET: number of key sets (1: image rows, 2: prompt rows); with two sets
// the first set's share waits in registers for the second's.
template <int D, int NSET>
__global__ void __launch_bounds__(320, 1) sdpa_tc_kernel(const __grid_constant__ CUtensorMap mq,
                                                         const __grid_constant__ CUtensorMap mk1,
                                                         const __grid_constant__ CUtensorMap mv1,
                                                         const __grid_constant__ CUtensorMap mk2,
                                                         const __grid_constant__ CUtensorMap mv2,
                                                         const SdpaTcParams p) {
  using Cfg = SdpaTcCfg<D>;
  constexpr int NBX = Cfg::NBX, KS = Cfg::KS, NPV = Cfg::NPV, STAGES = Cfg::STAGES, QB = Cfg::QB;
  constexpr int QBOX = Cfg::QBOX, VBOX = Cfg::VBOX, OC = Cfg::OC, OC0 = Cfg::OC0, OCH = Cfg::OCH;
  constexpr int CW = 32, NCW = 2;  // S columns read at a time (a chunk at a time keeps registers for the rest)
  constexpr int NOLD = 16 * OCH / 8;  // 16-byte pieces of a thread's share of an output row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sQ = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sQ + Cfg::Q_BYTES;
  uint8_t* sV = sK + Cfg::K_BYTES;
  uint8_t* sP = sV + Cfg::V_BYTES;
  float* mx = reinterpret_cast<float*>(sP + Cfg::P_BYTES);  // [2 tiles][2 halves][128 rows]
  float* lsum = mx + 2 * 2 * 128;                          // [128 rows]
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sP + Cfg::P_BYTES + Cfg::XCH_BYTES);
  uint64_t* q_empty = q_full + QB;
  uint64_t* kv_full = q_empty + QB;
  uint64_t* kv_empty = kv_full + STAGES;
  uint64_t* s_full = kv_empty + STAGES;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* o_empty = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < QB; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);  // one arrival per softmax warp
      mbar_init(&p_full[i], 8);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mq);
    tma_prefetch_desc(&mk1);
    tma_prefetch_desc(&mv1);
    if (p.n2 > 0) {
      tma_prefetch_desc(&mk2);
      tma_prefetch_desc(&mv2);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  const int qtiles = (p.Nq + 127) / 128;
  const long nitems = static_cast<long>(p.nimg) * p.heads * qtiles;
  const int T1 = (p.n1 + 127) / 128, T2 = (p.n2 + 127) / 128, T = T1 + T2;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      long g = 0;
      int li = 0;
      bool ok = true;
      for (long it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
        const int qt = static_cast<int>(it % qtiles);
        const long bh = it / qtiles;
        const int h = static_cast<int>(bh % p.heads), b = static_cast<int>(bh / p.heads);
        const int qb = li % QB;
        if (!mbar_wait(&q_empty[qb], ((li / QB) & 1) ^ 1, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&q_full[qb], NBX * QBOX);
#pragma unroll
        for (int bx = 0; bx < NBX; ++bx)
          tma_load_3d(&mq, &q_full[qb], sQ + (qb * NBX + bx) * QBOX, 64 * bx, h, b * p.Nq + qt * 128);
        for (int t = 0; t < T; ++t, ++g) {
          const bool one = t < T1;
          const int tt = one ? t : t - T1;
          const int n = one ? p.n1 : p.n2;
          const int st = static_cast<int>(g % STAGES);
          if (!mbar_wait(&kv_empty[st], static_cast<uint32_t>((g / STAGES) & 1) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[st], NBX * QBOX + 2 * VBOX);
#pragma unroll
          for (int bx = 0; bx < NBX; ++bx)
            tma_load_3d(one ? &mk1 : &mk2, &kv_full[st], sK + (st * NBX + bx) * QBOX, 64 * bx, h, b * n + tt * 128);
#pragma unroll
          for (int kx = 0; kx < 2; ++kx)
            tma_load_2d(one ? &mv1 : &mv2, &kv_full[st], sV + (st * 2 + kx) * VBOX, tt * 128 + 64 * kx,
                        (b * p.heads + h) * NPV);
        }
      }
      if (*abort_flag) {  // let copies already issued land before the block exits
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      long g = 0;
      int li = 0;
      bool ok = true;
      // O_gg = P_gg [V_gg | 1]^T for a tile whose P the softmax warps have written
      auto issue_pv = [&](long gg) -> bool {
        const int ob = static_cast<int>(gg & 1);
        const uint32_t ph = static_cast<uint32_t>((gg >> 1) & 1);
        if (!mbar_wait(&p_full[ob], ph, abort_flag, p.status)) return false;
        if (!mbar_wait(&o_empty[ob], ph ^ 1u, abort_flag, p.status)) return false;
        tc_fence_after();
        const int st = static_cast<int>(gg % STAGES);
        const uint32_t pa = smem_u32(sP + ob * 2 * QBOX), va = smem_u32(sV + st * 2 * VBOX);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint64_t ad = sdesc_kmajor_sw128(pa + (s >> 2) * QBOX + (s & 3) * 32);
          const uint64_t bd = sdesc_kmajor_sw128(va + (s >> 2) * VBOX + (s & 3) * 32);
          umma_bf16(tmem_base + 256 + 128 * ob, ad, bd, Cfg::IDESC_O, s > 0 ? 1u : 0u);
        }
        umma_commit(&o_full[ob]);
        umma_commit(&kv_empty[st]);
        return true;
      };
      for (long it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
        const int qb = li % QB;
        if (!mbar_wait(&q_full[qb], (li / QB) & 1, abort_flag, p.status)) break;
        const uint32_t qa = smem_u32(sQ + qb * NBX * QBOX);
        for (int t = 0; t < T; ++t, ++g) {
          const int st = static_cast<int>(g % STAGES);
          const int sb = static_cast<int>(g & 1);
          if (!mbar_wait(&kv_full[st], static_cast<uint32_t>((g / STAGES) & 1), abort_flag, p.status) ||
              !mbar_wait(&s_empty[sb], static_cast<uint32_t>((g >> 1) & 1) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ka = smem_u32(sK + st * NBX * QBOX);
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            const uint64_t ad = sdesc_kmajor_sw128(qa + (kk >> 2) * QBOX + (kk & 3) * 32);
            const uint64_t bd = sdesc_kmajor_sw128(ka + (kk >> 2) * QBOX + (kk & 3) * 32);
            umma_bf16(tmem_base + 128 * sb, ad, bd, Cfg::IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[sb]);
          if (t == T - 1) umma_commit(&q_empty[qb]);  // the item's last reads of its Q tile
          if (g > 0 && !issue_pv(g - 1)) {
            ok = false;
            break;
          }
        }
      }
      if (ok && g > 0) issue_pv(g - 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / output
    // Two warps per TMEM lane quarter: half hf of the warps takes keys
    // 64 hf .. 64 hf + 63 of every tile (one 64-key sub-buffer of P) and the
    // accumulator columns [16 OC0 hf, ...) (the l column d lies in half 1).
    const int q4 = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int row = q4 * 32 + lane;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q4 * 32) << 16);
    const float c = rsqrtf(static_cast<float>(D)) * 1.4426950408889634f;  // 1/sqrt(d) * log2(e): base-2 exponent
    const uint32_t psw = static_cast<uint32_t>(row & 7);
    uint8_t* prow = sP + hf * QBOX + row * 128;  // + sb * 2 * QBOX: P buffer of the tile
    const int col0 = hf ? 16 * OC0 : 0;  // first accumulator column of this half
    const int nch = hf ? OC - OC0 : OC0;  // its 16-column chunks
    long g = 0;
    bool ok = true;
    float R[16 * OCH];
    float acc[NSET == 2 ? 16 * OCH : 1];  // the first set's share (two sets only)
    for (long it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const int qt = static_cast<int>(it % qtiles);
      const long bh = it / qtiles;
      const int h = static_cast<int>(bh % p.heads), b = static_cast<int>(bh / p.heads);
      float sc = 0.f;
      // the output row's current values (blended in at the end), fetched now
      // so that their latency hides behind the item's tiles
      const int r = qt * 128 + row;
      __nv_bfloat16* og =
          reinterpret_cast<__nv_bfloat16*>(p.out) + (static_cast<long>(b) * p.Nq + r) * p.ldo + h * D + col0;
      // (one key set only: with two, the registers hold the first set's share)
      uint4 oldv[NSET == 1 ? NOLD : 1];
      if (NSET == 1) {
#pragma unroll
        for (int k = 0; k < NOLD; ++k)
          oldv[NSET == 1 ? k : 0] = (p.blend_in && r < p.Nq && col0 + 8 * k < D)
                                        ? *reinterpret_cast<const uint4*>(og + 8 * k)
                                        : make_uint4(0u, 0u, 0u, 0u);
      }
      // exact: log2 of the other part's normaliser (the linear part's den, one set)
      float lz_other = 0.f, lz0 = 0.f;
      if (NSET == 1 && p.exact && r < p.Nq) lz_other = log2f(p.den[(static_cast<long>(b) * p.Nq + r) * p.heads + h]);
      for (int set = 0; set < NSET && ok; ++set) {
        const int n = set == 0 ? p.n1 : p.n2;
        const int Ts = set == 0 ? T1 : T2;
        if (Ts == 0) continue;
#pragma unroll
        for (int i = 0; i < 16 * OCH; ++i) R[i] = 0.f;
        float m_run = -INFINITY, m_acc = -INFINITY, m_pend = -INFINITY;
        // R = R 2^(m_acc - m_j) + O_j (this half's columns) for tile gg whose P used the max m_j
        auto accumulate = [&](long gg, float m_j) -> bool {
          const int ob = static_cast<int>(gg & 1);
          if (!warp_wait(&o_full[ob], static_cast<uint32_t>((gg >> 1) & 1), abort_flag, p.status)) return false;
          tc_fence_after();
          const float alpha = ex2_approx(m_acc - m_j);
          m_acc = m_j;
#pragma unroll
          for (int ch = 0; ch < OCH; ++ch) {
            if (ch < nch) {
              float v[16];
              tmem_ld16(t_lane + 256 + 128 * ob + col0 + 16 * ch, v);
#pragma unroll
              for (int i = 0; i < 16; ++i) R[16 * ch + i] = fmaf(R[16 * ch + i], alpha, v[i]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_empty[ob]);
          return true;
        };
        for (int tt = 0; tt < Ts; ++tt, ++g) {
          const int sb = static_cast<int>(g & 1);
          if (!warp_wait(&s_full[sb], static_cast<uint32_t>((g >> 1) & 1), abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // valid keys of this half: 0 .. nv - 1
          int nv = n - tt * 128 - 64 * hf;
          nv = nv < 0 ? 0 : (nv > 64 ? 64 : nv);
          const uint32_t s_addr = t_lane + 128 * sb + 64 * hf;
          float v[CW];
          float mt = -INFINITY;
#pragma unroll
          for (int k = 0; k < NCW; ++k) {
            if (nv > CW * k) {
              tmem_ld_cols<CW>(s_addr + CW * k, v);
              if (nv == 64) {
#pragma unroll
                for (int i = 0; i < CW; ++i) mt = fmaxf(mt, v[i]);
              } else {
#pragma unroll
                for (int i = 0; i < CW; ++i)
                  if (CW * k + i < nv) mt = fmaxf(mt, v[i]);
              }
            }
          }
          // the row max of the tile: both halves exchange theirs
          float* mxb = mx + (g & 1) * 256;
          mxb[hf * 128 + row] = mt;
          named_bar_sync(1 + q4, 64);
          const float m_new = fmaxf(m_run, fmaxf(mt, mxb[(hf ^ 1) * 128 + row]) * c);
          m_run = m_new;
          // P = 2^(S c - m) in bf16, 128-byte-swizzled K-major rows of this half's sub-buffer
#pragma unroll
          for (int k = 0; k < NCW; ++k) {
            if (NCW > 1 && nv > CW * k) tmem_ld_cols<CW>(s_addr + CW * k, v);  // (one chunk held at a time)
#pragma unroll
            for (int q8 = 0; q8 < CW / 8; ++q8) {
              float e[8];
              const int key0 = CW * k + 8 * q8;
              if (nv == 64) {
#pragma unroll
                for (int i = 0; i < 8; ++i) e[i] = ex2_approx(fmaf(v[8 * q8 + i], c, -m_new));
              } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) e[i] = key0 + i < nv ? ex2_approx(fmaf(v[8 * q8 + i], c, -m_new)) : 0.f;
              }
              uint4 w;
              w.x = pack_bf16x2(e[0], e[1]);
              w.y = pack_bf16x2(e[2], e[3]);
              w.z = pack_bf16x2(e[4], e[5]);
              w.w = pack_bf16x2(e[6], e[7]);
              *reinterpret_cast<uint4*>(prow + sb * 2 * QBOX + ((static_cast<uint32_t>(key0 >> 3) ^ psw) << 4)) = w;
            }
          }
          fence_proxy_async_smem();  // P is read by the tensor cores (async proxy)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&s_empty[sb]);
            mbar_arrive(&p_full[sb]);
          }
          if (tt > 0 && !accumulate(g - 1, m_pend)) {
            ok = false;
            break;
          }
          m_pend = m_new;
          if (tt == Ts - 1 && !accumulate(g, m_new)) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        // l = column d (half 1) to both halves, then acc += w R / l
        if (hf) lsum[row] = R[D - 16 * OC0];
        named_bar_sync(1 + q4, 64);
        const float l = lsum[row];
        named_bar_sync(1 + q4, 64);  // (lsum is rewritten at the next set's end)
        const float w = p.exact ? 1.f : (set == 0 ? p.w1 : p.w2);
        sc = l > 0.f ? w / l : 0.f;
        if (set == 0) lz0 = m_run + log2f(l);  // log2 of the set's normaliser sum_j exp(q.k_j / sqrt(d))
        if (NSET == 2 && set == 1) lz_other = m_run + log2f(l);
        if (NSET == 2 && set == 0) {
#pragma unroll
          for (int i = 0; i < 16 * OCH; ++i) acc[NSET == 2 ? i : 0] = R[i] * sc;
        }
      }
      if (!ok) break;
      if (r < p.Nq) {
        float w0e = p.w0;  // weight of the blended-in values (eta when exact)
#pragma unroll
        for (int c8 = 0; c8 < 16 * OCH; c8 += 8) {
          if (col0 + c8 < D) {
            float o[8];
            if (p.exact) {
              // eta = A / (A + B) as 1 / (1 + 2^(log2 B - log2 A)): one set, A = the linear
              // part's normaliser, B = this set's; two sets, A = the first's, B = the second's
              const float eta = NSET == 2 ? 1.f / (1.f + exp2f(lz_other - lz0)) : 1.f / (1.f + exp2f(lz0 - lz_other));
#pragma unroll
              for (int i = 0; i < 8; ++i)
                o[i] = NSET == 2 ? eta * acc[NSET == 2 ? c8 + i : 0] + (1.f - eta) * R[c8 + i] * sc
                                 : (1.f - eta) * R[c8 + i] * sc;
              w0e = eta;
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                o[i] = NSET == 2 ? fmaf(R[c8 + i], sc, acc[NSET == 2 ? c8 + i : 0]) : R[c8 + i] * sc;
            }
            if (p.blend_in) {
              const uint4 old = NSET == 1 ? oldv[NSET == 1 ? c8 / 8 : 0] : *reinterpret_cast<const uint4*>(og + c8);
              const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                o[2 * i] = fmaf(w0e, __uint_as_float(ow[i] << 16), o[2 * i]);
                o[2 * i + 1] = fmaf(w0e, __uint_as_float(ow[i] & 0xffff0000u), o[2 * i + 1]);
              }
            }
            uint4 wv;
            wv.x = pack_bf16x2(o[0], o[1]);
            wv.y = pack_bf16x2(o[2], o[3]);
            wv.z = pack_bf16x2(o[4], o[5]);
            wv.w = pack_bf16x2(o[6], o[7]);
            *reinterpret_cast<uint4*>(og + c8) = wv;
          }
        }
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

// [V | 1]^T operand of the softmax blocks: VT[b][h][c][j] = V[b][j][h d + c]
// for c < d, row d = 1 for the set's n keys, every other row and every key
// j >= n zero; rows NPV per head, keys padded to nkp (a multiple of 128).
// One block per (64 keys, head, image): the 64 token rows are read with
// 16-byte loads into shared memory and written out transposed, 16 bytes per
// thread.
template <int D, int NPV>
__global__ void __launch_bounds__(256) vt_ones_kernel(const __nv_bfloat16* __restrict__ V, long ldv, int n, int nkp,
                                                     int heads, __nv_bfloat16* __restrict__ VT) {
  pdl_wait();
  __shared__ __align__(16) __nv_bfloat16 tile[64][D + 8];
  const int j0 = blockIdx.x * 64, h = blockIdx.y, b = blockIdx.z;
  for (int e = threadIdx.x; e < 64 * (D / 8); e += blockDim.x) {
    const int r = e / (D / 8), c8 = (e - r * (D / 8)) * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j0 + r < n) v = *reinterpret_cast<const uint4*>(V + (static_cast<long>(b) * n + j0 + r) * ldv + h * D + c8);
    *reinterpret_cast<uint4*>(&tile[r][c8]) = v;
  }
  __syncthreads();
  const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
  for (int e = threadIdx.x; e < NPV * 8; e += blockDim.x) {
    const int c = e >> 3, k8 = (e & 7) * 8;
    __align__(16) __nv_bfloat16 o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool in = j0 + k8 + i < n;
      o[i] = c < D ? (in ? tile[k8 + i][c] : zero) : (c == D && in ? one : zero);
    }
    *reinterpret_cast<uint4*>(VT + ((static_cast<long>(b) * heads + h) * NPV + c) * nkp + j0 + k8) =
        *reinterpret_cast<const uint4*>(o);
  }
}

}  // namespace edit

// Softmax attention blocks of MM-EDiT (section "MM-EDiT", eq. (A^Hybrid)) on
// the tensor cores, bf16 in, fp32 accumulate:
//
//   out = [w0 * out] + sum_s w_s * softmax(q K_s^T / sqrt(d)) V_s
//
// over one or two key sets s, each normalised over its own keys. Flash-style
// (one pass over the keys, online softmax): a block holds 64 query rows of one
// (image, head), 16 per warp; Q stays in registers as mma.sync A fragments;
// each 64-key tile of K (row-major) and V (transposed, so its B fragments are
// contiguous pairs) is staged in shared memory with rows padded by 16 bytes,
// which makes every fragment load bank-conflict free. S = Q K^T and O += P V
// are m16n8k16 MMAs; the S accumulator tiles are repacked in registers as the
// A fragments of P. Head widths that are not a multiple of 16 (d = 72) are
// zero-padded to whole k-steps for q . k; the output keeps d columns.
//
// mma.sync rather than tcgen05: the work is 11 GFLOP at the MM-EDiT 1024 px
// shape, in blocks of 333 prompt keys or 333 prompt queries, which a register
// pipeline with no TMEM round trip serves well.
#pragma once

#include "common.cuh"

namespace edit {

// Parameters of one softmax-attention launch (token-major operands).
struct SdpaParams {
  const void* q;
  long ldq;
  const void* k1;
  const void* v1;
  long ld1;
  int n1;
  const void* k2;
  const void* v2;
  long ld2;
  int n2;
  void* out;
  long ldo;
  int Nq, heads, d;
  float w0, w1, w2;
  int blend_in;
  // Key-split mode (part != nullptr): the first key set is cut into nchunk1
  // ranges and every block handles one (64-query tile, key range) item; the
  // second set, if any, is one more item. Each item writes its unnormalised
  // accumulator, running max (log2 units) and sum per query row to
  // part [img][head][Nq][items][d + 2]; sdpa_combine_kernel merges them.
  int nchunk1, nimg;
  float* part;
};

namespace {

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

template <int D>
struct SdpaMmaCfg {
  static_assert(D % 8 == 0 && D <= 128, "head width");
  static constexpr int DP = (D + 15) / 16 * 16;  // q . k depth padded to whole k-steps
  static constexpr int KS = DP / 16;             // k-steps of q . k
  static constexpr int NO = D / 8;               // 8-column output tiles
  static constexpr int RS = DP + 8;              // Q / K row stride in shared memory (elements)
  static constexpr int KT = 64;                  // keys per tile
  static constexpr int VS = KT + 8;              // V^T row stride (elements)
};

template <int D>
__global__ void __launch_bounds__(128) sdpa_mma_kernel(SdpaParams p) {
  using Cfg = SdpaMmaCfg<D>;
  constexpr int DP = Cfg::DP, KS = Cfg::KS, NO = Cfg::NO, RS = Cfg::RS, KT = Cfg::KT, VS = Cfg::VS;
  pdl_wait();
  __shared__ __align__(16) __nv_bfloat16 qs[64 * RS];
  __shared__ __align__(16) __nv_bfloat16 ks[KT * RS];
  __shared__ __align__(16) __nv_bfloat16 vt[DP * VS];
  const int h = blockIdx.y, b = blockIdx.z;
  const int nitem = p.part ? p.nchunk1 + (p.n2 > 0 ? 1 : 0) : 1;
  const int qt = blockIdx.x / nitem, item = blockIdx.x - qt * nitem;
  const int row0 = qt * 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  // ---- this block's 64 query rows (rows >= Nq and columns >= D read as 0)
  {
    const __nv_bfloat16* qg = reinterpret_cast<const __nv_bfloat16*>(p.q) + static_cast<long>(b) * p.Nq * p.ldq + h * D;
    for (int e = threadIdx.x; e < 64 * (DP / 8); e += 128) {
      const int r = e / (DP / 8), c8 = (e - r * (DP / 8)) * 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row0 + r < p.Nq && c8 < D) v = *reinterpret_cast<const uint4*>(qg + static_cast<long>(row0 + r) * p.ldq + c8);
      *reinterpret_cast<uint4*>(qs + r * RS + c8) = v;
    }
  }
  __syncthreads();
  uint32_t qa[KS][4];  // A fragments of the warp's 16 rows
  {
    const __nv_bfloat16* qw = qs + warp * 16 * RS;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = lds32(qw + g * RS + 16 * kk + 2 * t);
      qa[kk][1] = lds32(qw + (g + 8) * RS + 16 * kk + 2 * t);
      qa[kk][2] = lds32(qw + g * RS + 16 * kk + 8 + 2 * t);
      qa[kk][3] = lds32(qw + (g + 8) * RS + 16 * kk + 8 + 2 * t);
    }
  }
  const float qscale = rsqrtf(static_cast<float>(D)) * 1.4426950408889634f;  // 1/sqrt(d) * log2(e): exp2 below
  float res[NO][4];
#pragma unroll
  for (int o = 0; o < NO; ++o) res[o][0] = res[o][1] = res[o][2] = res[o][3] = 0.f;
  float pm[2] = {0.f, 0.f}, pl[2] = {0.f, 0.f};  // key-split mode: the item's running max and sum per row

  // one key set: res += w * softmax(q K^T / sqrt(d)) V for rows g and g + 8 of this warp
  // (raw: res = the unnormalised accumulator, max and sum kept in pm / pl)
  auto one_set = [&](const __nv_bfloat16* kb, const __nv_bfloat16* vb, long ld, int nk, float w, bool raw) {
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float acc[NO][4];
#pragma unroll
    for (int o = 0; o < NO; ++o) acc[o][0] = acc[o][1] = acc[o][2] = acc[o][3] = 0.f;
    for (int j0 = 0; j0 < nk; j0 += KT) {
      __syncthreads();  // the previous tile has been read by every warp
      for (int e = threadIdx.x; e < KT * (DP / 8); e += 128) {  // K rows, 16 bytes per thread
        const int r = e / (DP / 8), c8 = (e - r * (DP / 8)) * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (j0 + r < nk && c8 < D) v = *reinterpret_cast<const uint4*>(kb + static_cast<long>(j0 + r) * ld + c8);
        *reinterpret_cast<uint4*>(ks + r * RS + c8) = v;
      }
      for (int e = threadIdx.x; e < KT * (DP / 8); e += 128) {  // V transposed: consecutive threads, consecutive keys
        const int r = e % KT, c8 = (e / KT) * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (j0 + r < nk && c8 < D) v = *reinterpret_cast<const uint4*>(vb + static_cast<long>(j0 + r) * ld + c8);
        const __nv_bfloat16* v8 = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
        for (int i = 0; i < 8; ++i) vt[(c8 + i) * VS + r] = v8[i];
      }
      __syncthreads();
      // S = Q K^T: 8 tiles of 8 keys
      float s[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          const __nv_bfloat16* kr = ks + (8 * nt + g) * RS + 16 * kk + 2 * t;
          mma_16816(s[nt], qa[kk], lds32(kr), lds32(kr + 8));
        }
      }
      // scale, mask keys >= nk, running max of rows g (0, 1) and g + 8 (2, 3)
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = j0 + 8 * nt + 2 * t + (e & 1);
          const float v = key < nk ? s[nt][e] * qscale : -INFINITY;
          s[nt][e] = v;
          if (e < 2)
            mx0 = fmaxf(mx0, v);
          else
            mx1 = fmaxf(mx1, v);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: every tile has a key < nk
      const float c0 = exp2f(m0 - mn0), c1 = exp2f(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      l0 *= c0;
      l1 *= c1;
#pragma unroll
      for (int o = 0; o < NO; ++o) {
        acc[o][0] *= c0;
        acc[o][1] *= c0;
        acc[o][2] *= c1;
        acc[o][3] *= c1;
      }
      // P (row sums in fp32, A fragments in bf16) and O += P V
      uint32_t pa[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f(s[nt][0] - m0), p1 = exp2f(s[nt][1] - m0);
        const float p2 = exp2f(s[nt][2] - m1), p3 = exp2f(s[nt][3] - m1);
        l0 += p0 + p1;
        l1 += p2 + p3;
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(p2, p3);
      }
#pragma unroll
      for (int o = 0; o < NO; ++o) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const __nv_bfloat16* vr = vt + (8 * o + g) * VS + 16 * kk + 2 * t;
          mma_16816(acc[o], pa[kk], lds32(vr), lds32(vr + 8));
        }
      }
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (raw) {
      pm[0] = m0;
      pm[1] = m1;
      pl[0] = l0;
      pl[1] = l1;
#pragma unroll
      for (int o = 0; o < NO; ++o)
#pragma unroll
        for (int e = 0; e < 4; ++e) res[o][e] = acc[o][e];
      return;
    }
    const float s0 = l0 > 0.f ? w / l0 : 0.f, s1 = l1 > 0.f ? w / l1 : 0.f;
#pragma unroll
    for (int o = 0; o < NO; ++o) {
      res[o][0] = fmaf(acc[o][0], s0, res[o][0]);
      res[o][1] = fmaf(acc[o][1], s0, res[o][1]);
      res[o][2] = fmaf(acc[o][2], s1, res[o][2]);
      res[o][3] = fmaf(acc[o][3], s1, res[o][3]);
    }
  };

  const __nv_bfloat16* k1 = reinterpret_cast<const __nv_bfloat16*>(p.k1) + static_cast<long>(b) * p.n1 * p.ld1 + h * D;
  const __nv_bfloat16* v1 = reinterpret_cast<const __nv_bfloat16*>(p.v1) + static_cast<long>(b) * p.n1 * p.ld1 + h * D;
  const __nv_bfloat16* k2 = reinterpret_cast<const __nv_bfloat16*>(p.k2) + static_cast<long>(b) * p.n2 * p.ld2 + h * D;
  const __nv_bfloat16* v2 = reinterpret_cast<const __nv_bfloat16*>(p.v2) + static_cast<long>(b) * p.n2 * p.ld2 + h * D;
  if (p.part) {
    // one item: a range of the first key set, or the whole second set
    if (item < p.nchunk1) {
      const int j0 = static_cast<int>(static_cast<long>(item) * p.n1 / p.nchunk1);
      const int j1 = static_cast<int>(static_cast<long>(item + 1) * p.n1 / p.nchunk1);
      one_set(k1 + static_cast<long>(j0) * p.ld1, v1 + static_cast<long>(j0) * p.ld1, p.ld1, j1 - j0, 1.f, true);
    } else {
      one_set(k2, v2, p.ld2, p.n2, 1.f, true);
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = row0 + warp * 16 + g + 8 * half;
      if (r >= p.Nq) continue;
      float* pp = p.part + ((static_cast<long>(b * p.heads + h) * p.Nq + r) * nitem + item) * (D + 2);
#pragma unroll
      for (int o = 0; o < NO; ++o)
        *reinterpret_cast<float2*>(pp + 8 * o + 2 * t) = make_float2(res[o][2 * half], res[o][2 * half + 1]);
      if (t == 0) {
        pp[D] = pm[half];
        pp[D + 1] = pl[half];
      }
    }
    return;
  }
  one_set(k1, v1, p.ld1, p.n1, p.w1, false);
  if (p.n2 > 0) one_set(k2, v2, p.ld2, p.n2, p.w2, false);

  // ---- store (blending in w0 * out): rows g and g + 8, columns 8 o + 2 t, 2 t + 1
  __nv_bfloat16* og = reinterpret_cast<__nv_bfloat16*>(p.out) + static_cast<long>(b) * p.Nq * p.ldo + h * D;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = row0 + warp * 16 + g + 8 * half;
    if (r >= p.Nq) continue;
#pragma unroll
    for (int o = 0; o < NO; ++o) {
      float v0 = res[o][2 * half], v1 = res[o][2 * half + 1];
      uint32_t* dst = reinterpret_cast<uint32_t*>(og + static_cast<long>(r) * p.ldo + 8 * o + 2 * t);
      if (p.blend_in) {
        const uint32_t old = *dst;
        v0 = fmaf(p.w0, __uint_as_float(old << 16), v0);
        v1 = fmaf(p.w0, __uint_as_float(old & 0xffff0000u), v1);
      }
      *dst = pack_bf16x2(v0, v1);
    }
  }
}

// Merge of the key-split items, one warp per (image, head, query row), fixed
// order: the first set's ranges by the usual max / rescale / sum rule, then
// out = [w0 out +] w1 softmax_1 V_1 + w2 softmax_2 V_2.
__global__ void __launch_bounds__(256) sdpa_combine_kernel(SdpaParams p) {
  pdl_wait();
  const int D = p.d, nitem = p.nchunk1 + (p.n2 > 0 ? 1 : 0);
  const long row = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;  // (img * heads + h) * Nq + r
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long>(p.nimg) * p.heads * p.Nq) return;
  const int r = static_cast<int>(row % p.Nq);
  const long bh = row / p.Nq;
  const int h = static_cast<int>(bh % p.heads), b = static_cast<int>(bh / p.heads);
  const float* pp = p.part + row * nitem * (D + 2);
  float M = -INFINITY;
  for (int c = 0; c < p.nchunk1; ++c) M = fmaxf(M, pp[c * (D + 2) + D]);
  float L = 0.f;
  for (int c = 0; c < p.nchunk1; ++c) L += pp[c * (D + 2) + D + 1] * exp2f(pp[c * (D + 2) + D] - M);
  const float s1 = p.w1 / L;
  const float* p2 = pp + p.nchunk1 * (D + 2);
  const float s2 = p.n2 > 0 ? p.w2 / p2[D + 1] : 0.f;
  __nv_bfloat16* og = reinterpret_cast<__nv_bfloat16*>(p.out) + (static_cast<long>(b) * p.Nq + r) * p.ldo + h * D;
  for (int col = lane; col < D; col += 32) {
    float a = 0.f;
    for (int c = 0; c < p.nchunk1; ++c) a += pp[c * (D + 2) + col] * exp2f(pp[c * (D + 2) + D] - M);
    float v = a * s1;
    if (p.n2 > 0) v += p2[col] * s2;
    if (p.blend_in) v = fmaf(p.w0, __bfloat162float(og[col]), v);
    og[col] = __float2bfloat16_rn(v);
  }
}

}  // namespace
}  // namespace edit

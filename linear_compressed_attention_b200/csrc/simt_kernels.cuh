// CUDA-core kernels of the EDiT layer: the memory-bound steps (GroupNorm,
// depthwise stride-2 conv, KV-state reduction, apply, softmax attention for
// the prompt blocks of MM-EDiT) and an fp32 tiled GEMM used by the fp32 path
// (fp32 storage must stay fp32 end to end, so it does not go to the bf16
// tensor cores).
#pragma once

#include "common.cuh"

namespace edit {

// Parameters of one softmax-attention launch of the CUDA-core path (fp32),
// token-major operands: out = [w0 * out] + w1 softmax(q k1^T / sqrt(d)) v1
// (+ w2 softmax(q k2^T / sqrt(d)) v2 when n2 > 0).
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
  // exact mixing weights instead of w0..w2 (one key set with blend_in: eta
  // from den [b][row][head] = the linear part's normaliser; two key sets:
  // eta from the two softmax normalisers)
  int exact;
  const float* den;
};
namespace {  // internal linkage: each translation unit that uses these keeps its own copy

// ====================================================================== GEMM
// out[m, n] = act(sum_k A(m, k) * Bw(n, k) + bias(n)), fp32.
// A(m, k): conv mode: implicit 3x3 im2col of X[B,H,W,Cin] with zero padding,
//          k = tap * Cin + c, tap = kh * 3 + kw;
//          else [A0 | A1] with A0 [M][K0], A1 [M][K1].
// Bw(n, k): source s = n / n_split holds rows [s*n_split, (s+1)*n_split) of
//          the first K0 columns; bk [N][K1] holds columns K0.. .
struct SimtGemmParams {
  const float* a0;
  const float* a1;
  int K0, K1;
  const float* b[3];
  const float* bk;
  int n_split;
  int M, N;
  int conv, B, H, W, Cin;
  float* out;
  int ldo;
  const float* bias[3];
  int relu;
};

__device__ __forceinline__ float simt_load_a(const SimtGemmParams& p, int m, int k) {
  if (m >= p.M || k >= p.K0 + p.K1) return 0.f;
  if (p.conv) {
    const int hw = p.H * p.W;
    const int b = m / hw, r = m - b * hw;
    const int h = r / p.W, w = r - h * p.W;
    const int tap = k / p.Cin, c = k - tap * p.Cin;
    const int hh = h + tap / 3 - 1, ww = w + tap % 3 - 1;
    if (hh < 0 || hh >= p.H || ww < 0 || ww >= p.W) return 0.f;
    return p.a0[((static_cast<long>(b) * p.H + hh) * p.W + ww) * p.Cin + c];
  }
  if (k < p.K0) return p.a0[static_cast<long>(m) * p.K0 + k];
  return p.a1[static_cast<long>(m) * p.K1 + (k - p.K0)];
}

__device__ __forceinline__ float simt_load_b(const SimtGemmParams& p, int n, int k) {
  if (n >= p.N || k >= p.K0 + p.K1) return 0.f;
  if (k < p.K0) {
    const int s = n / p.n_split;
    return p.b[s][static_cast<long>(n - s * p.n_split) * p.K0 + k];
  }
  return p.bk[static_cast<long>(n) * p.K1 + (k - p.K0)];
}

// 64 x 64 output tile, 256 threads, 4 x 4 outputs per thread (strided by 16).
__global__ void __launch_bounds__(256) simt_gemm_f32(SimtGemmParams p) {
  pdl_wait();
  __shared__ float As[16][65];
  __shared__ float Bs[16][65];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  const int K = p.K0 + p.K1;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 1024; i += 256) {
      const int r = i >> 4, kk = i & 15;
      As[kk][r] = simt_load_a(p, m0 + r, k0 + kk);
      Bs[kk][r] = simt_load_b(p, n0 + r, k0 + kk);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty + 16 * i];
        b[i] = Bs[kk][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= p.N) continue;
      const int s = n / p.n_split;
      float v = acc[i][j];
      if (p.bias[s]) v += p.bias[s][n - s * p.n_split];
      if (p.relu) v = act_apply(v, p.relu);
      p.out[static_cast<long>(m) * p.ldo + n] = v;
    }
  }
}

// ================================================================ GroupNorm
// Partial sums of U [B][HW][Cr] over token chunks: part[b][chunk][g][2].
template <typename T>
__global__ void gn_partial_kernel(const T* __restrict__ U, int HW, int Cr, int groups, int chunks,
                                  float* __restrict__ part) {
  pdl_wait();
  const int b = blockIdx.y, chunk = blockIdx.x;
  const int cpg = Cr / groups;
  const int t0 = static_cast<int>((static_cast<long>(HW) * chunk) / chunks);
  const int t1 = static_cast<int>((static_cast<long>(HW) * (chunk + 1)) / chunks);
  __shared__ float red[32][2];
  for (int g = 0; g < groups; ++g) {
    float s1 = 0.f, s2 = 0.f;
    const long cnt = static_cast<long>(t1 - t0) * cpg;
    for (long e = threadIdx.x; e < cnt; e += blockDim.x) {
      const long t = t0 + e / cpg;
      const int c = g * cpg + static_cast<int>(e % cpg);
      const float v = to_f32(U[(static_cast<long>(b) * HW + t) * Cr + c]);
      s1 += v;
      s2 += v * v;
    }
    s1 = warp_sum(s1);
    s2 = warp_sum(s2);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
      red[w][0] = s1;
      red[w][1] = s2;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float a = 0.f, q = 0.f;
      for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) {
        a += red[i][0];
        q += red[i][1];
      }
      float* o = part + ((static_cast<long>(b) * chunks + chunk) * groups + g) * 2;
      o[0] = a;
      o[1] = q;
    }
    __syncthreads();
  }
}

// GroupNorm + LeakyReLU in one cooperative grid (bf16, channels per group >= 8,
// Cr % 8 == 0). Each block owns a contiguous token range of every image:
//  1. per-thread sums of 8-channel vectors (at most two groups per vector),
//     fixed-order block reduction -> part[b][block][group][2];
//  2. grid barrier: one arrival per block on a zeroed counter, then a bounded
//     spin until `expect` arrivals (gridDim.x in every forward call;
//     EDIT_ERR_TIMEOUT and wait site 30 after `limit_ns`, 2 s in a forward
//     call; the launch is cooperative, so every block is resident);
//  3. per image: every block combines all blocks' partials in the same fixed
//     order (one warp per group, fp64), forms the per-channel affine form
//     scale = gamma * rstd, shift = beta - mean * scale, and applies
//     G = LeakyReLU(scale * U + shift) to its tokens (U is re-read from L2).
// Block 0 also writes stats [b][group] = (mean, rstd) and ss [b][c] = (scale,
// shift). Dynamic shared memory: blockDim * 4 + Cr * 4 floats. At most
// GN_FUSED_MAXB blocks (part is [B][groups][2][nblk]).
constexpr int GN_FUSED_MAXB = 320;

__global__ void __launch_bounds__(512) gn_fused_bf16_kernel(const __nv_bfloat16* __restrict__ U, int B, long HW,
                                                            int Cr, int groups, float eps,
                                                            const __nv_bfloat16* __restrict__ gamma,
                                                            const __nv_bfloat16* __restrict__ beta, float slope,
                                                            float* __restrict__ part, unsigned int* arrive,
                                                            float* __restrict__ stats, float* __restrict__ ss,
                                                            __nv_bfloat16* __restrict__ G, int* status,
                                                            unsigned int expect, uint64_t limit_ns) {
  pdl_wait();
  extern __shared__ float gf_sm[];
  float* red = gf_sm;                      // [blockDim][4]
  float* aff = gf_sm + blockDim.x * 4;     // [Cr][2] scale, shift of the current image
  float* gb = aff + Cr * 2;                // [Cr][2] gamma, beta
  __shared__ int gf_abort;
  const int nblk = gridDim.x, blk = blockIdx.x;
  const int nvec = Cr / 8, kt_n = blockDim.x / nvec;
  const int t = threadIdx.x, v = t % nvec, kt = t / nvec;
  const bool active = kt < kt_n;
  const int cpg = Cr / groups, c0 = v * 8, g0 = c0 / cpg;
  const long chunk = (HW + nblk - 1) / nblk;
  const long t0 = blk * chunk, t1 = t0 + chunk < HW ? t0 + chunk : HW;
  for (int c = t; c < Cr; c += blockDim.x) {  // the affine weights, fetched while the statistics run
    gb[c * 2] = __bfloat162float(gamma[c]);
    gb[c * 2 + 1] = __bfloat162float(beta[c]);
  }
  // ---- 1. partial sums of this block's tokens, per image
  for (int b = 0; b < B; ++b) {
    float a0 = 0.f, q0 = 0.f, a1 = 0.f, q1 = 0.f;
    auto accum = [&](const uint4& raw) {
      const __nv_bfloat16* u = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float x = __bfloat162float(u[j]);
        if ((c0 + j) / cpg == g0) {
          a0 += x;
          q0 = fmaf(x, x, q0);
        } else {
          a1 += x;
          q1 = fmaf(x, x, q1);
        }
      }
    };
    if (active) {
      const __nv_bfloat16* ub = U + static_cast<long>(b) * HW * Cr + c0;
      long tok = t0 + kt;
      for (; tok + 3 * kt_n < t1; tok += 4 * kt_n) {  // four independent loads in flight
        uint4 r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) r[j] = *reinterpret_cast<const uint4*>(ub + (tok + j * kt_n) * Cr);
#pragma unroll
        for (int j = 0; j < 4; ++j) accum(r[j]);
      }
      for (; tok < t1; tok += kt_n) accum(*reinterpret_cast<const uint4*>(ub + tok * Cr));
    }
    red[t * 4 + 0] = a0;
    red[t * 4 + 1] = q0;
    red[t * 4 + 2] = a1;
    red[t * 4 + 3] = q1;
    __syncthreads();
    for (int g = t; g < groups; g += blockDim.x) {
      double s1 = 0.0, s2 = 0.0;
      const int vlo = (g * cpg) / 8, vhi = ((g + 1) * cpg - 1) / 8;
      for (int vv = vlo; vv <= vhi; ++vv) {
        const int slot = ((vv * 8) / cpg == g) ? 0 : 2;
        for (int k = 0; k < kt_n; ++k) {
          s1 += red[(k * nvec + vv) * 4 + slot];
          s2 += red[(k * nvec + vv) * 4 + slot + 1];
        }
      }
      float* o = part + (static_cast<long>(b) * groups + g) * 2 * nblk + blk;  // [b][g][sum | sumsq][block]
      o[0] = static_cast<float>(s1);
      o[nblk] = static_cast<float>(s2);
    }
    __syncthreads();
  }
  // ---- 2. grid barrier
  if (t == 0) {
    gf_abort = 0;
    __threadfence();
    atomicAdd(arrive, 1u);
    const uint64_t w0 = globaltimer_ns();
    unsigned int seen;
    while ((seen = *reinterpret_cast<volatile unsigned int*>(arrive)) < expect) {
      if (globaltimer_ns() - w0 > limit_ns) {
        record_status(status, EDIT_ERR_TIMEOUT);
        record_wait_site(status, 30, static_cast<int>(seen), static_cast<int>(expect), nblk, 0);
        gf_abort = 1;
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  if (gf_abort) return;
  // ---- 3. per image: combine, affine form, apply
  const int warp = t >> 5, lane = t & 31, nwarps = blockDim.x >> 5;
  const long cnt = HW * cpg;
  for (int b = 0; b < B; ++b) {
    for (int g = warp; g < groups; g += nwarps) {
      // lane l sums blocks l, l + 32, ... in that order (all loads issued first), then a fixed butterfly
      const float* ps = part + (static_cast<long>(b) * groups + g) * 2 * nblk;
      float r1[GN_FUSED_MAXB / 32], r2[GN_FUSED_MAXB / 32];
#pragma unroll
      for (int j = 0; j < GN_FUSED_MAXB / 32; ++j) {
        const int kk = lane + 32 * j;
        r1[j] = kk < nblk ? ps[kk] : 0.f;
        r2[j] = kk < nblk ? ps[nblk + kk] : 0.f;
      }
      double s1 = 0.0, s2 = 0.0;
#pragma unroll
      for (int j = 0; j < GN_FUSED_MAXB / 32; ++j) {
        s1 += r1[j];
        s2 += r2[j];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
        s2 += __shfl_xor_sync(0xffffffffu, s2, off);
      }
      const double mean = s1 / static_cast<double>(cnt);
      double var = s2 / static_cast<double>(cnt) - mean * mean;
      if (var < 0.0) var = 0.0;
      const double rstd = 1.0 / sqrt(var + static_cast<double>(eps));
      for (int c = g * cpg + lane; c < (g + 1) * cpg; c += 32) {
        const double sc = static_cast<double>(gb[c * 2]) * rstd;
        const double sh = static_cast<double>(gb[c * 2 + 1]) - mean * sc;
        aff[c * 2] = static_cast<float>(sc);
        aff[c * 2 + 1] = static_cast<float>(sh);
        if (blk == 0) {
          ss[(static_cast<long>(b) * Cr + c) * 2] = static_cast<float>(sc);
          ss[(static_cast<long>(b) * Cr + c) * 2 + 1] = static_cast<float>(sh);
        }
      }
      if (blk == 0 && lane == 0) {
        stats[(b * groups + g) * 2] = static_cast<float>(mean);
        stats[(b * groups + g) * 2 + 1] = static_cast<float>(rstd);
      }
    }
    __syncthreads();
    if (active) {
      float sc[8], sh[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sc[j] = aff[(c0 + j) * 2];
        sh[j] = aff[(c0 + j) * 2 + 1];
      }
      auto apply = [&](const uint4& raw) {
        const __nv_bfloat16* u = reinterpret_cast<const __nv_bfloat16*>(&raw);
        float o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float y = fmaf(__bfloat162float(u[j]), sc[j], sh[j]);
          o[j] = y >= 0.f ? y : y * slope;
        }
        uint4 out;
        out.x = pack_bf16x2(o[0], o[1]);
        out.y = pack_bf16x2(o[2], o[3]);
        out.z = pack_bf16x2(o[4], o[5]);
        out.w = pack_bf16x2(o[6], o[7]);
        return out;
      };
      const long base = static_cast<long>(b) * HW * Cr + c0;
      long tok = t0 + kt;
      for (; tok + 3 * kt_n < t1; tok += 4 * kt_n) {  // four independent loads in flight
        uint4 r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) r[j] = *reinterpret_cast<const uint4*>(U + base + (tok + j * kt_n) * Cr);
#pragma unroll
        for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(G + base + (tok + j * kt_n) * Cr) = apply(r[j]);
      }
      for (; tok < t1; tok += kt_n)
        *reinterpret_cast<uint4*>(G + base + tok * Cr) = apply(*reinterpret_cast<const uint4*>(U + base + tok * Cr));
    }
    __syncthreads();
  }
}

// Fixed-order (deterministic) combine of the partials in fp64, then the
// per-channel affine form of GN: scale = gamma * rstd, shift = beta - mean * scale.
// part: [B][P][groups][2]; stats out: [B][groups][2] (mean, rstd);
// ss out: [B][Cr][2] (scale, shift). A block of up to 256 threads handles one
// (group, image): thread t sums partials t, t+blockDim, ... in order, then a
// fixed shared-memory tree (blockDim a power of two).
template <typename T>
__device__ void gn_finalize_body(const float* __restrict__ part, int P, int cols, int groups, int Cr, long count,
                                 float eps, const T* __restrict__ gamma, const T* __restrict__ beta,
                                 float* __restrict__ stats, float* __restrict__ ss, int g, int b, double* r1,
                                 double* r2) {
  const int cpg = Cr / groups;
  const int nt = blockDim.x;  // a power of two, at most the length of r1 / r2
  double s1 = 0.0, s2 = 0.0;
  // element e = (partial i, column j) of group g, e = i * cols + j: thread t
  // sums e = t, t + nt, ... in that order
  const int n = P * cols;
#pragma unroll 8
  for (int e = threadIdx.x; e < n; e += nt) {
    const int i = e / cols, j = e - i * cols;
    const float2 q = *reinterpret_cast<const float2*>(part + (((static_cast<long>(b) * P + i) * groups + g) * cols + j) * 2);
    s1 += q.x;
    s2 += q.y;
  }
  __syncthreads();
  r1[threadIdx.x] = s1;
  r2[threadIdx.x] = s2;
  __syncthreads();
  for (int w = nt / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      r1[threadIdx.x] += r1[threadIdx.x + w];
      r2[threadIdx.x] += r2[threadIdx.x + w];
    }
    __syncthreads();
  }
  const double mean = r1[0] / static_cast<double>(count);
  double var = r2[0] / static_cast<double>(count) - mean * mean;
  if (var < 0.0) var = 0.0;
  const double rstd = 1.0 / sqrt(var + static_cast<double>(eps));
  if (threadIdx.x == 0) {
    stats[(b * groups + g) * 2] = static_cast<float>(mean);
    stats[(b * groups + g) * 2 + 1] = static_cast<float>(rstd);
  }
  for (int c = g * cpg + threadIdx.x; c < (g + 1) * cpg; c += blockDim.x) {
    const double sc = static_cast<double>(to_f32(gamma[c])) * rstd;
    ss[(static_cast<long>(b) * Cr + c) * 2] = static_cast<float>(sc);
    ss[(static_cast<long>(b) * Cr + c) * 2 + 1] = static_cast<float>(static_cast<double>(to_f32(beta[c])) - mean * sc);
  }
  __syncthreads();
}

// Block (g, b): group g of image b from part [b][P][groups][cols][2] (sum,
// sum of squares), summed in a fixed order in fp64: cols = 1 for the token-chunk
// partials of gn_partial_kernel, cols = Cr / groups for the column sums the
// conv writes per 32-row slot of each tile.
template <typename T>
__global__ void __launch_bounds__(1024) gn_finalize_kernel(const float* __restrict__ part, int P, int cols, int groups,
                                                          int Cr, long count, float eps, const T* __restrict__ gamma,
                                                          const T* __restrict__ beta, float* __restrict__ stats,
                                                          float* __restrict__ ss) {
  pdl_wait();
  __shared__ double r1[1024], r2[1024];
  gn_finalize_body<T>(part, P, cols, groups, Cr, count, eps, gamma, beta, stats, ss, blockIdx.x, blockIdx.y, r1, r2);
}

// G = LeakyReLU(scale * U + shift), elementwise over [B][HW][Cr].
template <typename T>
__global__ void gn_apply_leaky_kernel(const T* __restrict__ U, const float* __restrict__ ss, long HW, int Cr,
                                      float slope, T* __restrict__ G, long total) {
  pdl_wait();
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % Cr);
    const long b = i / (HW * Cr);
    const float sc = ss[(b * Cr + c) * 2], sh = ss[(b * Cr + c) * 2 + 1];
    float v = fmaf(to_f32(U[i]), sc, sh);
    v = v >= 0.f ? v : v * slope;
    G[i] = from_f32<T>(v);
  }
}

// bf16 variant, 8 channels per thread with 16-byte loads/stores (Cr % 8 == 0),
// image blockIdx.y. Thread t always handles channel vector t % (Cr/8) (blockDim
// a multiple of Cr/8), so its scale/shift stay in registers; it visits tokens
// blockDim/(Cr/8) * gridDim.x apart, four loads in flight.
__global__ void gn_apply_leaky_bf16x8(const __nv_bfloat16* __restrict__ U, const float* __restrict__ ss, long HW,
                                      int Cr, float slope, __nv_bfloat16* __restrict__ G) {
  pdl_wait();
  const int nvec = Cr / 8;
  const int per_block = blockDim.x / nvec;
  const int v = threadIdx.x % nvec, kt = threadIdx.x / nvec;
  if (kt >= per_block) return;
  const int c = v * 8;
  const long b = blockIdx.y;
  float sc[8], sh[8];
  {
    const float4* s4 = reinterpret_cast<const float4*>(ss + (b * Cr + c) * 2);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 q = s4[j];
      sc[2 * j] = q.x;
      sh[2 * j] = q.y;
      sc[2 * j + 1] = q.z;
      sh[2 * j + 1] = q.w;
    }
  }
  auto apply = [&](const uint4& raw) {
    const __nv_bfloat16* u = reinterpret_cast<const __nv_bfloat16*>(&raw);
    float o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float y = fmaf(__bfloat162float(u[j]), sc[j], sh[j]);
      o[j] = y >= 0.f ? y : y * slope;
    }
    uint4 out;
    out.x = pack_bf16x2(o[0], o[1]);
    out.y = pack_bf16x2(o[2], o[3]);
    out.z = pack_bf16x2(o[4], o[5]);
    out.w = pack_bf16x2(o[6], o[7]);
    return out;
  };
  const __nv_bfloat16* ub = U + b * HW * Cr + c;
  __nv_bfloat16* gb = G + b * HW * Cr + c;
  const long step = static_cast<long>(gridDim.x) * per_block;
  long tok = static_cast<long>(blockIdx.x) * per_block + kt;
  for (; tok + 3 * step < HW; tok += 4 * step) {
    uint4 r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) r[j] = *reinterpret_cast<const uint4*>(ub + (tok + j * step) * Cr);
#pragma unroll
    for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(gb + (tok + j * step) * Cr) = apply(r[j]);
  }
  for (; tok < HW; tok += step) *reinterpret_cast<uint4*>(gb + tok * Cr) = apply(*reinterpret_cast<const uint4*>(ub + tok * Cr));
}

// ============================================================ weight folding
// The 1x1 conv feeds only Linear_Q, so Linear_Q(X + G W1^T + b1) =
// X Wq^T + G (Wq W1)^T + (Wq b1 + bq). dst[c][r] = sum_k Wq[c][k] W1[k][r]
// is formed on the tensor cores from W1 transposed; this kernel transposes
// W1 [C][Cr] -> W1t [Cr][C] and forms the folded bias (fp32).
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ src, int rows, int cols, T* __restrict__ dst) {
  pdl_wait();
  __shared__ T tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = src[static_cast<long>(r) * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) dst[static_cast<long>(c) * rows + r] = tile[threadIdx.x][i];
  }
}

// bq' = Wq b1 + bq, one warp per output row (fp32).
template <typename T>
__device__ __forceinline__ void fold_bias_rows(const T* __restrict__ wq, const T* __restrict__ bq,
                                               const T* __restrict__ b1, int C, float* __restrict__ out, int blk) {
  const int row = blk * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= C) return;
  float s = 0.f;
  if (sizeof(T) == 2 && (C & 7) == 0) {  // 8 elements per 16-byte load
    for (int k = lane * 8; k < C; k += 256) {
      const uint4 wv = *reinterpret_cast<const uint4*>(wq + static_cast<long>(row) * C + k);
      const uint4 bv = *reinterpret_cast<const uint4*>(b1 + k);
      const T* w8 = reinterpret_cast<const T*>(&wv);
      const T* b8 = reinterpret_cast<const T*>(&bv);
#pragma unroll
      for (int j = 0; j < 8; ++j) s = fmaf(to_f32(w8[j]), to_f32(b8[j]), s);
    }
  } else {
    for (int k = lane; k < C; k += 32) s = fmaf(to_f32(wq[static_cast<long>(row) * C + k]), to_f32(b1[k]), s);
  }
  s = warp_sum(s);
  if (lane == 0) out[row] = s + to_f32(bq[row]);
}

template <typename T>
__global__ void fold_bias_kernel(const T* __restrict__ wq, const T* __restrict__ bq, const T* __restrict__ b1,
                                 int C, float* __restrict__ out) {
  pdl_wait();
  fold_bias_rows(wq, bq, b1, C, out, blockIdx.x);
}

// The two inputs of the weight folding in one launch of 256-thread blocks:
// blocks [0, tiles_r * tiles_c) transpose W1 [C][Cr] -> W1t [Cr][C] in 32 x 32
// tiles, the following ceil(C / 8) blocks form bq' = Wq b1 + bq (fp32).
template <typename T>
__global__ void __launch_bounds__(256) fold_prep_kernel(const T* __restrict__ w1, int C, int Cr, T* __restrict__ w1t,
                                                        const T* __restrict__ wq, const T* __restrict__ bq,
                                                        const T* __restrict__ b1, float* __restrict__ bout) {
  pdl_wait();
  __shared__ T tile[32][33];
  const int tiles_c = (Cr + 31) / 32, ntr = tiles_c * ((C + 31) / 32);
  if (static_cast<int>(blockIdx.x) >= ntr) {
    fold_bias_rows(wq, bq, b1, C, bout, blockIdx.x - ntr);
    return;
  }
  const int c0 = (blockIdx.x % tiles_c) * 32, r0 = (blockIdx.x / tiles_c) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + tx;
    if (r < C && c < Cr) tile[i][tx] = w1[static_cast<long>(r) * Cr + c];
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + tx;
    if (r < C && c < Cr) w1t[static_cast<long>(c) * C + r] = tile[tx][i];
  }
}

// ====================================================== depthwise stride-2
// KVp [B][H][W][2C] (Linear_K | Linear_V) -> K = ReLU(DW_K), V = DW_V, each
// [B][Ho][Wo][C]; tap (a, e) of output (i, j) reads input (2i+a-1, 2j+e-1).
template <typename T, int VEC>
__global__ void dwconv_s2_kernel(const T* __restrict__ kvp, int B, int H, int W, int C,
                                 const T* __restrict__ kw, const T* __restrict__ kb, const T* __restrict__ vw,
                                 const T* __restrict__ vb, T* __restrict__ K, T* __restrict__ V) {
  pdl_wait();
  const int Ho = (H + 1) / 2, Wo = (W + 1) / 2;
  const int C2v = 2 * C / VEC;
  const long total = static_cast<long>(B) * Ho * Wo * C2v;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int cv = static_cast<int>(idx % C2v);
    long pix = idx / C2v;
    const int j = static_cast<int>(pix % Wo);
    pix /= Wo;
    const int i = static_cast<int>(pix % Ho);
    const int b = static_cast<int>(pix / Ho);
    const int ch = cv * VEC;  // channel in [0, 2C)
    const bool isk = ch < C;
    const int c = isk ? ch : ch - C;
    const T* wt = isk ? kw : vw;
    const T* bs = isk ? kb : vb;
    float acc[VEC];
#pragma unroll
    for (int u = 0; u < VEC; ++u) acc[u] = to_f32(bs[c + u]);
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const int hh = 2 * i + a - 1;
      if (hh < 0 || hh >= H) continue;
#pragma unroll
      for (int e = 0; e < 3; ++e) {
        const int ww = 2 * j + e - 1;
        if (ww < 0 || ww >= W) continue;
        const T* src = kvp + ((static_cast<long>(b) * H + hh) * W + ww) * (2L * C) + ch;
        T vals[VEC];
        if (VEC == 8 && sizeof(T) == 2) {
          *reinterpret_cast<uint4*>(vals) = *reinterpret_cast<const uint4*>(src);
        } else {
#pragma unroll
          for (int u = 0; u < VEC; ++u) vals[u] = src[u];
        }
#pragma unroll
        for (int u = 0; u < VEC; ++u) acc[u] = fmaf(to_f32(wt[(c + u) * 9 + a * 3 + e]), to_f32(vals[u]), acc[u]);
      }
    }
    T* dst = (isk ? K : V) + ((static_cast<long>(b) * Ho + i) * Wo + j) * C + c;
    T outv[VEC];
#pragma unroll
    for (int u = 0; u < VEC; ++u) outv[u] = from_f32<T>(isk ? fmaxf(acc[u], 0.f) : acc[u]);
    if (VEC == 8 && sizeof(T) == 2) {
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(outv);
    } else {
#pragma unroll
      for (int u = 0; u < VEC; ++u) dst[u] = outv[u];
    }
  }
}

// TMA version of the channel-major depthwise conv (same outputs as
// dwconv_s2_t_kernel): the 3 x 65-pixel, 64-channel input patch arrives in one
// tensor load (zero-filled outside the grid). Thread (tg, c) computes the 8
// consecutive output tokens 8*tg .. 8*tg+7 of channel c (51 patch reads for
// 72 taps) and writes them as one 16-byte chunk of the channel-major block,
// placed with the 64-byte swizzle (chunk j of row r at j ^ ((r >> 1) & 3)) so
// the 16-byte writes of a warp hit distinct banks; the tensor stores undo the
// swizzle. KT leaves as one 64-row x 32-token block, VTx as eight 8-row
// blocks (a head boundary never splits one since d % 8 == 0), and the
// token-major copies (MM-EDiT) as one 32-token x 64-channel block clipped at
// the end of the output row. The load wait is bounded (status on timeout).
struct DwTmaMaps {
  CUtensorMap in;    // KVp as [B][H][W][2C], box 64 x 65 x 3 x 1, no swizzle
  CUtensorMap kt;    // KT as [B*C][Mp], box 32 x 64, 64-byte swizzle
  CUtensorMap vtx;   // VTx as [B*heads][NP][Mp], box 32 x 8 x 1, 64-byte swizzle
  CUtensorMap ktok;  // K as [B][Ho][Wo][C], box 64 x 32 x 1 x 1, no swizzle (MM only)
  CUtensorMap vtok;  // V likewise
};

__global__ void __launch_bounds__(256) dwconv_s2_tma_kernel(const __grid_constant__ DwTmaMaps m, int H, int W, int C,
                                                            int d, int heads, int Wop,
                                                            const __nv_bfloat16* __restrict__ kw,
                                                            const __nv_bfloat16* __restrict__ kb,
                                                            const __nv_bfloat16* __restrict__ vw,
                                                            const __nv_bfloat16* __restrict__ vb, int tokmajor,
                                                            int row_shift, int* status) {
  pdl_wait();
  constexpr int JT = 32, CB = 64, PW = 2 * JT + 1;
  __shared__ __align__(1024) __nv_bfloat16 out_s[CB * JT];  // [channel][token], 64-byte swizzled rows
  __shared__ __align__(128) __nv_bfloat16 in_s[3][PW][CB];
  // [token][channel] copy for the token-major stores (MM-EDiT only): dynamic
  // shared memory, so the EDiT layer's blocks do without it (7 per SM, not 6)
  extern __shared__ __align__(128) __nv_bfloat16 dw_tok[];
  __nv_bfloat16(*tok_s)[CB] = reinterpret_cast<__nv_bfloat16(*)[CB]>(dw_tok);
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const int Wo = (W + 1) / 2;
  // grid (column tiles, image x channel blocks, output rows): rows vary slowest and
  // run bottom-up, so the rows the K|V GEMM wrote last (still in L2) are read first
  const int j0 = blockIdx.x * JT, i = gridDim.z - 1 - blockIdx.z;
  const int nblk = 2 * C / CB;
  const int b = blockIdx.y / nblk, cb = blockIdx.y - b * nblk;
  const int gc0 = cb * CB;
  const bool isk = gc0 < C;
  const int ch0 = isk ? gc0 : gc0 - C;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&m.in);
    mbar_arrive_expect_tx(&bar, 3 * PW * CB * 2);
    tma_load_4d(&m.in, &bar, &in_s[0][0][0], gc0, 2 * j0 - 1, 2 * i - 1 + row_shift, b);
  }
  const int c = threadIdx.x & (CB - 1);
  const int tg = threadIdx.x >> 6;  // tokens 8*tg .. 8*tg + 7
  const __nv_bfloat16* wt = isk ? kw : vw;
  float wr[9];
#pragma unroll
  for (int q = 0; q < 9; ++q) wr[q] = __bfloat162float(wt[(ch0 + c) * 9 + q]);
  const float bias = __bfloat162float((isk ? kb : vb)[ch0 + c]);
  const bool ok = mbar_wait(&bar, 0, &abort_flag, status);
  if (ok) {
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = bias;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
#pragma unroll
      for (int col = 0; col < 17; ++col) {  // patch columns 16*tg + col
        const float x = __bfloat162float(in_s[a][16 * tg + col][c]);
#pragma unroll
        for (int e = 0; e < 3; ++e) {
          const int t2 = col - e;  // output 2t + e == col
          if (t2 >= 0 && (t2 & 1) == 0 && t2 / 2 < 8) acc[t2 / 2] = fmaf(wr[a * 3 + e], x, acc[t2 / 2]);
        }
      }
    }
    float o[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      float v = isk ? fmaxf(acc[t], 0.f) : acc[t];
      o[t] = (j0 + 8 * tg + t >= Wo) ? 0.f : v;
    }
    uint4 pk;
    pk.x = pack_bf16x2(o[0], o[1]);
    pk.y = pack_bf16x2(o[2], o[3]);
    pk.z = pack_bf16x2(o[4], o[5]);
    pk.w = pack_bf16x2(o[6], o[7]);
    // row c (64 bytes = 4 chunks), chunk tg, 64-byte swizzle
    *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out_s) + c * 64 + 16 * (tg ^ ((c >> 1) & 3))) = pk;
    if (tokmajor) {
      const __nv_bfloat16* ob = reinterpret_cast<const __nv_bfloat16*>(&pk);
#pragma unroll
      for (int t = 0; t < 8; ++t) tok_s[8 * tg + t][c] = ob[t];
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0 && ok) {
    const int t0 = i * Wop + j0;
    if (isk) {
      tma_store_2d(&m.kt, out_s, t0, b * C + ch0);
    } else {
#pragma unroll 1
      for (int g = 0; g < CB / 8; ++g) {
        const int ch = ch0 + 8 * g;
        const int h = ch / d, rr = ch - h * d;
        tma_store_3d(&m.vtx, out_s + 8 * g * JT, t0, rr, b * heads + h);
      }
    }
    if (tokmajor && j0 < Wo) tma_store_4d(isk ? &m.ktok : &m.vtok, &tok_s[0][0], ch0, j0, i, b);
    bulk_commit();
    bulk_wait_read<0>();  // shared memory may be released once the stores have read it
  }
}


// Keys and values without the Spatial Compressor (ablation variants whose
// keys and values keep all N tokens): the token-major rows kvp [B][N][2C]
// (first C channels the key, already the Linear output or ReLU'd, the rest
// the value) become the channel-major operands of the tensor-core KV state,
// KT [B*C][Mp] = ReLU(key) and rows 0..d-1 of each head block of VTx
// [B*heads][NP][Mp] = value; tokens N..Mp-1 are written as zeros (Mp % 8 == 0,
// C % 64 == 0). One block moves 64 tokens x 64 channels through shared
// memory: 16-byte loads along the channels, 16-byte stores along the tokens
// (lane pairs write the two halves of one 32-byte sector).
__global__ void __launch_bounds__(256) kv_transpose_kernel(const __nv_bfloat16* __restrict__ kvp, long N, int C,
                                                           int d, int heads, int NP, long Mp,
                                                           __nv_bfloat16* __restrict__ KT,
                                                           __nv_bfloat16* __restrict__ VTx) {
  pdl_wait();
  __shared__ __align__(16) __nv_bfloat16 tile[64][72];  // [token][channel], rows padded to 144 bytes
  const long t0 = static_cast<long>(blockIdx.x) * 64;
  const int nblk = 2 * C / 64;
  const int b = blockIdx.y / nblk, gc0 = (blockIdx.y - b * nblk) * 64;
  for (int e = threadIdx.x; e < 64 * 8; e += 256) {
    const int tt = e >> 3, v = e & 7;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (t0 + tt < N) val = *reinterpret_cast<const uint4*>(kvp + (static_cast<long>(b) * N + t0 + tt) * (2L * C) + gc0 + 8 * v);
    *reinterpret_cast<uint4*>(&tile[tt][8 * v]) = val;
  }
  __syncthreads();
  const bool isk = gc0 < C;
  for (int e = threadIdx.x; e < 64 * 8; e += 256) {
    const int c = (e >> 1) & 63, v = 2 * (e >> 7) + (e & 1);
    const long n0 = t0 + 8 * v;
    if (n0 >= Mp) continue;
    float o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float x = __bfloat162float(tile[8 * v + j][c]);
      o[j] = isk ? fmaxf(x, 0.f) : x;
    }
    uint4 pk;
    pk.x = pack_bf16x2(o[0], o[1]);
    pk.y = pack_bf16x2(o[2], o[3]);
    pk.z = pack_bf16x2(o[4], o[5]);
    pk.w = pack_bf16x2(o[6], o[7]);
    __nv_bfloat16* dst;
    if (isk) {
      dst = KT + (static_cast<long>(b) * C + gc0 + c) * Mp + n0;
    } else {
      const int ch = gc0 - C + c, h = ch / d, r = ch - h * d;
      dst = VTx + ((static_cast<long>(b) * heads + h) * NP + r) * Mp + n0;
    }
    *reinterpret_cast<uint4*>(dst) = pk;
  }
}

// U of the conv tiles that ran split over k: bias + the ksplit fp32 partials
// of each tile, summed in part order (deterministic), bf16 out. Pair tiles
// [pt_first, pt_first + pt_count) are split; part is [(local pair tile * ksplit
// + k) * 2 + rank][Cr / 4][128][4], and row r of CTA tile m_tile = 2 * pair tile
// + rank is pixel (h0 + r / TW, w0 + r % TW) of a TH x TW tile (TH * TW = 128).
// A block (256 threads, Cr / 4 a multiple of 8) takes 32 rows x 8 column quads
// of one tile: warp w sums quad w of the 32 rows (lane = row, so each part is
// read as 512 contiguous bytes), the results meet in shared memory, and the
// block writes U as 64 contiguous bytes per row. When gn_col is set, each warp
// also writes its quad's GroupNorm column sums of the 32 rows (bf16 values;
// pixels outside the image add nothing), in the layout the conv epilogue
// writes for the tiles it finishes itself.
__global__ void __launch_bounds__(256) conv_parts_fixup_kernel(const float* __restrict__ part, int ksplit,
                                                               int pt_first, int pt_count, int tiles_w, int tiles_h,
                                                               int TH, int TW, int H, int W, int Cr,
                                                               const __nv_bfloat16* __restrict__ bias,
                                                               int num_m_tiles, __nv_bfloat16* __restrict__ U,
                                                               float* __restrict__ gn_col) {
  pdl_wait();
  __shared__ uint2 tile[32][9];  // [row][quad] of the block's results (padded: fewer bank conflicts)
  const int cv = Cr / 4, ngroups = cv / 8;
  const long nblocks = static_cast<long>(pt_count) * 2 * 4 * ngroups;  // (tile, row group, quad group)
  const int per_img = tiles_h * tiles_w;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (long blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {  // uniform across the block
    const int qg = static_cast<int>(blk % ngroups);
    const int rg = static_cast<int>((blk / ngroups) & 3);
    const int rank = static_cast<int>((blk / ngroups / 4) & 1);
    const int pt = static_cast<int>(blk / ngroups / 8);
    const int m_tile = 2 * (pt_first + pt) + rank;
    if (m_tile >= num_m_tiles) continue;  // the pair grid's empty tile (whole block)
    const int img = m_tile / per_img, u = m_tile - img * per_img;
    const int h0 = (u / tiles_w) * TH, w0 = (u % tiles_w) * TW;
    // ---- warp w: quad qg * 8 + w of rows 32 rg + lane
    {
      const int row = rg * 32 + lane, c4 = qg * 8 + w, c = c4 * 4;
      const bool inside = h0 + row / TW < H && w0 + row % TW < W;
      float4 a = make_float4(__bfloat162float(bias[c]), __bfloat162float(bias[c + 1]), __bfloat162float(bias[c + 2]),
                             __bfloat162float(bias[c + 3]));
      for (int k = 0; k < ksplit; ++k) {
        const float4 q = *reinterpret_cast<const float4*>(
            part + ((((static_cast<long>(pt) * ksplit + k) * 2 + rank) * cv + c4) * 128 + row) * 4);
        a.x += q.x;
        a.y += q.y;
        a.z += q.z;
        a.w += q.w;
      }
      const uint2 o = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
      tile[lane][w] = o;
      if (gn_col != nullptr) {
        float v[4] = {__uint_as_float(o.x << 16), __uint_as_float(o.x & 0xffff0000u), __uint_as_float(o.y << 16),
                      __uint_as_float(o.y & 0xffff0000u)};
        float r[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          r[2 * j] = inside ? v[j] : 0.f;
          r[2 * j + 1] = inside ? v[j] * v[j] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) r[j] = warp_sum(r[j]);
        if (lane == 0) {
          float* dst = gn_col + ((static_cast<long>(img) * per_img * 4 + u * 4 + rg) * Cr + c) * 2;
          *reinterpret_cast<float4*>(dst) = make_float4(r[0], r[1], r[2], r[3]);
          *reinterpret_cast<float4*>(dst + 4) = make_float4(r[4], r[5], r[6], r[7]);
        }
      }
    }
    __syncthreads();
    // ---- thread t: quad t % 8 of row t / 8: eight threads write one row's 64 bytes
    {
      const int row = rg * 32 + (threadIdx.x >> 3), q = threadIdx.x & 7;
      const int hh = h0 + row / TW, ww = w0 + row % TW;
      if (hh < H && ww < W)
        *reinterpret_cast<uint2*>(U + ((static_cast<long>(img) * H + hh) * W + ww) * Cr + (qg * 8 + q) * 4) =
            tile[threadIdx.x >> 3][q];
    }
    __syncthreads();
  }
}

// ================================================================ KV state
// Partial [S_h | z_h] over a chunk of compressed tokens:
// part[b][h][chunk][a][c], a < d, c <= d, with column d = sum_j K_ja.
// Thread block: ceil(d/4)^2 threads (padded to a warp multiple), each owning a
// 4 x 4 block of S; tokens staged through shared memory 32 at a time.
template <typename T>
__global__ void kv_state_partial_kernel(const T* __restrict__ K, const T* __restrict__ V, int M, int C, int heads,
                                        int chunks, float* __restrict__ part) {
  pdl_wait();
  const int d = C / heads;
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = static_cast<int>((static_cast<long>(M) * chunk) / chunks);
  const int t1 = static_cast<int>((static_cast<long>(M) * (chunk + 1)) / chunks);
  extern __shared__ float kv_sm[];
  constexpr int TT = 32;
  float* Ks = kv_sm;            // [TT][d]
  float* Vs = kv_sm + TT * d;   // [TT][d]
  const int nb = (d + 3) / 4;
  const int tid = threadIdx.x;
  const int ba = tid / nb, bc = tid % nb;
  const bool owner = ba < nb;
  float acc[4][4] = {};
  float zacc = 0.f;  // threads tid < d accumulate z[tid]
  for (int tb = t0; tb < t1; tb += TT) {
    const int cnt = min(TT, t1 - tb);
    for (int e = tid; e < TT * d; e += blockDim.x) {
      const int t = e / d, c = e - t * d;
      float kv = 0.f, vv = 0.f;
      if (t < cnt) {
        const long off = (static_cast<long>(b) * M + tb + t) * C + h * d + c;
        kv = to_f32(K[off]);
        vv = to_f32(V[off]);
      }
      Ks[e] = kv;
      Vs[e] = vv;
    }
    __syncthreads();
    if (owner) {
      for (int t = 0; t < cnt; ++t) {
        float ka[4], vc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int a = ba * 4 + u, c = bc * 4 + u;
          ka[u] = a < d ? Ks[t * d + a] : 0.f;
          vc[u] = c < d ? Vs[t * d + c] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(ka[u], vc[v], acc[u][v]);
      }
    }
    if (tid < d)
      for (int t = 0; t < cnt; ++t) zacc += Ks[t * d + tid];
    __syncthreads();
  }
  float* o = part + ((static_cast<long>(b) * heads + h) * chunks + chunk) * d * (d + 1);
  if (owner) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int a = ba * 4 + u, c = bc * 4 + v;
        if (a < d && c < d) o[a * (d + 1) + c] = acc[u][v];
      }
  }
  if (tid < d) o[tid * (d + 1) + d] = zacc;
}

// Fixed-order sum of the chunk partials: Sz[b][h][a][c] (fp32).
__global__ void kv_state_combine_kernel(const float* __restrict__ part, int chunks, int per_head, long total,
                                        float* __restrict__ Sz) {
  pdl_wait();
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const long bh = i / per_head;
    const int e = static_cast<int>(i - bh * per_head);
    const float* q = part + bh * chunks * per_head + e;
    float s = 0.f;
    for (int k = 0; k < chunks; ++k) s += q[static_cast<long>(k) * per_head];
    Sz[i] = s;
  }
}

// Same fixed-order combine, also writing [S_h | z_h] as the bf16 B operand of
// the tensor-core apply: one thread per element of SzT [BH][NP][KP] (total
// elements); SzT[(b*heads + h)*NP + c][a] = Sz[b][h][a][c], summed over the
// chunks in order (and stored to Sz fp32 [BH][d][d+1]), for c <= d, a < d;
// every other element is zero padding.
__global__ void kv_state_combine_pack_kernel(const float* __restrict__ part, int chunks, int d, int NP, int KP,
                                             long total, float* __restrict__ Sz, __nv_bfloat16* __restrict__ SzT) {
  pdl_wait();
  const int per_head = d * (d + 1);
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const int a = static_cast<int>(i % KP);
    const long r = i / KP;
    const int c = static_cast<int>(r % NP);
    const long bh = r / NP;
    float s = 0.f;
    if (c <= d && a < d) {
      const int e = a * (d + 1) + c;
      const float* q = part + bh * chunks * per_head + e;
      for (int k = 0; k < chunks; ++k) s += q[static_cast<long>(k) * per_head];
      Sz[bh * per_head + e] = s;
    }
    SzT[i] = __float2bfloat16_rn(s);
  }
}

// ==================================================================== apply
// y_ih = (Q_ih S_h) / (Q_ih . z_h + eps) on CUDA cores (fp32 path).
// One block per (token block, head, batch); [S_h | z_h] staged in shared memory.
template <typename T>
__global__ void apply_simt_kernel(const T* __restrict__ Q, const float* __restrict__ Sz, int N, int C, int heads,
                                  float eps, T* __restrict__ out, float* __restrict__ den_out) {
  pdl_wait();
  const int d = C / heads;
  const int h = blockIdx.y, b = blockIdx.z;
  extern __shared__ float ap_sm[];  // [d][d+1]
  const float* src = Sz + (static_cast<long>(b) * heads + h) * d * (d + 1);
  for (int e = threadIdx.x; e < d * (d + 1); e += blockDim.x) ap_sm[e] = src[e];
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const T* q = Q + (static_cast<long>(b) * N + n) * C + h * d;
  T* o = out + (static_cast<long>(b) * N + n) * C + h * d;
  float den = 0.f;
  for (int a = 0; a < d; ++a) den = fmaf(to_f32(q[a]), ap_sm[a * (d + 1) + d], den);
  const float inv = 1.f / (den + eps);
  if (den_out) den_out[(static_cast<long>(b) * N + n) * heads + h] = den + eps;  // [b][n][head]
  for (int c = 0; c < d; ++c) {
    float s = 0.f;
    for (int a = 0; a < d; ++a) s = fmaf(to_f32(q[a]), ap_sm[a * (d + 1) + c], s);
    o[c] = from_f32<T>(s * inv);
  }
}

// ============================================================ MM-EDiT SDPA
// out[b, i, head] = w0 * out[b, i, head] (or 0 when `blend_in` is 0)
//                 + w1 * softmax(q k1^T / sqrt(d)) v1 + w2 * softmax(q k2^T / sqrt(d)) v2
// with each softmax over its own key set (k2 absent when n2 == 0). One thread
// per (query, head); keys staged through shared memory; online softmax with
// exp2f. q: [B][Nq][ldq]; k*, v*: [B][n*][ld*] (head h at columns h*d).

// Accumulates w * softmax(q K^T) V over one key set into res (registers).
// q rows live in shared memory (qs, stride D + 1), one row per thread.
template <typename T, int D>
__device__ __forceinline__ void sdpa_one_set(const T* kb, const T* vb, long ld, int nk, const float* qrow,
                                             bool active, float w, float (&res)[D], float* ks, float* vs, int h,
                                             float* lz = nullptr) {
  constexpr int KT = 64;
  float m = -INFINITY, l = 0.f;
  float acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) acc[c] = 0.f;
  for (int j0 = 0; j0 < nk; j0 += KT) {
    const int cnt = min(KT, nk - j0);
    __syncthreads();
    for (int e = threadIdx.x; e < KT * D; e += blockDim.x) {
      const int j = e / D, c = e - j * D;
      float kv = 0.f, vv = 0.f;
      if (j < cnt) {
        kv = to_f32(kb[(j0 + j) * ld + h * D + c]);
        vv = to_f32(vb[(j0 + j) * ld + h * D + c]);
      }
      ks[e] = kv;
      vs[e] = vv;
    }
    __syncthreads();
    if (active) {
      for (int j = 0; j < cnt; ++j) {
        float s = 0.f;
#pragma unroll 16
        for (int c = 0; c < D; ++c) s = fmaf(qrow[c], ks[j * D + c], s);
        const float mn = fmaxf(m, s);
        const float corr = exp2f(m - mn);
        const float pj = exp2f(s - mn);
        l = l * corr + pj;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = fmaf(pj, vs[j * D + c], acc[c] * corr);
        m = mn;
      }
    }
  }
  const float sc = l > 0.f ? w / l : 0.f;
#pragma unroll
  for (int c = 0; c < D; ++c) res[c] = fmaf(acc[c], sc, res[c]);
  if (lz) *lz = m + log2f(l);  // log2 of the set's normaliser sum_j exp(q.k_j / sqrt(d))
}

template <typename T, int D>
__global__ void __launch_bounds__(128) sdpa_blend_kernel(SdpaParams p) {
  pdl_wait();
  extern __shared__ float sd_sm[];
  float* ks = sd_sm;                 // [64][D]
  float* vs = sd_sm + 64 * D;        // [64][D]
  float* qs = sd_sm + 128 * D;       // [blockDim][D + 1]
  const int h = blockIdx.y, b = blockIdx.z;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const bool active = i < p.Nq;
  const float qscale = rsqrtf(static_cast<float>(D)) * 1.4426950408889634f;  // 1/sqrt(d) * log2(e)
  float* qrow = qs + threadIdx.x * (D + 1);
  const T* qp = reinterpret_cast<const T*>(p.q) + (static_cast<long>(b) * p.Nq + (active ? i : 0)) * p.ldq + h * D;
  for (int c = 0; c < D; ++c) qrow[c] = active ? to_f32(qp[c]) * qscale : 0.f;
  float res[D], res2[D];
#pragma unroll
  for (int c = 0; c < D; ++c) res[c] = res2[c] = 0.f;
  float lz1 = 0.f, lz2 = 0.f;
  sdpa_one_set<T, D>(reinterpret_cast<const T*>(p.k1) + static_cast<long>(b) * p.n1 * p.ld1,
                     reinterpret_cast<const T*>(p.v1) + static_cast<long>(b) * p.n1 * p.ld1, p.ld1, p.n1, qrow,
                     active, p.exact ? 1.f : p.w1, res, ks, vs, h, &lz1);
  if (p.n2 > 0)
    sdpa_one_set<T, D>(reinterpret_cast<const T*>(p.k2) + static_cast<long>(b) * p.n2 * p.ld2,
                       reinterpret_cast<const T*>(p.v2) + static_cast<long>(b) * p.n2 * p.ld2, p.ld2, p.n2, qrow,
                       active, p.exact ? 1.f : p.w2, p.exact ? res2 : res, ks, vs, h, &lz2);
  if (!active) return;
  T* op = reinterpret_cast<T*>(p.out) + (static_cast<long>(b) * p.Nq + i) * p.ldo + h * D;
  // exact: eta = A / (A + B) as 1 / (1 + 2^(log2 B - log2 A)); one set blends with the
  // linear part (A = den), two sets share one softmax (A, B their normalisers)
  float eta = 0.f;
  if (p.exact) {
    const float lza = p.n2 > 0 ? lz1 : log2f(p.den[(static_cast<long>(b) * p.Nq + i) * p.heads + h]);
    eta = 1.f / (1.f + exp2f((p.n2 > 0 ? lz2 : lz1) - lza));
  }
#pragma unroll
  for (int c = 0; c < D; ++c) {
    float v = res[c];
    if (p.exact)
      v = p.n2 > 0 ? eta * res[c] + (1.f - eta) * res2[c] : (1.f - eta) * res[c];
    if (p.blend_in) v = fmaf(p.exact ? eta : p.w0, to_f32(op[c]), v);
    op[c] = from_f32<T>(v);
  }
}

// ============================================================ DiT block
// 8 consecutive elements (16-byte aligned) to / from fp32 registers.
__device__ __forceinline__ void load8(const float* p, float (&o)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&o)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void store8(float* p, const float (&o)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(o[4], o[5], o[6], o[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&o)[8]) {
  uint4 u;
  u.x = pack_bf16x2(o[0], o[1]);
  u.y = pack_bf16x2(o[2], o[3]);
  u.z = pack_bf16x2(o[4], o[5]);
  u.w = pack_bf16x2(o[6], o[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

// Residual stream and LayerNorm modulation of the DiT block around the
// attention, one warp per token row (C % 8 == 0, C <= 2048):
//   r = base + g * delta (delta optional; g = sst[kg] + t6[b][kg], or 1 when kg < 0)
//   h = LN(r) (1 + sst[ks] + t6[b][ks]) + sst[kh] + t6[b][kh]   (LN without affine)
// r is written to r_out and h to h_out when they are non-NULL. Row stats in
// fp32 (two passes over the row held in registers).
template <typename T>
__global__ void __launch_bounds__(256) dit_residual_ln_kernel(const T* __restrict__ base, const T* __restrict__ delta,
                                                              const T* __restrict__ sst, const T* __restrict__ t6,
                                                              int kg, int ks, int kh, long rows_per_img, long rows,
                                                              int C, float eps, T* __restrict__ r_out,
                                                              T* __restrict__ h_out) {
  pdl_wait();
  constexpr int MAXV = 8;  // 8-element vectors per lane: C <= 32 * 8 * 8
  const int lane = threadIdx.x & 31;
  const long row = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= rows) return;
  const long b = row / rows_per_img;
  const int nv = C / 8;
  const T* mb = t6 + b * 6L * C;
  float v[MAXV][8];
  float s1 = 0.f;
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = lane + 32 * k;
    if (vi < nv) {
      const long off = row * C + 8L * vi;
      load8(base + off, v[k]);
      if (delta) {
        float dl[8], g[8], gt[8];
        load8(delta + off, dl);
        if (kg >= 0) {
          load8(sst + kg * C + 8 * vi, g);
          load8(mb + kg * C + 8 * vi, gt);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) v[k][i] = fmaf(kg >= 0 ? g[i] + gt[i] : 1.f, dl[i], v[k][i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) s1 += v[k][i];
      if (r_out) store8(r_out + off, v[k]);
    }
  }
  if (!h_out) return;
  const float mean = warp_sum(s1) / static_cast<float>(C);
  float s2 = 0.f;
#pragma unroll
  for (int k = 0; k < MAXV; ++k)
    if (lane + 32 * k < nv)
#pragma unroll
      for (int i = 0; i < 8; ++i) s2 = fmaf(v[k][i] - mean, v[k][i] - mean, s2);
  const float rstd = rsqrtf(warp_sum(s2) / static_cast<float>(C) + eps);
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int vi = lane + 32 * k;
    if (vi < nv) {
      float sc[8], sct[8], sh[8], sht[8], o[8];
      load8(sst + ks * C + 8 * vi, sc);
      load8(mb + ks * C + 8 * vi, sct);
      load8(sst + kh * C + 8 * vi, sh);
      load8(mb + kh * C + 8 * vi, sht);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = fmaf((v[k][i] - mean) * rstd, 1.f + sc[i] + sct[i], sh[i] + sht[i]);
      store8(h_out + row * C + 8L * vi, o);
    }
  }
}

// ================================================================ row bands
// One image split into row bands over several ranks (edit_attn_band_*): each
// band contributes partial sums to the layer's two global reductions, the
// GroupNorm statistics of U and the per-head [S | z]; every rank then sums all
// bands' records in band order.

// Band GroupNorm sums: (sum, sum of squares) per group over this band's
// tokens, from the gn_partial_kernel partials part [P][groups][2] (one image),
// in fp64 with a fixed order (thread t sums partials t, t + 256, ..., then a
// fixed tree). One block of 256 threads per group.
__global__ void __launch_bounds__(256) gn_band_sums_kernel(const float* __restrict__ part, int P, int groups,
                                                          double* __restrict__ out) {
  pdl_wait();
  __shared__ double r1[256], r2[256];
  const int g = blockIdx.x, t = threadIdx.x;
  double s1 = 0.0, s2 = 0.0;
  for (int i = t; i < P; i += 256) {
    const float2 q = *reinterpret_cast<const float2*>(part + (static_cast<long>(i) * groups + g) * 2);
    s1 += q.x;
    s2 += q.y;
  }
  r1[t] = s1;
  r2[t] = s2;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (t < w) {
      r1[t] += r1[t + w];
      r2[t] += r2[t + w];
    }
    __syncthreads();
  }
  if (t == 0) {
    out[g * 2] = r1[0];
    out[g * 2 + 1] = r2[0];
  }
}

// Global GroupNorm from all bands' records (rec_stride bytes apart, the fp64
// sums first): totals summed in band order in fp64, then mean, biased
// variance, rstd over `count` elements per group and the per-channel affine
// form scale = gamma * rstd, shift = beta - mean * scale. One block per group.
__global__ void __launch_bounds__(64) gn_band_finalize_kernel(const uint8_t* __restrict__ recs, int nrec,
                                                             long rec_stride, int groups, int Cr, long count, float eps,
                                                             const __nv_bfloat16* __restrict__ gamma,
                                                             const __nv_bfloat16* __restrict__ beta,
                                                             float* __restrict__ stats, float* __restrict__ ss) {
  pdl_wait();
  const int g = blockIdx.x;
  double s1 = 0.0, s2 = 0.0;
  for (int r = 0; r < nrec; ++r) {
    const double* q = reinterpret_cast<const double*>(recs + r * rec_stride) + 2 * g;
    s1 += q[0];
    s2 += q[1];
  }
  const double mean = s1 / static_cast<double>(count);
  double var = s2 / static_cast<double>(count) - mean * mean;
  if (var < 0.0) var = 0.0;
  const double rstd = 1.0 / sqrt(var + static_cast<double>(eps));
  if (threadIdx.x == 0) {
    stats[g * 2] = static_cast<float>(mean);
    stats[g * 2 + 1] = static_cast<float>(rstd);
  }
  const int cpg = Cr / groups;
  for (int c = g * cpg + threadIdx.x; c < (g + 1) * cpg; c += blockDim.x) {
    const double sc = static_cast<double>(__bfloat162float(gamma[c])) * rstd;
    ss[c * 2] = static_cast<float>(sc);
    ss[c * 2 + 1] = static_cast<float>(static_cast<double>(__bfloat162float(beta[c])) - mean * sc);
  }
}

// Global [S | z] from all bands' records (the fp32 [heads][d][d + 1] block at
// byte sz_off of each record), summed in band order; writes Sz and the bf16
// apply operand SzT [heads][NP][KP] (SzT[h][c][a] = [S | z]_h[a][c], zero
// outside c <= d, a < d), as kv_state_combine_pack_kernel does for one image.
__global__ void sz_band_combine_pack_kernel(const uint8_t* __restrict__ recs, int nrec, long rec_stride, long sz_off,
                                            int d, int NP, int KP, long total, float* __restrict__ Sz,
                                            __nv_bfloat16* __restrict__ SzT) {
  pdl_wait();
  const int per_head = d * (d + 1);
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const int a = static_cast<int>(i % KP);
    const long r = i / KP;
    const int c = static_cast<int>(r % NP);
    const long h = r / NP;
    float s = 0.f;
    if (c <= d && a < d) {
      const long e = h * per_head + a * (d + 1) + c;
      for (int k = 0; k < nrec; ++k) s += reinterpret_cast<const float*>(recs + k * rec_stride + sz_off)[e];
      Sz[e] = s;
    }
    SzT[i] = __float2bfloat16_rn(s);
  }
}

}  // namespace
}  // namespace edit

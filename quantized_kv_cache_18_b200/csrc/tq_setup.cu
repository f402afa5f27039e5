// TurboQuant-style deployment constants and the per-step query rotation.
//
// The rotation Pi is a random orthogonal matrix: the Q factor of the QR
// decomposition of a seeded N(0, 1) draw, with the sign of each column fixed so
// that diag(R) > 0 ("Quantification du KV-Cache : TurboQuant et l'etat de l'art
// en 2026", "TurboQuant : les cinq innovations", item 1; zubnet.ai survey,
// "Famille deux ..."), or, in the Walsh-Hadamard variant that item 1 names,
// H_d / sqrt(d) in Sylvester order.  Each rotated coordinate then has the law N(0, 1/d), and
// the scalar quantizer is the 8-level Lloyd-Max quantizer of that law, fixed at
// deployment (same page, item 2): levels are the Lloyd-Max levels of N(0, 1)
// scaled by 1/sqrt(d) and stored in fp16, thresholds are the midpoints of
// adjacent levels.  The QJL projection S is the caller's N(0, 1) draw as is.
//
// turbo_setup_kernel   one CTA: Householder QR in fp64 in shared memory, the
//                      Lloyd-Max fixed point in fp64, then the fp32 tables.
// tq_query_prep_kernel four CTAs per (batch, kv head): q' = Pi q and
//                      q'' = (S Pi) q for the row's query heads, split into
//                      fp16 hi + lo and stored in the A-fragment order of the
//                      decode kernel.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kSetupThreads = 256;

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// A (column-major, A[j * D + i] = element (i, j)) is factored in place: column
// k keeps the Householder vector v_k on rows k..D-1 (v_k[k] included), tau[k] =
// 2 / (v_k . v_k) (0 for an identity step) and rdiag[k] = R[k][k].
__global__ void __launch_bounds__(kSetupThreads, 1)
    turbo_setup_kernel(const float* __restrict__ rot_gauss, const float* __restrict__ qjl_gauss,
                       unsigned char* __restrict__ params, uint32_t* status, int wht) {
  constexpr int D = kTqD, M = kTqM;
  extern __shared__ __align__(16) double A[];   // [D][D]
  __shared__ double tau[D], rdiag[D];
  __shared__ uint32_t s_flags;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NW = kSetupThreads / 32;
  if (tid == 0) s_flags = 0;
  __syncthreads();

  uint32_t flags = 0;
  float* Pi = reinterpret_cast<float*>(params + kTqPi);
  float* PiT = reinterpret_cast<float*>(params + kTqPiT);
  if (wht) {
    // Walsh-Hadamard rotation: Pi[i][j] = (-1)^popcount(i & j) / sqrt(d)
    // (Sylvester order), exactly +-fp32(1 / sqrt(d)); symmetric, so Pi^T = Pi
    const float c = (float)(1.0 / sqrt((double)D));
    for (int e = tid; e < D * D; e += kSetupThreads) {
      const int i = e / D, j = e - i * D;
      const float v = (__popc(i & j) & 1) ? -c : c;
      Pi[e] = v;
      PiT[e] = v;
    }
  } else {
  for (int e = tid; e < D * D; e += kSetupThreads) {
    const int i = e / D, j = e - i * D;
    const float g = rot_gauss[e];   // row-major [i][j]
    if (!isfinite(g)) flags |= KVQ_DEV_NONFINITE_INPUT;
    A[j * D + i] = (double)g;
  }
  __syncthreads();

  // ---------------------------------------------------------------- Householder QR
  for (int k = 0; k < D; ++k) {
    if (warp == 0) {
      double s = 0.0;
      for (int i = k + lane; i < D; i += 32) s += A[k * D + i] * A[k * D + i];
      s = warp_sum_d(s);
      if (lane == 0) {
        const double x0 = A[k * D + k];
        const double nrm = sqrt(s);
        if (nrm == 0.0) {
          tau[k] = 0.0;
          rdiag[k] = 0.0;
        } else {
          const double alpha = x0 >= 0.0 ? -nrm : nrm;   // reflect x onto alpha e_1, away from x
          A[k * D + k] = x0 - alpha;                      // v = x - alpha e_1
          tau[k] = 1.0 / (nrm * (nrm + fabs(x0)));        // 2 / (v . v)
          rdiag[k] = alpha;
        }
      }
    }
    __syncthreads();
    const double tk = tau[k];
    if (tk != 0.0) {
      for (int j = k + 1 + warp; j < D; j += NW) {
        double dot = 0.0;
        for (int i = k + lane; i < D; i += 32) dot += A[k * D + i] * A[j * D + i];
        const double f = tk * warp_sum_d(dot);
        for (int i = k + lane; i < D; i += 32) A[j * D + i] -= f * A[k * D + i];
      }
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------- Q = H_0 H_1 ... H_{D-1}, column by column
  for (int j = warp; j < D; j += NW) {
    double x[D / 32];
#pragma unroll
    for (int r = 0; r < D / 32; ++r) x[r] = (lane + 32 * r == j) ? 1.0 : 0.0;
    // H_k e_j = e_j for k > j (v_k vanishes above row k)
    for (int k = j; k >= 0; --k) {
      const double tk = tau[k];
      if (tk == 0.0) continue;
      double dot = 0.0;
#pragma unroll
      for (int r = 0; r < D / 32; ++r) {
        const int i = lane + 32 * r;
        if (i >= k) dot += A[k * D + i] * x[r];
      }
      const double f = tk * warp_sum_d(dot);
#pragma unroll
      for (int r = 0; r < D / 32; ++r) {
        const int i = lane + 32 * r;
        if (i >= k) x[r] -= f * A[k * D + i];
      }
    }
    const double sg = rdiag[j] < 0.0 ? -1.0 : 1.0;   // diag(R) > 0 after the sign fix (0 counts as +)
#pragma unroll
    for (int r = 0; r < D / 32; ++r) {
      const int i = lane + 32 * r;
      const float v = (float)(sg * x[r]);
      Pi[i * D + j] = v;
      PiT[j * D + i] = v;
    }
  }
  }   // QR rotation

  // ---------------------------------------------------------------- S^T
  float* ST = reinterpret_cast<float*>(params + kTqST);
  for (int e = tid; e < M * D; e += kSetupThreads) {
    const int i = e / D, j = e - i * D;   // S row-major [i][j]
    const float g = qjl_gauss[e];
    if (!isfinite(g)) flags |= KVQ_DEV_NONFINITE_INPUT;
    ST[j * M + i] = g;
  }

  // ---------------------------------------------------------------- Lloyd-Max for N(0, 1), 8 levels
  // Alternate: thresholds = midpoints of the levels, levels = conditional
  // means of their cells, E[X | a < X < b] = (phi(a) - phi(b)) / (Phi(b) - Phi(a)),
  // from levels evenly spaced on [-2, 2] until no level moves by 1e-15.
  if (warp == 0) {
    const double inv_sqrt_2pi = 1.0 / sqrt(2.0 * 3.14159265358979323846);
    const int l = lane & 7;
    double c = l == 7 ? 2.0 : -2.0 + (double)l * (4.0 / 7.0);
    for (int it = 0; it < 10000; ++it) {
      const double cm = __shfl_up_sync(0xffffffffu, c, 1, 8);
      const double cp = __shfl_down_sync(0xffffffffu, c, 1, 8);
      const double lo = l == 0 ? -INFINITY : 0.5 * (c + cm);
      const double hi = l == 7 ? INFINITY : 0.5 * (cp + c);
      const double plo = l == 0 ? 0.0 : exp(-0.5 * lo * lo) * inv_sqrt_2pi;
      const double phi_hi = l == 7 ? 0.0 : exp(-0.5 * hi * hi) * inv_sqrt_2pi;
      const double mass = normcdf(hi) - normcdf(lo);
      const double nc = (plo - phi_hi) / mass;
      double diff = fabs(nc - c);
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) diff = fmax(diff, __shfl_xor_sync(0xffffffffu, diff, o, 8));
      c = nc;
      if (diff < 1e-15) break;
    }
    // deployed: fp16 levels of N(0, 1/d); midpoints are exact in fp32.  The
    // quantizer is odd-symmetric; the lower four levels are taken as the
    // negatives of the upper four, so the deployed thresholds are exactly
    // symmetric with the middle one 0 (the tensor-core quantizer relies on it).
    const uint16_t hu = __half_as_ushort(__double2half(c / sqrt((double)D)));
    const uint16_t hm = __shfl_sync(0xffffffffu, hu, 7 - l, 8);
    const __half h = __ushort_as_half(l < 4 ? (uint16_t)(hm ^ 0x8000u) : hu);
    const float lv = __half2float(h);
    const float lv_next = __shfl_down_sync(0xffffffffu, lv, 1, 8);
    float* levels = reinterpret_cast<float*>(params + kTqLevels);
    float* thr = reinterpret_cast<float*>(params + kTqThr);
    uint16_t* lv16 = reinterpret_cast<uint16_t*>(params + kTqLevels16);
    if (lane < 8) {
      levels[l] = lv;
      lv16[l] = __half_as_ushort(h);
      thr[l] = l < 7 ? 0.5f * (lv + lv_next) : INFINITY;
    }
    const uint16_t h_lo = __shfl_sync(0xffffffffu, __half_as_ushort(h), lane & 7);
    const uint16_t h_hi = __shfl_sync(0xffffffffu, __half_as_ushort(h), (lane >> 3) & 7);
    uint32_t* lut = reinterpret_cast<uint32_t*>(params + kTqLut);
    // lanes 0..31 write indices 0..31 (hi = lane >> 3 in 0..3), then 32..63
    lut[lane] = (uint32_t)h_lo | ((uint32_t)h_hi << 16);
    const uint16_t h_hi2 = __shfl_sync(0xffffffffu, __half_as_ushort(h), 4 + ((lane >> 3) & 3));
    lut[32 + lane] = (uint32_t)h_lo | ((uint32_t)h_hi2 << 16);
  }
  // ---------------------------------------------------------------- (S Pi)^T, fp64 sums of the fp32 tables
  // q'' = S Pi q is then one product with q, like q' = Pi q
  __syncthreads();   // Pi and S^T are in the parameter block
  {
    const float* PiG = reinterpret_cast<const float*>(params + kTqPi);
    float* SPiT = reinterpret_cast<float*>(params + kTqSPiT);
    for (int e = tid; e < D * M; e += kSetupThreads) {
      const int j = e / M, i = e - j * M;   // SPiT[j][i] = sum_k S[i][k] Pi[k][j]
      double acc = 0.0;
      for (int k = 0; k < D; ++k) acc += (double)ST[k * M + i] * (double)PiG[k * D + j];
      SPiT[e] = (float)acc;
    }
    // ---------------------------------------------------------------- tcgen05 operand images of 16 Pi and S
    // (the quantizer scales u by 16 as well, so the lo parts of both stay
    // clear of fp16 subnormals)
    __half* img = reinterpret_cast<__half*>(params + kTqBImg);
    __nv_bfloat16* imb = reinterpret_cast<__nv_bfloat16*>(params + kTqBImg + kTqBImgSet);
    constexpr int kHalves = kTqBImgBytes / 2;
    for (int e = tid; e < D * D; e += kSetupThreads) {
      const int n = e / D, k = e - n * D;
      const int off = ((k >> 3) * 2048 + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2) / 2;
      const float p = 16.f * PiG[n * D + k];   // B[n][k] = 16 Pi[n][k]
      const float q = ST[k * M + n];           // B[n][k] = S[n][k]
      const __half ph = __float2half_rn(p), qh = __float2half_rn(q);
      img[off] = ph;
      img[kHalves + off] = __float2half_rn(p - __half2float(ph));
      img[2 * kHalves + off] = qh;
      img[3 * kHalves + off] = __float2half_rn(q - __half2float(qh));
      const __nv_bfloat16 pb = __float2bfloat16_rn(p), qb = __float2bfloat16_rn(q);
      imb[off] = pb;
      imb[kHalves + off] = __float2bfloat16_rn(p - __bfloat162float(pb));
      imb[2 * kHalves + off] = qb;
      imb[3 * kHalves + off] = __float2bfloat16_rn(q - __bfloat162float(qb));
    }
  }
  if (flags) atomicOr(&s_flags, flags);
  __syncthreads();
  if (tid == 0 && s_flags) atomicOr(status, s_flags);
}

// ---------------------------------------------------------------- query rotation
// q' = Pi q and q'' = (S Pi) q of every query head of a row, split into fp16
// hi + lo in the A-fragment order of the decode kernel.  The 256 outputs of a
// head (128 of q', 128 of q'') are cut into four quarters, one CTA each, so a
// row takes four CTAs and each stages only its 64 columns of Pi^T or (S Pi)^T
// (32 KB): every output is one 128-term fp32 dot product, no product waits
// for another.
constexpr int kPrepThreads = 256;
constexpr int kPrepCols = 64;   // outputs per CTA

__device__ __forceinline__ uint32_t pack_h2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

__global__ void __launch_bounds__(kPrepThreads)
    tq_query_prep_kernel(Geom gm, const uint16_t* __restrict__ q, unsigned char* __restrict__ qprep) {
  constexpr int D = kTqD;
  __shared__ __align__(16) float sW[D][kPrepCols];   // column slice of Pi^T or (S Pi)^T
  __shared__ float qf[8][D];                          // raw q of the row's heads
  __shared__ float y[8][kPrepCols + 1];               // this quarter of Pi q or S Pi q
  const int row = blockIdx.x, k = blockIdx.y;         // quarter k: outputs 64 k .. 64 k + 63 of [q' | q'']
  const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
  const int g = gm.g;
  const int tid = threadIdx.x;
  const int vec = k >> 1, c0 = kPrepCols * (k & 1);
  const float* W = reinterpret_cast<const float*>(gm.params + (vec == 0 ? kTqPiT : kTqSPiT));
  // the slice is requested at once (8 x 16-byte loads per thread)
  uint4 v[D * kPrepCols / 4 / kPrepThreads];
#pragma unroll
  for (int u = 0; u < D * kPrepCols / 4 / kPrepThreads; ++u) {
    const int e = tid + u * kPrepThreads;   // float4 index in the slice: row e / 16, column 4 (e % 16)
    v[u] = __ldg(reinterpret_cast<const uint4*>(W + (e >> 4) * D + c0) + (e & 15));
  }
  const uint16_t* qrow = q + ((int64_t)b * gm.Hq + (int64_t)hkv * g) * D;
  for (int e = tid; e < 8 * D; e += kPrepThreads) {
    const int h = e / D;
    qf[h][e - h * D] = h < g ? in16_to_float(qrow[e], gm.dtype) : 0.f;
  }
#pragma unroll
  for (int u = 0; u < D * kPrepCols / 4 / kPrepThreads; ++u) {
    const int e = tid + u * kPrepThreads;
    reinterpret_cast<uint4*>(&sW[e >> 4][0])[e & 15] = v[u];
  }
  __syncthreads();
  {
    const int i = tid & (kPrepCols - 1), h0 = tid / kPrepCols;   // heads h0 and h0 + 4
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
    for (int j = 0; j < D; ++j) {
      const float w = sW[j][i];
      acc0 = fmaf(w, qf[h0][j], acc0);
      acc1 = fmaf(w, qf[h0 + 4][j], acc1);
    }
    y[h0][i] = acc0;
    y[h0 + 4][i] = acc1;
  }
  __syncthreads();
  // fragments: [vector (q', q'')][kt][lane] uint4 =
  //   {hi(gr, c..c+1), lo(gr, c..c+1), hi(gr, c+8..c+9), lo(gr, c+8..c+9)}, c = 16 kt + 2 tc
  if (tid < 4 * 32) {
    const int ktl = tid >> 5, lane = tid & 31, kt = (c0 >> 4) + ktl;
    const int gr = lane >> 2, tc = lane & 3;
    uint32_t w[4];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int c = 16 * ktl + 8 * half + 2 * tc;   // column of this quarter
      const float x0 = y[gr][c], x1 = y[gr][c + 1];
      const __half h0v = __float2half_rn(x0), h1v = __float2half_rn(x1);
      const __half l0 = __float2half_rn(x0 - __half2float(h0v)), l1 = __float2half_rn(x1 - __half2float(h1v));
      w[2 * half] = pack_h2(h0v, h1v);
      w[2 * half + 1] = pack_h2(l0, l1);
    }
    uint4* out = reinterpret_cast<uint4*>(qprep + (int64_t)row * kTqQPrepBytes);
    out[(vec * (D / 16) + kt) * 32 + lane] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

void launch_turbo_setup(const Geom& g, const float* rot_gauss, const float* qjl_gauss, bool wht, cudaStream_t st) {
  const int smem = kTqD * kTqD * (int)sizeof(double);
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(turbo_setup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    attr_set = true;
  }
  turbo_setup_kernel<<<1, kSetupThreads, smem, st>>>(rot_gauss, qjl_gauss, g.params, g.status, wht ? 1 : 0);
  count_launch(1);
}

void launch_tq_query_prep(const Geom& g, const uint16_t* q, unsigned char* qprep, cudaStream_t st) {
  tq_query_prep_kernel<<<dim3(g.B * g.Hkv, 4), kPrepThreads, 0, st>>>(g, q, qprep);
  count_launch(1);
}

}  // namespace kvq

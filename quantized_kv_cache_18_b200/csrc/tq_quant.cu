// TurboQuant-style quantization of 32-token blocks (prefill and window flush).
//
// Per token vector x (one kv head): n = ||x||, u = x / n, y = Pi u; each
// coordinate of y gets the 3-bit index of its Lloyd-Max cell ("Quantification du
// KV-Cache : TurboQuant et l'etat de l'art en 2026", "TurboQuant : les cinq
// innovations", items 1-2).  Keys also keep a 1-bit Johnson-Lindenstrauss
// sketch of the quantization residual e = y - c_hat: the signs of S e and
// gamma = n ||e|| (item 3; zubnet.ai survey, "Famille deux ..."), which the
// decode kernel uses to correct the key inner products.  n and gamma are
// stored in fp16.
//
// Readings: the residual is taken in rotated coordinates; a coordinate equal
// to a threshold goes to the lower cell; a sketch value of exactly 0 gives bit
// 1; the zero vector has u = 0.  Codes are decided on y computed in fp32 (Pi
// in fp32, fp32 accumulation).
//
// One persistent CTA per SM keeps 16 Pi and S in shared memory as mma.sync
// A fragments, each split into fp16 hi + lo, and loops over (row, block)
// tasks.  Each task runs three 128 x 128 x 32 products on the tensor cores
// (keys: Pi U and S E, values: Pi U) as hi*hi + hi*lo + lo*hi with fp32
// accumulation (about 22 significant bits, the dropped lo*lo term below
// 2^-22 of each product); U is scaled by 16 and E by 64 so that the lo parts
// stay clear of fp16 subnormals.  With the Walsh-Hadamard rotation, Pi U is
// the in-register fast transform instead (7 add/sub stages per vector),
// leaving S E as the one product.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kQThreads = 256;
constexpr int kTok = 32;

struct QSmem {
  // A operands of the two products, split fp16 hi + lo, in mma fragment order:
  // [m-tile 8][k-tile 8][lane 32] x (hi a0..a3, lo a0..a3) = 32 bytes
  static constexpr int AP = 0;                                // 16 Pi
  static constexpr int AS = AP + 8 * 8 * 32 * 32;             // S
  static constexpr int X = AS + 8 * 8 * 32 * 32;              // uint16 [32][128] input tile
  static constexpr int U = X + kTok * kTqD * 2;               // float [128][32] unit vectors (or y)
  static constexpr int E = U + kTqD * kTok * 4;               // float [128][32] key residuals
  static constexpr int CK = E + kTqD * kTok * 4;              // uint8 [32][128] key codes
  static constexpr int CV = CK + kTok * kTqD;                 // uint8 [32][128] value codes
  static constexpr int SG = CV + kTok * kTqD;                 // uint8 [32][128] sign bits
  static constexpr int NK = SG + kTok * kTqM;                 // double [32] key norms
  static constexpr int NV = NK + kTok * 8;                    // double [32] value norms
  static constexpr int ESQ = NV + kTok * 8;                   // double [8 warps][32] partial ||e||^2
  static constexpr int XF = ESQ + 8 * kTok * 8;               // float [32][128] FP8 input tile, exact values;
  static constexpr int BF = XF;                               // reused for the B operands [8][4][32] x 16 B
  static constexpr int BYTES = XF + kTok * kTqD * 4;
};

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// fp16 hi + lo split of two fp32 values, packed as fp16x2 pairs
__device__ __forceinline__ void split2(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(v0, v1);
  const float2 hf = __half22float2(h);
  hi = h2_as_u32(h);
  lo = h2_as_u32(__floats2half2_rn(v0 - hf.x, v1 - hf.y));
}

// A operand of a 128 x 128 product (W[i][j] * scale, i = output row, j =
// summed index; W read from global memory, stored row-major, or transposed
// as W[j][i]) into mma fragment order, split hi + lo.
__device__ __forceinline__ void build_a_frags(const float* W, float scale, bool transposed, unsigned char* dst,
                                              int tid) {
  auto w = [&](int i, int j) { return __ldg(transposed ? W + j * kTqD + i : W + i * kTqD + j) * scale; };
  for (int q = tid; q < 8 * 8 * 32; q += kQThreads) {
    const int mt = q >> 8, kt = (q >> 5) & 7, lane = q & 31;
    const int gr = lane >> 2, tc = lane & 3;
    const int r0 = 16 * mt + gr, c0 = 16 * kt + 2 * tc;
    uint32_t h[4], l[4];
    split2(w(r0, c0), w(r0, c0 + 1), h[0], l[0]);
    split2(w(r0 + 8, c0), w(r0 + 8, c0 + 1), h[1], l[1]);
    split2(w(r0, c0 + 8), w(r0, c0 + 9), h[2], l[2]);
    split2(w(r0 + 8, c0 + 8), w(r0 + 8, c0 + 9), h[3], l[3]);
    uint4* o = reinterpret_cast<uint4*>(dst + q * 32);
    o[0] = make_uint4(h[0], h[1], h[2], h[3]);
    o[1] = make_uint4(l[0], l[1], l[2], l[3]);
  }
}

// B operand (K = 128 summed index j, N = 32 tokens) from X[j][32] * scale into
// fragment order [k-tile 8][n-tile 4][lane 32] x (hi b0, hi b1, lo b0, lo b1).
__device__ __forceinline__ void build_b_frags(const float* X, float scale, unsigned char* dst, int tid) {
  for (int q = tid; q < 8 * 4 * 32; q += kQThreads) {
    const int kt = q >> 7, nt = (q >> 5) & 3, lane = q & 31;
    const int gr = lane >> 2, tc = lane & 3;
    const int j0 = 16 * kt + 2 * tc, t = 8 * nt + gr;
    uint32_t h0, l0, h1, l1;
    split2(X[j0 * kTok + t] * scale, X[(j0 + 1) * kTok + t] * scale, h0, l0);
    split2(X[(j0 + 8) * kTok + t] * scale, X[(j0 + 9) * kTok + t] * scale, h1, l1);
    reinterpret_cast<uint4*>(dst)[q] = make_uint4(h0, h1, l0, l1);
  }
}

// acc[nt] = rows 16 mt .. 16 mt + 15 (the warp's m-tile) x tokens 8 nt .. 8 nt + 7
// of A B, as hi hi + hi lo + lo hi (about 22 bits; the lo lo term is dropped).
// C layout: acc[nt][0..1] = row 16 mt + gr, tokens 8 nt + 2 tc + {0, 1};
// acc[nt][2..3] = row 16 mt + 8 + gr, the same tokens.
__device__ __forceinline__ void product_tile(const unsigned char* A, const unsigned char* B, int mt, int lane,
                                             float acc[4][4]) {
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 2
  for (int kt = 0; kt < 8; ++kt) {
    const uint4 ah = *reinterpret_cast<const uint4*>(A + ((mt * 8 + kt) * 32 + lane) * 32);
    const uint4 al = *reinterpret_cast<const uint4*>(A + ((mt * 8 + kt) * 32 + lane) * 32 + 16);
    const uint32_t ahv[4] = {ah.x, ah.y, ah.z, ah.w}, alv[4] = {al.x, al.y, al.z, al.w};
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const uint4 b = reinterpret_cast<const uint4*>(B)[(kt * 4 + nt) * 32 + lane];
      mma_f16_16816(acc[nt], ahv, b.x, b.y);
      mma_f16_16816(acc[nt], ahv, b.z, b.w);
      mma_f16_16816(acc[nt], alv, b.x, b.y);
    }
  }
}

// In-register Walsh-Hadamard transform (Sylvester order, unnormalised) of a
// 128-vector held as element lane + 32 r in v[r]: butterflies of span 1..16
// across lanes, of span 32 and 64 across the four registers.
__device__ __forceinline__ void fwht128(float v[4], int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float p = __shfl_xor_sync(0xffffffffu, v[r], h);
      v[r] = (lane & h) ? p - v[r] : v[r] + p;
    }
  }
  const float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2;
  v[2] = a0 - a2;
  v[1] = a1 + a3;
  v[3] = a1 - a3;
}

// Norms and unit vectors of the 32 tokens in X (16-bit) or XF (exact fp32
// values of FP8 rows): warp w handles tokens 4w..4w+3.
// With wht, U receives y = H u / sqrt(d) instead of u (the rotation applied by
// the fast transform; Pi = H / sqrt(d) holds exactly +-fp32(1 / sqrt(d))).
__device__ __forceinline__ uint32_t unit_vectors(const uint16_t* X, const float* XF, float* U, double* nrm,
                                                 int dtype, int warp, int lane, bool wht) {
  uint32_t flags = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int t = 4 * warp + k;
    float x[4];
    double s = 0.0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      x[r] = XF != nullptr ? XF[t * kTqD + lane + 32 * r] : in16_to_float(X[t * kTqD + lane + 32 * r], dtype);
      if (!isfinite(x[r])) flags |= KVQ_DEV_NONFINITE_INPUT;
      s += (double)x[r] * (double)x[r];
    }
    const double n = sqrt(warp_sum_d(s));
    const double inv = n > 0.0 ? 1.0 / n : 0.0;
    float u[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) u[r] = (float)((double)x[r] * inv);
    if (wht) {
      fwht128(u, lane);
      const float c = (float)(1.0 / sqrt((double)kTqD));
#pragma unroll
      for (int r = 0; r < 4; ++r) u[r] *= c;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) U[(lane + 32 * r) * kTok + t] = u[r];
    if (lane == 0) nrm[t] = n;
  }
  return flags;
}

__global__ void __launch_bounds__(kQThreads, 1) tq_quantize_kernel(QuantArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* sX = reinterpret_cast<uint16_t*>(smem + QSmem::X);
  float* sU = reinterpret_cast<float*>(smem + QSmem::U);
  float* sE = reinterpret_cast<float*>(smem + QSmem::E);
  uint8_t* sCK = smem + QSmem::CK;
  uint8_t* sCV = smem + QSmem::CV;
  uint8_t* sSG = smem + QSmem::SG;
  double* sNK = reinterpret_cast<double*>(smem + QSmem::NK);
  double* sNV = reinterpret_cast<double*>(smem + QSmem::NV);
  double* sESQ = reinterpret_cast<double*>(smem + QSmem::ESQ);
  float* sXF = reinterpret_cast<float*>(smem + QSmem::XF);
  unsigned char* sBF = smem + QSmem::BF;
  __shared__ float s_thr[8], s_lv[8];
  __shared__ uint32_t s_flags;

  const Geom& gm = a.geom;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, tc = lane & 3;   // C fragment: rows 16 warp + gr (+8), tokens 8 nt + 2 tc (+1)

  {
    const float* P = reinterpret_cast<const float*>(gm.params);
    if (!gm.rot_wht) build_a_frags(P + kTqPi / 4, 16.f, false, smem + QSmem::AP, tid);
    build_a_frags(P + kTqST / 4, 1.f, true, smem + QSmem::AS, tid);
    if (tid < 8) {
      s_thr[tid] = P[kTqThr / 4 + tid];
      s_lv[tid] = P[kTqLevels / 4 + tid];
    }
    if (tid == 0) s_flags = 0;
  }
  __syncthreads();
  float thr[7];
#pragma unroll
  for (int k = 0; k < 7; ++k) thr[k] = s_thr[k];

  uint32_t flags = 0;
  const int64_t n_tasks = (int64_t)gm.B * gm.Hkv * a.n_groups;
  for (int64_t task = blockIdx.x; task < n_tasks; task += gridDim.x) {
    const int row = (int)(task / a.n_groups);
    const int blk = (int)(task - (int64_t)row * a.n_groups);
    for (int kv = 0; kv < 2; ++kv) {
      // ---------------------------------------------------------- stage the 32 tokens
      if (a.src_fp8 == nullptr) {
        const uint16_t* src =
            (kv == 0 ? a.src_k : a.src_v) + (int64_t)row * a.src_row_stride + (int64_t)blk * kTok * kTqD;
        for (int i = tid; i < kTok * kTqD / 8; i += kQThreads)
          reinterpret_cast<uint4*>(sX)[i] = ldg_nc_v4(reinterpret_cast<const uint4*>(src) + i);
      } else {
        // FP8 window rows (ring layout): x_hat = e4m3(code) * s, exact in fp32
        const unsigned char* src8 = a.src_fp8 + (int64_t)row * 2 * gm.cap * kFp8RowBytes +
                                    (int64_t)kv * gm.cap * kFp8RowBytes + (int64_t)blk * kTok * kFp8RowBytes;
        for (int i = tid; i < kTok * kTqD; i += kQThreads) {
          const int t = i / kTqD, c = i - t * kTqD;
          const unsigned char* rowp = src8 + t * kFp8RowBytes;
          const float sc = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(rowp + kTqD)));
          const float code = __half2float(__half(__nv_cvt_fp8_to_halfraw(rowp[c], __NV_E4M3)));
          sXF[i] = code * sc;
        }
      }
      __syncthreads();
      flags |= unit_vectors(sX, a.src_fp8 != nullptr ? sXF : nullptr, sU, kv == 0 ? sNK : sNV, gm.dtype, warp, lane,
                            gm.rot_wht != 0);
      __syncthreads();
      // ---------------------------------------------------------- y = Pi u, codes
      float acc[4][4];
      if (gm.rot_wht) {
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float2 y2 = *reinterpret_cast<const float2*>(sU + (16 * warp + gr + 8 * h) * kTok + 8 * nt + 2 * tc);
            acc[nt][2 * h] = y2.x;
            acc[nt][2 * h + 1] = y2.y;
          }
      } else {
        build_b_frags(sU, 16.f, sBF, tid);
        __syncthreads();
        product_tile(smem + QSmem::AP, sBF, warp, lane, acc);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nt][e] *= 1.f / 256.f;
      }
      uint8_t* codes = kv == 0 ? sCK : sCV;
      double esq[4][2] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float y = acc[nt][e];
          int c = 0;
#pragma unroll
          for (int k = 0; k < 7; ++k) c += y > thr[k] ? 1 : 0;
          const int i = 16 * warp + gr + 8 * (e >> 1), t = 8 * nt + 2 * tc + (e & 1);
          codes[t * kTqD + i] = (uint8_t)c;
          if (kv == 0) {
            const float r = y - s_lv[c];
            sE[i * kTok + t] = r;
            esq[nt][e & 1] += (double)r * (double)r;
          }
        }
      if (kv == 0) {
        // partial ||e||^2 of the warp's 16 rows, per token
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            double s = esq[nt][b];
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            s += __shfl_xor_sync(0xffffffffu, s, 8);
            s += __shfl_xor_sync(0xffffffffu, s, 16);
            if (gr == 0) sESQ[warp * kTok + 8 * nt + 2 * tc + b] = s;
          }
        __syncthreads();
        // ---------------------------------------------------------- sketch signs of S e
        build_b_frags(sE, 64.f, sBF, tid);
        __syncthreads();
        product_tile(smem + QSmem::AS, sBF, warp, lane, acc);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            sSG[(8 * nt + 2 * tc + (e & 1)) * kTqM + 16 * warp + gr + 8 * (e >> 1)] = acc[nt][e] >= 0.f ? 1 : 0;
      }
      __syncthreads();
    }

    // ---------------------------------------------------------- pack and store the token block
    uint32_t* dst = reinterpret_cast<uint32_t*>(record_ptr(gm, row, a.dst_group0 + blk));
    if (dst == nullptr) flags |= KVQ_DEV_BAD_PAGE;   // page outside the pool: nothing is written
    for (int qw = dst != nullptr ? tid : 2 * 416 + 128 + 32; qw < 2 * 416 + 128 + 32; qw += kQThreads) {
      if (qw < 2 * 416) {
        const int vblk = qw >= 416;
        const int q = qw - 416 * vblk;
        const int ln = q < 384 ? (q >> 2) & 31 : q - 384;
        const int w = q < 384 ? 4 * (q >> 7) + (q & 3) : 12;
        const int gr = ln >> 2, tc = ln & 3;
        uint32_t word = 0;
#pragma unroll
        for (int f = 0; f < 5; ++f) {
          const int slot = 5 * w + f;
          if (slot < 64) {
            uint32_t idx;
            if (!vblk) {
              const int nt = slot >> 4, kt = (slot >> 1) & 7, rho = slot & 1;
              const int t = 8 * nt + gr, c0 = 16 * kt + 8 * rho + 2 * tc;
              idx = sCK[t * kTqD + c0] + 8u * sCK[t * kTqD + c0 + 1];
            } else {
              const int kt = slot >> 5, nt = (slot >> 1) & 15, rho = slot & 1;
              const int c = 8 * nt + gr, t0 = 16 * kt + 8 * rho + 2 * tc;
              idx = sCV[t0 * kTqD + c] + 8u * sCV[(t0 + 1) * kTqD + c];
            }
            word |= idx << (6 * f);
          }
        }
        dst[(vblk ? kTqVCodes : kTqKCodes) / 4 + q] = word;
      } else if (qw < 2 * 416 + 128) {
        const int q = qw - 2 * 416;
        const int ln = q >> 2, w = q & 3;
        const int gr = ln >> 2, tc = ln & 3;
        const int t = 8 * w + gr;
        uint32_t word = 0;
#pragma unroll
        for (int s = 0; s < 16; ++s) {
          const int kt = s >> 1, rho = s & 1;
          const int i0 = 16 * kt + 8 * rho + 2 * tc;
          word |= (uint32_t)sSG[t * kTqM + i0] << s;
          word |= (uint32_t)sSG[t * kTqM + i0 + 1] << (16 + s);
        }
        dst[kTqSigns / 4 + q] = word;
      } else {
        const int t = qw - 2 * 416 - 128;   // token of the block
        const int kt = t >> 4, rho = (t >> 3) & 1, tc = (t >> 1) & 3, e = t & 1;
        const int entry = 8 * tc + 4 * kt + 2 * rho + e;
        const double nk = sNK[t], nv = sNV[t];
        const __half hn = __double2half(nk);
        double esq = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) esq += sESQ[w * kTok + t];
        const __half hg = __double2half(nk * sqrt(esq));
        const __half hv = __double2half(nv);
        if (isinf(__half2float(hn)) || isinf(__half2float(hg)) || isinf(__half2float(hv)))
          flags |= KVQ_DEV_PARAM_OVERFLOW;
        dst[kTqKMeta / 4 + entry] = (uint32_t)__half_as_ushort(hn) | ((uint32_t)__half_as_ushort(hg) << 16);
        reinterpret_cast<uint16_t*>(reinterpret_cast<unsigned char*>(dst) + kTqVMeta)[entry] = __half_as_ushort(hv);
      }
    }
    __syncthreads();
  }
  if (flags) atomicOr(&s_flags, flags);
  __syncthreads();
  if (tid == 0 && s_flags) atomicOr(gm.status, s_flags);
}

}  // namespace

void launch_tq_quantize(const QuantArgs& a, cudaStream_t st) {
  const int64_t tasks = (int64_t)a.geom.B * a.geom.Hkv * a.n_groups;
  if (tasks <= 0) return;
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(tq_quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, QSmem::BYTES);
    attr_set = true;
  }
  const int grid = (int)(tasks < num_sms() ? tasks : num_sms());
  tq_quantize_kernel<<<grid, kQThreads, QSmem::BYTES, st>>>(a);
  count_launch(1);
}

}  // namespace kvq

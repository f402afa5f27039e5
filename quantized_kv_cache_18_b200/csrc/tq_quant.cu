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
// One persistent CTA per SM keeps Pi^T and S^T (fp32, 64 KB each) in shared
// memory and loops over (row, block) tasks.  Each task runs three 32 x 128 x 128
// products on the CUDA cores (keys: Pi U and S E, values: Pi U); with the
// Walsh-Hadamard rotation, Pi U is the in-register fast transform instead
// (7 add/sub stages per vector), leaving S E as the one product.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kQThreads = 256;
constexpr int kTok = 32;

struct QSmem {
  static constexpr int PIT = 0;                               // float [128][128]
  static constexpr int ST = PIT + kTqD * kTqD * 4;            // float [128][128]
  static constexpr int X = ST + kTqD * kTqM * 4;              // uint16 [32][128] input tile
  static constexpr int U = X + kTok * kTqD * 2;               // float [128][32]
  static constexpr int E = U + kTqD * kTok * 4;               // float [128][32]
  static constexpr int CK = E + kTqD * kTok * 4;              // uint8 [32][128] key codes
  static constexpr int CV = CK + kTok * kTqD;                 // uint8 [32][128] value codes
  static constexpr int SG = CV + kTok * kTqD;                 // uint8 [32][128] sign bits
  static constexpr int NK = SG + kTok * kTqM;                 // double [32] key norms
  static constexpr int NV = NK + kTok * 8;                    // double [32] value norms
  static constexpr int ESQ = NV + kTok * 8;                   // double [32] ||e||^2
  static constexpr int XF = ESQ + kTok * 8;                   // float [32][128] FP8 input tile, exact values
  static constexpr int BYTES = XF + kTok * kTqD * 4;
};

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// acc[a][b] = sum_j WT[j][4 ti + a] * X[j][4 tt + b]   (WT [128][128], X [128][32])
__device__ __forceinline__ void matvec_tile(const float* WT, const float* X, int ti, int tt, float acc[4][4]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 4
  for (int j = 0; j < kTqD; ++j) {
    const float4 w = *reinterpret_cast<const float4*>(WT + j * kTqD + 4 * ti);
    const float4 x = *reinterpret_cast<const float4*>(X + j * kTok + 4 * tt);
    const float wv[4] = {w.x, w.y, w.z, w.w}, xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(wv[a], xv[b], acc[a][b]);
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
  float* sPiT = reinterpret_cast<float*>(smem + QSmem::PIT);
  float* sST = reinterpret_cast<float*>(smem + QSmem::ST);
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
  __shared__ float s_thr[8], s_lv[8];
  __shared__ uint32_t s_flags;

  const Geom& gm = a.geom;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ti = lane, tt = warp;   // matvec tile: rows 4ti..4ti+3, tokens 4tt..4tt+3

  {
    const uint4* p = reinterpret_cast<const uint4*>(gm.params + kTqPiT);
    uint4* d = reinterpret_cast<uint4*>(sPiT);
    for (int i = tid; i < 2 * kTqD * kTqD / 4; i += kQThreads) d[i] = __ldg(p + i);   // Pi^T then S^T
    if (tid < 8) {
      s_thr[tid] = reinterpret_cast<const float*>(gm.params + kTqThr)[tid];
      s_lv[tid] = reinterpret_cast<const float*>(gm.params + kTqLevels)[tid];
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
        for (int a4 = 0; a4 < 4; ++a4) {
          const float4 y4 = *reinterpret_cast<const float4*>(sU + (4 * ti + a4) * kTok + 4 * tt);
          acc[a4][0] = y4.x;
          acc[a4][1] = y4.y;
          acc[a4][2] = y4.z;
          acc[a4][3] = y4.w;
        }
      } else {
        matvec_tile(sPiT, sU, ti, tt, acc);
      }
      uint8_t* codes = kv == 0 ? sCK : sCV;
      double esq[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float y = acc[i4][b];
          int c = 0;
#pragma unroll
          for (int k = 0; k < 7; ++k) c += y > thr[k] ? 1 : 0;
          const int i = 4 * ti + i4, t = 4 * tt + b;
          codes[t * kTqD + i] = (uint8_t)c;
          if (kv == 0) {
            const float e = y - s_lv[c];
            sE[i * kTok + t] = e;
            esq[b] += (double)e * (double)e;
          }
        }
      if (kv == 0) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const double s = warp_sum_d(esq[b]);
          if (lane == 0) sESQ[4 * tt + b] = s;
        }
        __syncthreads();
        // ---------------------------------------------------------- sketch signs of S e
        matvec_tile(sST, sE, ti, tt, acc);
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4)
#pragma unroll
          for (int b = 0; b < 4; ++b) sSG[(4 * tt + b) * kTqM + 4 * ti + i4] = acc[i4][b] >= 0.f ? 1 : 0;
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
        const __half hg = __double2half(nk * sqrt(sESQ[t]));
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

// TurboQuant-style quantization of 32-token blocks from FP8 window rows (the
// mixed cache's flushes); 16-bit sources go to tq_quantize_tc_kernel
// (tq_quant_tc.cu), which launch_tq_quantize below routes them to.
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
// 1; the zero vector has u = 0.  Codes are decided on y computed to about
// fp32 precision (Pi in fp32 and u, each split into fp16 hi + lo, fp32
// accumulation; below).
//
// One persistent CTA per SM keeps 16 Pi^T and S^T in shared memory as
// mma.sync B fragments, each split into fp16 hi + lo, and runs three (row,
// block) tasks at a time, three warps per task: two take the keys of 16
// tokens each (Pi u, then S e), one the values of all 32 (Pi u).  A warp holds
// its 16 token vectors in registers as A fragments, so the products run
// without CTA-wide barriers; the three warps meet only to pack the block.
// The products are hi*hi + hi*lo + lo*hi with fp32 accumulation (about 22
// significant bits, the dropped lo*lo term below 2^-22 of each product); u is
// scaled by 16 and e by 64 so that the lo parts stay clear of fp16 subnormals.
// A lane loads 8 consecutive coordinates at a time, so the k index of an A
// fragment is a fixed permutation of the coordinates; the B fragments of the
// products over coordinates carry the same permutation.  With the
// Walsh-Hadamard rotation, Pi u is the fast transform in registers (7
// add/sub stages: 5 within a lane, 2 across the lanes of a quad), leaving S e
// as the one product.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kTok = 32;
// row stride of the code and sign tiles in shared memory: 34 words, so the
// byte stores of a C fragment (8 token rows x 4 lane pairs) hit distinct banks
constexpr int kRowS = 136;
constexpr int kQTasks = 2;                       // tasks in flight per CTA
constexpr int kQThreads = kQTasks * 3 * 32;      // three warps per task

struct QSmem {
  // B operands over coordinates, [k-tile 8][n-tile 16][lane 32] x uint4
  // (hi b0, hi b1, lo b0, lo b1)
  static constexpr int BP = 0;                                // 16 Pi^T
  static constexpr int BS = BP + 8 * 16 * 32 * 16;            // S^T
  static constexpr int SLOT = BS + 8 * 16 * 32 * 16;          // per task slot:
  static constexpr int CK = 0;                                //   uint8 [32][kRowS] key codes
  static constexpr int CV = CK + kTok * kRowS;                //   uint8 [32][kRowS] value codes
  static constexpr int SG = CV + kTok * kRowS;                //   uint8 [32][kRowS] sign bits
  static constexpr int NK = SG + kTok * kRowS;                //   double [32] key norms
  static constexpr int NV = NK + kTok * 8;                    //   double [32] value norms
  static constexpr int ESQ = NV + kTok * 8;                   //   double [32] ||e||^2
  static constexpr int SLOT_BYTES = ESQ + kTok * 8;
  static constexpr int BYTES = SLOT + kQTasks * SLOT_BYTES;
};
static_assert(QSmem::BYTES <= 227 * 1024, "TurboQuant quantizer exceeds shared memory");

// coordinate held by position q (0..3) of the (hi | lo) pairs of k-tile kt for
// quad lane tc: k-tile kt = 2v + w covers coordinates 32v + 8tc + 4w + 0..3
__device__ __forceinline__ int perm_coord(int kt, int tc, int q) { return 32 * (kt >> 1) + 8 * tc + 4 * (kt & 1) + q; }

// fp16 hi + lo split of two fp32 values, packed as fp16x2 pairs
__device__ __forceinline__ void split2(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(v0, v1);
  const float2 hf = __half22float2(h);
  hi = h2_as_u32(h);
  lo = h2_as_u32(__floats2half2_rn(v0 - hf.x, v1 - hf.y));
}

// B fragments of W^T (W[i][j] * scale, i = output, j = summed coordinate; W
// row-major, or transposed as W[j][i]) over the summed coordinates, in the
// permuted order (perm) or the natural one.
__device__ __forceinline__ void build_b_frags(const float* W, float scale, bool transposed, bool perm,
                                              unsigned char* dst, int tid) {
  auto w = [&](int i, int j) { return __ldg(transposed ? W + j * kTqD + i : W + i * kTqD + j) * scale; };
  for (int q = tid; q < 8 * 16 * 32; q += kQThreads) {
    const int kt = q >> 9, nt = (q >> 5) & 15, lane = q & 31;
    const int gr = lane >> 2, tc = lane & 3;
    const int i = 8 * nt + gr;
    int j0, j1, j2, j3;
    if (perm) {
      j0 = perm_coord(kt, tc, 0), j1 = j0 + 1, j2 = j0 + 2, j3 = j0 + 3;
    } else {
      j0 = 16 * kt + 2 * tc, j1 = j0 + 1, j2 = j0 + 8, j3 = j0 + 9;
    }
    uint32_t h0, l0, h1, l1;
    split2(w(i, j0), w(i, j1), h0, l0);
    split2(w(i, j2), w(i, j3), h1, l1);
    reinterpret_cast<uint4*>(dst)[q] = make_uint4(h0, h1, l0, l1);
  }
}

// acc[nt] += A(k-tile kt) B(kt, nt) for n-tiles nt0 .. nt0 + NT - 1, as
// hi*hi + hi*lo + lo*hi
template <int NT>
__device__ __forceinline__ void mma3(float (*acc)[4], const uint32_t* ah, const uint32_t* al, const unsigned char* B,
                                     int kt, int nt0, int lane) {
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const uint4 b = reinterpret_cast<const uint4*>(B)[(kt * 16 + nt0 + n) * 32 + lane];
    mma_f16_16816(acc[n], ah, b.x, b.y);
    mma_f16_16816(acc[n], ah, b.z, b.w);
    mma_f16_16816(acc[n], al, b.x, b.y);
  }
}

// Walsh-Hadamard transform (Sylvester order, unnormalised) of the 16-token
// tile in the quad layout: v[r][k] = coordinate 32 (k >> 3) + 8 tc + (k & 7) of
// row r; coordinate bits 0-2 and 5-6 are within a lane, bits 3-4 across the quad.
__device__ __forceinline__ void fwht_quad(float (*v)[32], int tc) {
#pragma unroll
  for (int r = 0; r < 2; ++r) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)          // bits 0-2
#pragma unroll
      for (int k = 0; k < 32; ++k)
        if (!(k & h)) {
          const float a = v[r][k], b = v[r][k + h];
          v[r][k] = a + b;
          v[r][k + h] = a - b;
        }
#pragma unroll
    for (int h = 8; h < 32; h <<= 1)         // bits 5-6
#pragma unroll
      for (int k = 0; k < 32; ++k)
        if (!(k & h)) {
          const float a = v[r][k], b = v[r][k + h];
          v[r][k] = a + b;
          v[r][k + h] = a - b;
        }
#pragma unroll
    for (int m = 1; m < 4; m <<= 1)          // bits 3-4
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float p = __shfl_xor_sync(0xffffffffu, v[r][k], m);
        v[r][k] = (tc & m) ? p - v[r][k] : v[r][k] + p;
      }
  }
}

// The 16 token vectors t0 + gr, t0 + 8 + gr of one kind (key or value) of a
// task into u[2][32] (quad layout) as unit vectors (with wht: y = H u / sqrt(d));
// norms to nrm[token] (lanes tc = 0).  Source: 16-bit rows, or FP8 window rows
// (exact fp32 values e4m3(code) * s).
__device__ __forceinline__ uint32_t load_units(const QuantArgs& a, int row, int blk, int kv, int t0, float (*u)[32],
                                               double* nrm, int gr, int tc) {
  const Geom& gm = a.geom;
  uint32_t flags = 0;
  float x[2][32];
  if (a.src_fp8 == nullptr) {
    const uint16_t* src =
        (kv == 0 ? a.src_k : a.src_v) + (int64_t)row * a.src_row_stride + ((int64_t)blk * kTok + t0) * kTqD;
    uint4 raw[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int v = 0; v < 4; ++v) raw[r][v] = ldg_nc_v4(src + (gr + 8 * r) * kTqD + 32 * v + 8 * tc);
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint32_t wv[4] = {raw[r][v].x, raw[r][v].y, raw[r][v].z, raw[r][v].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          x[r][8 * v + 2 * q] = in16_to_float((uint16_t)(wv[q] & 0xFFFFu), gm.dtype);
          x[r][8 * v + 2 * q + 1] = in16_to_float((uint16_t)(wv[q] >> 16), gm.dtype);
        }
      }
  } else {
    // FP8 window rows (ring layout): x_hat = e4m3(code) * s, exact in fp32
    const unsigned char* src8 = a.src_fp8 + (int64_t)row * 2 * gm.cap * kFp8RowBytes +
                                (int64_t)kv * gm.cap * kFp8RowBytes + ((int64_t)blk * kTok + t0) * kFp8RowBytes;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const unsigned char* rowp = src8 + (gr + 8 * r) * kFp8RowBytes;
      const float sc = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(rowp + kTqD)));
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint2 c8 = *reinterpret_cast<const uint2*>(rowp + 32 * v + 8 * tc);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const unsigned char code = (unsigned char)(((e < 4 ? c8.x : c8.y) >> (8 * (e & 3))) & 0xFFu);
          x[r][8 * v + e] = __half2float(__half(__nv_cvt_fp8_to_halfraw(code, __NV_E4M3))) * sc;
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    double s = 0.0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      if (!isfinite(x[r][k])) flags |= KVQ_DEV_NONFINITE_INPUT;
      s += (double)x[r][k] * (double)x[r][k];
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    const double n = sqrt(s);
    const double inv = n > 0.0 ? 1.0 / n : 0.0;
#pragma unroll
    for (int k = 0; k < 32; ++k) u[r][k] = (float)((double)x[r][k] * inv);
    if (tc == 0) nrm[t0 + gr + 8 * r] = n;
  }
  if (gm.rot_wht) {
    fwht_quad(u, tc);
    const float c = (float)(1.0 / sqrt((double)kTqD));
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int k = 0; k < 32; ++k) u[r][k] *= c;
  }
  return flags;
}

// A fragments (hi, lo) of k-tile kt of the quad-layout tile u * scale
__device__ __forceinline__ void quad_a_frag(const float (*u)[32], int kt, float scale, uint32_t* ah, uint32_t* al) {
  const int v = kt >> 1, w = kt & 1;
  const int k0 = 8 * v + 4 * w;
  split2(u[0][k0] * scale, u[0][k0 + 1] * scale, ah[0], al[0]);
  split2(u[1][k0] * scale, u[1][k0 + 1] * scale, ah[1], al[1]);
  split2(u[0][k0 + 2] * scale, u[0][k0 + 3] * scale, ah[2], al[2]);
  split2(u[1][k0 + 2] * scale, u[1][k0 + 3] * scale, ah[3], al[3]);
}

__device__ __forceinline__ int code_of(float y, const float* thr) {
  int c = 0;
#pragma unroll
  for (int k = 0; k < 7; ++k) c += y > thr[k] ? 1 : 0;
  return c;
}

// One warp: the 16 tokens t0 + gr, t0 + 8 + gr of kind kv of a task: codes to
// codes[token][128], norms; keys also the sketch signs sg[token][128] and
// ||e||^2 to esq[token].
__device__ __forceinline__ uint32_t quantize16(const QuantArgs& a, int row, int blk, int kv, int t0,
                                               const unsigned char* sBP, const unsigned char* sBS, uint8_t* codes,
                                               uint8_t* sg, double* nrm, double* esq, const float* thr,
                                               const float* lv, int lane) {
  const Geom& gm = a.geom;
  const int gr = lane >> 2, tc = lane & 3;
  float u[2][32];
  const uint32_t flags = load_units(a, row, blk, kv, t0, u, nrm, gr, tc);
  const bool key = kv == 0;
  double es[2] = {0.0, 0.0};
  float sacc[16][4];
  if (key) {
#pragma unroll
    for (int n = 0; n < 16; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
  }
  if (gm.rot_wht) {
    // y = u (quad layout): codes, residuals, and the sketch over the permuted k-tiles
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
      float e[2][4];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = 8 * (kt >> 1) + 4 * (kt & 1) + q;
          const float y = u[r][k];
          const int c = code_of(y, thr);
          codes[(t0 + gr + 8 * r) * kRowS + perm_coord(kt, tc, q)] = (uint8_t)c;
          e[r][q] = y - lv[c];
          es[r] += (double)e[r][q] * (double)e[r][q];
        }
      if (key) {
        uint32_t eh[4], el[4];
        split2(e[0][0] * 64.f, e[0][1] * 64.f, eh[0], el[0]);
        split2(e[1][0] * 64.f, e[1][1] * 64.f, eh[1], el[1]);
        split2(e[0][2] * 64.f, e[0][3] * 64.f, eh[2], el[2]);
        split2(e[1][2] * 64.f, e[1][3] * 64.f, eh[3], el[3]);
        mma3<16>(sacc, eh, el, sBS, kt, 0, lane);
      }
    }
  } else {
    uint32_t ah[8][4], al[8][4];
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) quad_a_frag(u, kt, 16.f, ah[kt], al[kt]);
    // y = Pi u, four n-tiles (two k-tiles of the sketch) at a time
#pragma unroll 1
    for (int g4 = 0; g4 < 4; ++g4) {
      float acc[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
      for (int kt = 0; kt < 8; ++kt) mma3<4>(acc, ah[kt], al[kt], sBP, kt, 4 * g4, lane);
      float e[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float y = acc[n][q] * (1.f / 256.f);
          const int c = code_of(y, thr);
          const int r = q >> 1, i = 8 * (4 * g4 + n) + 2 * tc + (q & 1);
          codes[(t0 + gr + 8 * r) * kRowS + i] = (uint8_t)c;
          e[n][q] = y - lv[c];
          es[r] += (double)e[n][q] * (double)e[n][q];
        }
      if (key) {
        // C fragments of n-tiles 2m, 2m + 1 = A fragment of sketch k-tile 2 g4 + m
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          uint32_t eh[4], el[4];
          split2(e[2 * m][0] * 64.f, e[2 * m][1] * 64.f, eh[0], el[0]);
          split2(e[2 * m][2] * 64.f, e[2 * m][3] * 64.f, eh[1], el[1]);
          split2(e[2 * m + 1][0] * 64.f, e[2 * m + 1][1] * 64.f, eh[2], el[2]);
          split2(e[2 * m + 1][2] * 64.f, e[2 * m + 1][3] * 64.f, eh[3], el[3]);
          mma3<16>(sacc, eh, el, sBS, 2 * g4 + m, 0, lane);
        }
      }
    }
  }
  if (key) {
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        sg[(t0 + gr + 8 * (q >> 1)) * kRowS + 8 * n + 2 * tc + (q & 1)] = sacc[n][q] >= 0.f ? 1 : 0;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      double s = es[r];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (tc == 0) esq[t0 + gr + 8 * r] = s;
    }
  }
  return flags;
}


// named barrier (1 + slot) over the three warps of a task slot
__device__ __forceinline__ void task_bar(int slot) { asm volatile("bar.sync %0, 96;\n" ::"r"(1 + slot) : "memory"); }

__global__ void __launch_bounds__(kQThreads, 1) tq_quantize_kernel(QuantArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float s_thr[8], s_lv[8];
  __shared__ uint32_t s_flags;

  const Geom& gm = a.geom;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot = warp / 3, role = warp - 3 * slot;   // role 0, 1: keys of tokens 0-15, 16-31; 2: values
  const int stid = tid - 96 * slot;                     // thread rank within the task's three warps
  unsigned char* sl = smem + QSmem::SLOT + slot * QSmem::SLOT_BYTES;
  uint8_t* sCK = sl + QSmem::CK;
  uint8_t* sCV = sl + QSmem::CV;
  uint8_t* sSG = sl + QSmem::SG;
  double* sNK = reinterpret_cast<double*>(sl + QSmem::NK);
  double* sNV = reinterpret_cast<double*>(sl + QSmem::NV);
  double* sESQ = reinterpret_cast<double*>(sl + QSmem::ESQ);

  {
    const float* P = reinterpret_cast<const float*>(gm.params);
    if (!gm.rot_wht) build_b_frags(P + kTqPi / 4, 16.f, false, true, smem + QSmem::BP, tid);
    // sketch over coordinates of y: quad layout (wht) or C-fragment layout (Pi product)
    build_b_frags(P + kTqST / 4, 1.f, true, gm.rot_wht != 0, smem + QSmem::BS, tid);
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
  for (int64_t task = (int64_t)blockIdx.x * kQTasks + slot; task < n_tasks; task += (int64_t)gridDim.x * kQTasks) {
    const int row = (int)(task / a.n_groups);
    const int blk = (int)(task - (int64_t)row * a.n_groups);
    // one call site (the code is large: an instruction-fetch-bound kernel otherwise)
#pragma unroll 1
    for (int h = 0; h < (role < 2 ? 1 : 2); ++h) {
      const bool key = role < 2;
      flags |= quantize16(a, row, blk, key ? 0 : 1, key ? 16 * role : 16 * h, smem + QSmem::BP, smem + QSmem::BS,
                          key ? sCK : sCV, sSG, key ? sNK : sNV, sESQ, thr, s_lv, lane);
    }
    task_bar(slot);

    // ---------------------------------------------------------- pack and store the token block
    uint32_t* dst = reinterpret_cast<uint32_t*>(record_ptr(gm, row, a.dst_group0 + blk));
    if (dst == nullptr) flags |= KVQ_DEV_BAD_PAGE;   // page outside the pool: nothing is written
    for (int qw = dst != nullptr ? stid : 2 * 416 + 128 + 32; qw < 2 * 416 + 128 + 32; qw += 96) {
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
              idx = sCK[t * kRowS + c0] + 8u * sCK[t * kRowS + c0 + 1];
            } else {
              const int kt = slot >> 5, nt = (slot >> 1) & 15, rho = slot & 1;
              const int c = 8 * nt + gr, t0 = 16 * kt + 8 * rho + 2 * tc;
              idx = sCV[t0 * kRowS + c] + 8u * sCV[(t0 + 1) * kRowS + c];
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
          word |= (uint32_t)sSG[t * kRowS + i0] << s;
          word |= (uint32_t)sSG[t * kRowS + i0 + 1] << (16 + s);
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
    task_bar(slot);   // the slot is packed before its next task writes it
  }
  if (flags) atomicOr(&s_flags, flags);
  __syncthreads();
  if (tid == 0 && s_flags) atomicOr(gm.status, s_flags);
}

}  // namespace

void launch_tq_quantize(const QuantArgs& a, cudaStream_t st) {
  const int64_t tasks = (int64_t)a.geom.B * a.geom.Hkv * a.n_groups;
  if (tasks <= 0) return;
  if (a.src_fp8 == nullptr) {   // 16-bit rows, either rotation (Pi as a dense table): the tensor-core kernel
    launch_tq_quantize_tc(a, st);
    return;
  }
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(tq_quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, QSmem::BYTES);
    attr_set = true;
  }
  const int64_t ctas = (tasks + kQTasks - 1) / kQTasks;
  const int grid = (int)(ctas < num_sms() ? ctas : num_sms());
  tq_quantize_kernel<<<grid, kQThreads, QSmem::BYTES, st>>>(a);
  count_launch(1);
}

}  // namespace kvq

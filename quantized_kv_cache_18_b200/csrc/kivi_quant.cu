// KIVI quantization kernels: prefill, window flush, window writes.
//
// Keys are quantized per channel over groups of G tokens and values per token
// over the head's d channels, each with an fp16 scale s = (max - min) /
// (2^b - 1) and zero-point z = min ("Quantification du KV-Cache : TurboQuant et
// l'etat de l'art en 2026", section "KIVI (2024)"; zubnet.ai survey, "Famille
// deux, c'est la quantification").  Codes are packed 16 INT2 or 8 INT4 per
// 32-bit word ("TurboQuant : les cinq innovations", item 3) in the v1 order
// described in kvq_internal.cuh.
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kQuantThreads = 128;

__device__ __forceinline__ void flag_status(uint32_t* status, uint32_t bits) {
  if (bits) atomicOr(status, bits);
}

// One CTA quantizes one group record (G tokens of one row).
template <int BITS, int D, int G>
__global__ void __launch_bounds__(kQuantThreads) kivi_quantize_kernel(QuantArgs a) {
  constexpr int LEVELS = (1 << BITS) - 1;
  constexpr int NTB = G / kTB;
  constexpr int P = D * BITS / 32;              // words per lane per TB
  constexpr int PAIRS = 16 / BITS;              // pairs per word
  constexpr int J = BITS == 2 ? 4 : 2;          // pairs per half word
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* sk = reinterpret_cast<uint16_t*>(smem);            // [G][D]
  uint16_t* sv = sk + G * D;                                   // [G][D]
  uint8_t* ck = reinterpret_cast<uint8_t*>(sv + G * D);        // [G][D]
  uint8_t* cv = ck + G * D;                                    // [G][D]
  __shared__ double k_s[D], k_z[D], k_inv[D];
  __shared__ double v_s[G], v_z[G], v_inv[G];
  __shared__ uint16_t k_sb[D], k_zb[D], v_sb[G], v_zb[G];
  __shared__ uint32_t s_flags;

  const Geom& gm = a.geom;
  const int row = blockIdx.y;
  const int grp = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0) s_flags = 0;

  // 1. stage the key and value tiles
  const uint16_t* gk = a.src_k + (int64_t)row * a.src_row_stride + (int64_t)grp * G * D;
  const uint16_t* gv = a.src_v + (int64_t)row * a.src_row_stride + (int64_t)grp * G * D;
  for (int i = tid; i < G * D / 8; i += kQuantThreads) {
    reinterpret_cast<uint4*>(sk)[i] = ldg_nc_v4(reinterpret_cast<const uint4*>(gk) + i);
    reinterpret_cast<uint4*>(sv)[i] = ldg_nc_v4(reinterpret_cast<const uint4*>(gv) + i);
  }
  __syncthreads();

  uint32_t flags = 0;
  // 2. key parameters, one channel per thread
  for (int c = tid; c < D; c += kQuantThreads) {
    float mn = in16_to_float(sk[c], gm.dtype), mx = mn;
    bool fin = isfinite(mn);
    for (int t = 1; t < G; ++t) {
      const float x = in16_to_float(sk[t * D + c], gm.dtype);
      fin &= isfinite(x);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    const double range = (double)mx - (double)mn;
    const __half hs = __double2half(range / (double)LEVELS);
    const __half hz = __double2half((double)mn);
    const double s = (double)__half2float(hs), z = (double)__half2float(hz);
    if (!fin) flags |= KVQ_DEV_NONFINITE_INPUT;
    if (!isfinite(s) || !isfinite(z)) flags |= KVQ_DEV_PARAM_OVERFLOW;
    k_s[c] = s;
    k_z[c] = z;
    k_inv[c] = s > 0.0 ? 1.0 / s : 0.0;
    k_sb[c] = __half_as_ushort(hs);
    k_zb[c] = __half_as_ushort(hz);
  }
  // 3. value parameters, one token per warp
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int t = warp; t < G; t += kQuantThreads / 32) {
      float mn = INFINITY, mx = -INFINITY;
      bool fin = true;
      for (int c = lane; c < D; c += 32) {
        const float x = in16_to_float(sv[t * D + c], gm.dtype);
        fin &= isfinite(x);
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      fin = __all_sync(0xffffffffu, fin);
      if (lane == 0) {
        const __half hs = __double2half(((double)mx - (double)mn) / (double)LEVELS);
        const __half hz = __double2half((double)mn);
        const double s = (double)__half2float(hs), z = (double)__half2float(hz);
        if (!fin) flags |= KVQ_DEV_NONFINITE_INPUT;
        if (!isfinite(s) || !isfinite(z)) flags |= KVQ_DEV_PARAM_OVERFLOW;
        v_s[t] = s;
        v_z[t] = z;
        v_inv[t] = s > 0.0 ? 1.0 / s : 0.0;
        v_sb[t] = __half_as_ushort(hs);
        v_zb[t] = __half_as_ushort(hz);
      }
    }
  }
  __syncthreads();

  // 4. codes
  for (int i = tid; i < G * D; i += kQuantThreads) {
    const int t = i / D, c = i - t * D;
    const double xk = (double)in16_to_float(sk[i], gm.dtype);
    const double xv = (double)in16_to_float(sv[i], gm.dtype);
    ck[i] = (uint8_t)exact_code(xk, k_z[c], k_s[c], k_inv[c], LEVELS);
    cv[i] = (uint8_t)exact_code(xv, v_z[t], v_s[t], v_inv[t], LEVELS);
  }
  __syncthreads();

  // 5. pack: one 16-byte piece (4 words of one lane) per iteration
  char* rec = record_ptr(gm, row, a.dst_group0 + grp);
  constexpr int PIECES = NTB * 32 * (P / 4);   // per key (or value) part
  for (int i = tid; i < 2 * PIECES; i += kQuantThreads) {
    const bool is_v = i >= PIECES;
    const int pi = is_v ? i - PIECES : i;
    const int tb = pi / (32 * (P / 4));
    const int rem = pi - tb * 32 * (P / 4);
    const int p = rem / 32, lane = rem & 31;
    const int gr = lane >> 2, tc = lane & 3;
    const uint8_t* cc = (is_v ? cv : ck) + tb * kTB * D;
    uint32_t wv[4];
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
      const int w = 4 * p + e4;
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < PAIRS; ++j) {
        const int half = j / J, jp = j % J;
        const int slot = 2 * w + half;
        int t0, c0, dt, dc;   // first code's (token, channel) and the step to the second
        if (!is_v) {
          constexpr int SPN = BITS == 2 ? D / 32 : D / 16;   // slots per key n-tile
          const int nt = slot / SPN;
          const int u = BITS == 2 ? 4 * (slot % SPN) + jp : 2 * (slot % SPN) + jp;
          const int kt = u >> 1, rho = u & 1;
          t0 = 8 * nt + gr;
          c0 = 16 * kt + 8 * rho + 2 * tc;
          dt = 0;
          dc = 1;
        } else {
          int nt, u;
          if (BITS == 2) {
            nt = slot;
            u = jp;
          } else {
            nt = slot >> 1;
            u = 2 * (slot & 1) + jp;
          }
          const int kt = u >> 1, rho = u & 1;
          c0 = 8 * nt + gr;
          t0 = 16 * kt + 8 * rho + 2 * tc;
          dt = 1;
          dc = 0;
        }
        const uint32_t lo = cc[t0 * D + c0];
        const uint32_t hi = cc[(t0 + dt) * D + c0 + dc];
        word |= (lo << (BITS * j)) | (hi << (16 + BITS * j));
      }
      wv[e4] = word;
    }
    char* dst = rec + (is_v ? (NTB + tb) : tb) * (int64_t)(kTB * D * BITS / 8) + 16 * (32 * p + lane);
    *reinterpret_cast<uint4*>(dst) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }

  // 6. metadata
  uint16_t* ksc = reinterpret_cast<uint16_t*>(rec + rec_kscale_off(gm));
  uint16_t* kzr = reinterpret_cast<uint16_t*>(rec + rec_kzero_off(gm));
  for (int c = tid; c < D; c += kQuantThreads) {
    const int kt = c >> 4, rho = (c >> 3) & 1, tc = (c >> 1) & 3, e = c & 1;
    const int pos = 8 * (4 * (kt >> 1) + tc) + 4 * (kt & 1) + 2 * rho + e;
    ksc[pos] = k_sb[c];
    kzr[pos] = k_zb[c];
  }
  uint32_t* vm = reinterpret_cast<uint32_t*>(rec + rec_vmeta_off(gm));
  for (int t = tid; t < G; t += kQuantThreads) {
    const int tb = t / kTB, tt = t % kTB;
    const int kt = tt >> 4, rho = (tt >> 3) & 1, tc = (tt >> 1) & 3, e = tt & 1;
    vm[tb * kTB + 8 * tc + 4 * kt + 2 * rho + e] = (uint32_t)v_sb[t] | ((uint32_t)v_zb[t] << 16);
  }

  if (flags) atomicOr(&s_flags, flags);
  __syncthreads();
  if (tid == 0) flag_status(gm.status, s_flags);
}

// Copies window tokens [t0, t0 + n) of every row of a [B][Hkv][S][d] input into
// ring slots [0, n).
__global__ void window_copy_kernel(Geom g, const uint16_t* k, const uint16_t* v, int64_t seq_len, int64_t t0,
                                   int n) {
  const int row = blockIdx.y;
  const int64_t chunks = (int64_t)n * g.d / 8;
  const uint4* sk = reinterpret_cast<const uint4*>(k + ((int64_t)row * seq_len + t0) * g.d);
  const uint4* svv = reinterpret_cast<const uint4*>(v + ((int64_t)row * seq_len + t0) * g.d);
  uint4* dk = reinterpret_cast<uint4*>(ring_ptr(g, row, 0));
  uint4* dv = reinterpret_cast<uint4*>(ring_ptr(g, row, 1));
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += (int64_t)gridDim.x * blockDim.x) {
    dk[i] = ldg_nc_v4(sk + i);
    dv[i] = ldg_nc_v4(svv + i);
  }
}

// Writes one new token per row into ring slot `slot`.
__global__ void append_kernel(Geom g, const uint16_t* k, const uint16_t* v, int slot) {
  const int row = blockIdx.x;
  const int i = threadIdx.x;   // 16-byte chunk
  if (i < g.d / 8) {
    const uint4* sk = reinterpret_cast<const uint4*>(k + (int64_t)row * g.d);
    const uint4* svv = reinterpret_cast<const uint4*>(v + (int64_t)row * g.d);
    reinterpret_cast<uint4*>(ring_ptr(g, row, 0) + (int64_t)slot * g.d)[i] = sk[i];
    reinterpret_cast<uint4*>(ring_ptr(g, row, 1) + (int64_t)slot * g.d)[i] = svv[i];
  }
}

__global__ void clear_words_kernel(uint32_t* words, int n) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) words[i] = 0u;
}

template <int BITS, int D, int G>
void launch_q(const QuantArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)G * D * (2 + 2 + 1 + 1);
  auto kern = kivi_quantize_kernel<BITS, D, G>;
  static bool attr_set = false;   // per template instance; the attribute is per device function
  if (!attr_set) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attr_set = true;
  }
  dim3 grid(a.n_groups, a.geom.B * a.geom.Hkv);
  kern<<<grid, kQuantThreads, smem, st>>>(a);
}

}  // namespace

void launch_kivi_quantize(const QuantArgs& a, cudaStream_t st) {
  if (a.n_groups <= 0) return;
  const Geom& g = a.geom;
  if (g.bits == 2 && g.d == 128 && g.G == 32) launch_q<2, 128, 32>(a, st);
  else if (g.bits == 2 && g.d == 64 && g.G == 32) launch_q<2, 64, 32>(a, st);
  else if (g.bits == 4 && g.d == 128 && g.G == 64) launch_q<4, 128, 64>(a, st);
  else if (g.bits == 4 && g.d == 128 && g.G == 32) launch_q<4, 128, 32>(a, st);
  else if (g.bits == 2 && g.d == 128 && g.G == 64) launch_q<2, 128, 64>(a, st);
  else if (g.bits == 4 && g.d == 64 && g.G == 32) launch_q<4, 64, 32>(a, st);
  else if (g.bits == 2 && g.d == 64 && g.G == 64) launch_q<2, 64, 64>(a, st);
  else if (g.bits == 4 && g.d == 64 && g.G == 64) launch_q<4, 64, 64>(a, st);
  else return;
  count_launch();
}

void launch_window_copy(const Geom& g, const uint16_t* k, const uint16_t* v, int64_t seq_len, int64_t t0, int n,
                        cudaStream_t st) {
  if (n <= 0) return;
  const int64_t chunks = (int64_t)n * g.d / 8;
  const int bx = (int)((chunks + 255) / 256);
  window_copy_kernel<<<dim3(bx, g.B * g.Hkv), 256, 0, st>>>(g, k, v, seq_len, t0, n);
  count_launch();
}

void launch_append(const Geom& g, const uint16_t* k, const uint16_t* v, int slot, cudaStream_t st) {
  append_kernel<<<g.B * g.Hkv, 32, 0, st>>>(g, k, v, slot);
  count_launch();
}

void launch_clear_words(uint32_t* words, int n, cudaStream_t st) {
  clear_words_kernel<<<1, 256, 0, st>>>(words, n);
  count_launch();
}

}  // namespace kvq

// KIVI quantization kernels: prefill, window flush, window writes.
//
// Keys are quantized per channel over groups of G tokens and values per token
// over the head's d channels, each with an fp16 scale s = (max - min) /
// (2^b - 1) and zero-point z = min ("Quantification du KV-Cache : TurboQuant et
// l'etat de l'art en 2026", section "KIVI (2024)"; zubnet.ai survey, "Famille
// deux, c'est la quantification").  Codes are packed 16 INT2 or 8 INT4 per
// 32-bit word ("TurboQuant : les cinq innovations", item 3) in the fragment
// order described in kvq_internal.cuh.
//
// A CTA handles one group record in four passes over shared memory: stage the
// key and value tiles, reduce the parameters (key and value warps side by
// side), decide the codes (a thread keeps one channel pair's or one token
// pair's parameters in registers), pack 16-byte pieces of the record.
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kQuantThreads = 128;

__device__ __forceinline__ void flag_status(uint32_t* status, uint32_t bits) {
  if (bits) atomicOr(status, bits);
}

// Codes are round half to even of (x - z) / s, clamped to [0, levels], with
// s, z the fp16 scale and zero-point.  The fp32 estimate r = fma(x, 1/s, -z/s)
// differs from the exact quotient by less than 2^-24 (2 levels + |z| / s) up to
// second-order terms (one rounding each in 1/s, z/s and the fma; r is only used
// where it lies in [0, levels]); eb below is four times that.  An estimate more
// than eb away from every rounding boundary k + 1/2 decides.  Within eb, which
// takes in the exact ties that 16-bit inputs and fp16 scales often produce, the
// exact double-precision comparison of 2 (x - z) with (2k + 1) s decides.
struct CodeParams {
  float s, z, inv, zinv, eb;
};
__device__ __forceinline__ CodeParams code_params(float s, float z, int levels) {
  CodeParams p;
  p.s = s;
  p.z = z;
  p.inv = s > 0.f ? 1.f / s : 0.f;
  p.zinv = z * p.inv;
  p.eb = 2.384185791015625e-7f * (2.f * (float)levels + 2.f + fabsf(p.zinv));   // 2^-22 (...)
  return p;
}
// The exact decision, out of line: it runs for a small fraction of the
// elements, and inlining it at every call site bloated the kernel's code
// (instruction-cache misses were its top stall).
__device__ __noinline__ uint32_t code_exact(float x, float z, float s, int levels) {
  return (uint32_t)exact_code((double)x, (double)z, (double)s, s > 0.f ? 1.0 / (double)s : 0.0, levels);
}
__device__ __forceinline__ uint32_t code_of(float x, const CodeParams& p, int levels) {
  float r = fmaf(x, p.inv, -p.zinv);
  r = fminf(fmaxf(r, 0.f), (float)levels);   // also maps NaN to 0
  const float k = rintf(r);
  if (fabsf(fabsf(r - k) - 0.5f) > p.eb) return (uint32_t)k;
  return code_exact(x, p.z, p.s, levels);
}

template <bool BF>
__device__ __forceinline__ float in16f(uint16_t bits) {
  return BF ? __uint_as_float((uint32_t)bits << 16) : __half2float(__ushort_as_half(bits));
}

// One CTA quantizes one group record (G tokens of one row); BF: bf16 inputs
// (else fp16).
template <int BITS, int D, int G, bool BF>
__global__ void __launch_bounds__(kQuantThreads) kivi_quantize_kernel(QuantArgs a) {
  constexpr int LEVELS = (1 << BITS) - 1;
  constexpr int NTB = G / kTB;
  constexpr int P = D * BITS / 32;              // words per lane per TB
  constexpr int PAIRS = 16 / BITS;              // pairs per word
  constexpr int J = BITS == 2 ? 4 : 2;          // pairs per half word
  constexpr int PITCH = D + 8;                  // staged row pitch (halves): rows 8 apart land 4 banks apart
  // key codes: thread = (channel pair, token range); value codes: thread = (token pair, channel range)
  constexpr int KCP = D / 2, KTR = kQuantThreads / KCP, KTOK = G / KTR;
  constexpr int VTP = G / 2, VCR = kQuantThreads / VTP, VCH = D / VCR;
  static_assert(kQuantThreads % KCP == 0 && G % KTR == 0, "key code split");
  static_assert(kQuantThreads % VTP == 0 && D % VCR == 0 && VCH % 8 == 0, "value code split");
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* sk = reinterpret_cast<uint16_t*>(smem);            // [G][PITCH] staged keys
  uint16_t* sv = sk + G * PITCH;                               // [G][PITCH] staged values
  uint8_t* ck = reinterpret_cast<uint8_t*>(sv + G * PITCH);    // [G][D] key codes
  uint8_t* cvt = ck + G * D;                                   // [D][G] value codes (channel-major)
  __shared__ float k_s[D], k_z[D];
  __shared__ float v_s[G], v_z[G];
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
    const int t = i / (D / 8), c8 = i - t * (D / 8);
    *reinterpret_cast<uint4*>(sk + t * PITCH + 8 * c8) = ldg_nc_v4(reinterpret_cast<const uint4*>(gk) + i);
    *reinterpret_cast<uint4*>(sv + t * PITCH + 8 * c8) = ldg_nc_v4(reinterpret_cast<const uint4*>(gv) + i);
  }
  __syncthreads();

  uint32_t flags = 0;
  // 2. parameters.  Warps 0-1: keys, one channel pair per thread over the G
  // tokens; warps 2-3: values, one token per warp at a time.  An input that is
  // inf or NaN turns the running fma(x, 0, .) into NaN.
  static_assert(D / 2 <= 64, "key parameter split");
  if (tid < 64) {
    for (int cp = tid; cp < D / 2; cp += 64) {
      const int c = 2 * cp;
      float mn0 = INFINITY, mx0 = -INFINITY, mn1 = INFINITY, mx1 = -INFINITY, nf = 0.f;
#pragma unroll 8
      for (int t = 0; t < G; ++t) {
        const uint32_t x2 = *reinterpret_cast<const uint32_t*>(sk + t * PITCH + c);
        const float x0 = in16f<BF>((uint16_t)(x2 & 0xFFFFu)), x1 = in16f<BF>((uint16_t)(x2 >> 16));
        nf = fmaf(x0, 0.f, fmaf(x1, 0.f, nf));
        mn0 = fminf(mn0, x0);
        mx0 = fmaxf(mx0, x0);
        mn1 = fminf(mn1, x1);
        mx1 = fmaxf(mx1, x1);
      }
      if (nf != 0.f) flags |= KVQ_DEV_NONFINITE_INPUT;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float mn = e ? mn1 : mn0, mx = e ? mx1 : mx0;
        const __half hs = __double2half(((double)mx - (double)mn) / (double)LEVELS);
        const __half hz = __double2half((double)mn);
        const float sc = __half2float(hs), z = __half2float(hz);
        if (!isfinite(sc) || !isfinite(z)) flags |= KVQ_DEV_PARAM_OVERFLOW;
        k_s[c + e] = sc;
        k_z[c + e] = z;
        k_sb[c + e] = __half_as_ushort(hs);
        k_zb[c + e] = __half_as_ushort(hz);
      }
    }
  } else {
    // one token per step; lane k keeps step k's extremes, so the fp64
    // parameter arithmetic runs on one lane per token at the end
    const int warp = (tid >> 5) - 2, lane = tid & 31;
    float my_mn = 0.f, my_mx = 0.f;
    int my_t = -1;
    static_assert(G / 2 <= 32, "value parameter split");
    for (int t = warp, k = 0; t < G; t += 2, ++k) {
      float mn = INFINITY, mx = -INFINITY, nf = 0.f;
#pragma unroll
      for (int c2 = lane; c2 < D / 2; c2 += 32) {
        const uint32_t x2 = *reinterpret_cast<const uint32_t*>(sv + t * PITCH + 2 * c2);
        const float x0 = in16f<BF>((uint16_t)(x2 & 0xFFFFu)), x1 = in16f<BF>((uint16_t)(x2 >> 16));
        nf = fmaf(x0, 0.f, fmaf(x1, 0.f, nf));
        mn = fminf(mn, fminf(x0, x1));
        mx = fmaxf(mx, fmaxf(x0, x1));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (__any_sync(0xffffffffu, nf != 0.f)) flags |= KVQ_DEV_NONFINITE_INPUT;
      if (lane == k) {
        my_mn = mn;
        my_mx = mx;
        my_t = t;
      }
    }
    if (my_t >= 0) {
      const __half hs = __double2half(((double)my_mx - (double)my_mn) / (double)LEVELS);
      const __half hz = __double2half((double)my_mn);
      const float sc = __half2float(hs), z = __half2float(hz);
      if (!isfinite(sc) || !isfinite(z)) flags |= KVQ_DEV_PARAM_OVERFLOW;
      v_s[my_t] = sc;
      v_z[my_t] = z;
      v_sb[my_t] = __half_as_ushort(hs);
      v_zb[my_t] = __half_as_ushort(hz);
    }
  }
  __syncthreads();

  // 4. codes.  Keys: channels (2 cp, 2 cp + 1) of tokens [tr * KTOK, +KTOK);
  // the two codes of a token land side by side in ck.
  {
    const int cp = tid % KCP, tr = tid / KCP;
    const int c = 2 * cp;
    const CodeParams p0 = code_params(k_s[c], k_z[c], LEVELS), p1 = code_params(k_s[c + 1], k_z[c + 1], LEVELS);
#pragma unroll 4
    for (int t = tr * KTOK; t < (tr + 1) * KTOK; ++t) {
      const uint32_t x2 = *reinterpret_cast<const uint32_t*>(sk + t * PITCH + c);
      const uint32_t q0 = code_of(in16f<BF>((uint16_t)(x2 & 0xFFFFu)), p0, LEVELS);
      const uint32_t q1 = code_of(in16f<BF>((uint16_t)(x2 >> 16)), p1, LEVELS);
      *reinterpret_cast<uint16_t*>(ck + t * D + c) = (uint16_t)(q0 | (q1 << 8));
    }
  }
  // Values: tokens (2 tp, 2 tp + 1), channels [cr * VCH, +VCH); the two codes of
  // a channel land side by side in the channel-major cvt.
  {
    const int tp = tid % VTP, cr = tid / VTP;
    const int t = 2 * tp;
    const CodeParams p0 = code_params(v_s[t], v_z[t], LEVELS), p1 = code_params(v_s[t + 1], v_z[t + 1], LEVELS);
#pragma unroll 2
    for (int c8 = cr * VCH; c8 < (cr + 1) * VCH; c8 += 8) {
      const uint4 x0 = *reinterpret_cast<const uint4*>(sv + t * PITCH + c8);
      const uint4 x1 = *reinterpret_cast<const uint4*>(sv + (t + 1) * PITCH + c8);
      const uint32_t w0[4] = {x0.x, x0.y, x0.z, x0.w}, w1[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint16_t h0 = (uint16_t)(w0[e >> 1] >> (16 * (e & 1))), h1 = (uint16_t)(w1[e >> 1] >> (16 * (e & 1)));
        const uint32_t q0 = code_of(in16f<BF>(h0), p0, LEVELS);
        const uint32_t q1 = code_of(in16f<BF>(h1), p1, LEVELS);
        *reinterpret_cast<uint16_t*>(cvt + (c8 + e) * G + t) = (uint16_t)(q0 | (q1 << 8));
      }
    }
  }
  __syncthreads();

  // 5. packing: one 16-byte piece (4 words of one lane) per iteration; a pair
  // is the codes of two adjacent channels of a token (keys) or of two adjacent
  // tokens of a channel (values), one 16-bit load either way
  char* rec = record_ptr(gm, row, a.dst_group0 + grp);
  if (rec == nullptr) flags |= KVQ_DEV_BAD_PAGE;   // page outside the pool: nothing is written
  constexpr int PIECES = NTB * 32 * (P / 4);   // per key (or value) part
  for (int i = rec != nullptr ? tid : 2 * PIECES; i < 2 * PIECES; i += kQuantThreads) {
    const bool is_v = i >= PIECES;
    const int pi = is_v ? i - PIECES : i;
    const int tb = pi / (32 * (P / 4));
    const int rem = pi - tb * 32 * (P / 4);
    const int p = rem / 32, lane = rem & 31;
    const int gr = lane >> 2, tc = lane & 3;
    uint32_t wv[4];
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
      const int w = 4 * p + e4;
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < PAIRS; ++j) {
        const int half = j / J, jp = j % J;
        const int slot = 2 * w + half;
        uint32_t pr;
        if (!is_v) {
          constexpr int SPN = BITS == 2 ? D / 32 : D / 16;   // slots per key n-tile
          const int nt = slot / SPN;
          const int u = BITS == 2 ? 4 * (slot % SPN) + jp : 2 * (slot % SPN) + jp;
          const int kt = u >> 1, rho = u & 1;
          pr = *reinterpret_cast<const uint16_t*>(ck + (tb * kTB + 8 * nt + gr) * D + 16 * kt + 8 * rho + 2 * tc);
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
          pr = *reinterpret_cast<const uint16_t*>(cvt + (8 * nt + gr) * G + tb * kTB + 16 * kt + 8 * rho + 2 * tc);
        }
        // pr = lo | hi << 8  ->  lo at bit b j, hi at bit 16 + b j
        word |= ((pr | (pr << 8)) & 0x00FF00FFu) << (BITS * j);
      }
      wv[e4] = word;
    }
    char* dst = rec + (is_v ? (NTB + tb) : tb) * (int64_t)(kTB * D * BITS / 8) + 16 * (32 * p + lane);
    *reinterpret_cast<uint4*>(dst) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }

  // 6. metadata
  uint16_t* ksc = reinterpret_cast<uint16_t*>(rec + rec_kscale_off(gm));
  uint16_t* kzr = reinterpret_cast<uint16_t*>(rec + rec_kzero_off(gm));
  for (int c = rec != nullptr ? tid : D; c < D; c += kQuantThreads) {
    const int kt = c >> 4, rho = (c >> 3) & 1, tc = (c >> 1) & 3, e = c & 1;
    const int pos = 8 * (4 * (kt >> 1) + tc) + 4 * (kt & 1) + 2 * rho + e;
    ksc[pos] = k_sb[c];
    kzr[pos] = k_zb[c];
  }
  uint32_t* vm = reinterpret_cast<uint32_t*>(rec + rec_vmeta_off(gm));
  for (int t = rec != nullptr ? tid : G; t < G; t += kQuantThreads) {
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

template <int BITS, int D, int G, bool BF>
void launch_q_dtype(const QuantArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)G * (D + 8) * 2 * 2 + (size_t)G * D * 2;
  auto kern = kivi_quantize_kernel<BITS, D, G, BF>;
  static bool attr_set = false;   // per template instance; the attribute is per device function
  if (!attr_set) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attr_set = true;
  }
  dim3 grid(a.n_groups, a.geom.B * a.geom.Hkv);
  kern<<<grid, kQuantThreads, smem, st>>>(a);
}
template <int BITS, int D, int G>
void launch_q(const QuantArgs& a, cudaStream_t st) {
  if (a.geom.dtype == KVQ_BF16) launch_q_dtype<BITS, D, G, true>(a, st);
  else launch_q_dtype<BITS, D, G, false>(a, st);
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

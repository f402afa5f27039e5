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

#include "decode_common.cuh"
#include "kvq_internal.cuh"

namespace kvq {

namespace {

// Threads of a quantizer CTA: 128 (key warps 0-1, value warps 2-3), or 256
// for 4-bit records of 64 tokens and d = 128, whose longer code phase is split
// over four key and four value warps.
template <int BITS, int D, int G>
__host__ __device__ constexpr int quant_threads() { return BITS == 4 && D == 128 && G == 64 ? 256 : 128; }

// Barrier of one half of the CTA (the key half or the value half): from the
// parameters to the codes neither half reads what the other writes.
template <int NT>
__device__ __forceinline__ void half_bar_sync(bool value_half) {
  if (value_half) asm volatile("bar.sync 2, %0;\n" ::"n"(NT / 2) : "memory");
  else asm volatile("bar.sync 1, %0;\n" ::"n"(NT / 2) : "memory");
}

__device__ __forceinline__ void flag_status(uint32_t* status, uint32_t bits) {
  if (bits) atomicOr(status, bits);
}

// Codes are round half to even of (x - z) / s, clamped to [0, levels], with
// s, z the fp16 scale and zero-point.  4-bit codes start from the fp32
// estimate r = fma(x, 1/s, -z/s), which differs from the exact quotient by less
// than 2^-24 (2 levels + |z| / s) up to second-order terms (one rounding each
// in 1/s, z/s and the fma); eb = 4 times that.  An estimate more than eb away
// from every rounding boundary k + 1/2 decides.  Within eb, which takes in the
// exact ties that 16-bit inputs and fp16 scales often produce, the exact
// double-precision comparison of 2 (x - z) with (2k + 1) s decides.  (2-bit
// codes are decided exactly by 16-bit thresholds, below.)
//
// The exact decision, out of line: it runs for a small fraction of the
// elements, and inlining it at every call site bloated the kernel's code
// (instruction-cache misses were its top stall).
__device__ __noinline__ uint32_t code_exact(float x, float z, float s, int levels) {
  return (uint32_t)exact_code((double)x, (double)z, (double)s, s > 0.f ? 1.0 / (double)s : 0.0, levels);
}

// ------------------------------------------------------------------ per-unit parameters
// A unit is one key channel of the group or one value token.  mn and mx are its
// extremes as floats (exact); mx propagates a nan input.
template <int BITS, bool BF>
struct UnitOut {
  uint16_t sb, zb;          // fp16 scale and zero-point (record metadata)
  float s, z;
  uint16_t c[3];            // 2-bit: 16-bit code thresholds
  float inv, zinv, thr;     // 4-bit: code estimate constants
  uint32_t flags;
};

template <bool BF>
__device__ __forceinline__ uint16_t to16_rn(double x) {
  if (BF) return __bfloat16_as_ushort(__double2bfloat16(x));
  return __half_as_ushort(__double2half(x));
}
template <bool BF>
__device__ __forceinline__ double from16(uint16_t b) {
  return BF ? (double)__uint_as_float((uint32_t)b << 16) : (double)__half2float(__ushort_as_half(b));
}
// The next larger value of the 16-bit input format (nan and +inf stay).
template <bool BF>
__device__ __forceinline__ uint16_t next_up16(uint16_t b) {
  constexpr uint16_t kInf = BF ? 0x7F80 : 0x7C00;
  if ((b & 0x7FFF) >= kInf && b != (uint16_t)(kInf | 0x8000)) return b;
  if (b == 0x8000) return 1;
  return (b & 0x8000) ? (uint16_t)(b - 1) : (uint16_t)(b + 1);
}
// The smallest input value v with v >= X (strict: v > X); X is exact in double.
// Then "x >= v" for an input x says exactly "x >= X" (or "x > X").
template <bool BF>
__device__ __forceinline__ uint16_t threshold16(double X, bool strict) {
  uint16_t c = to16_rn<BF>(X);
  const double cd = from16<BF>(c);
  if (cd < X || (strict && cd == X)) c = next_up16<BF>(c);
  return c;
}

// Parameters s = fp16((max - min) / L) (the quotient rounded once in double,
// then to fp16) and z = fp16(min).  2-bit codes count the thresholds
// X_k = z + (k + 1/2) s that x passes: x > X_k for even k, x >= X_k for odd k,
// which is round half to even of (x - z) / s clamped to [0, 3]; X_k is exact
// in double, so each test becomes "x >= c_k" for one 16-bit constant.  s == 0
// gives code 0 (thresholds +inf).  4-bit codes use the fp32 estimate described
// above, with thr = 0.5 - eb, or -1 (every code decided exactly) when z is
// far enough from min, or s small enough against max - z, that an estimate
// could leave [0, 15].
template <int BITS, bool BF>
__device__ __forceinline__ UnitOut<BITS, BF> unit_params(float mn, float mx) {
  constexpr int L = (1 << BITS) - 1;
  UnitOut<BITS, BF> u;
  u.flags = (isfinite(mn) && isfinite(mx)) ? 0u : (uint32_t)KVQ_DEV_NONFINITE_INPUT;
  const double dmn = mn, dmx = mx;
  const __half hs = __double2half((dmx - dmn) / (double)L), hz = __double2half(dmn);
  u.sb = __half_as_ushort(hs);
  u.zb = __half_as_ushort(hz);
  u.s = __half2float(hs);
  u.z = __half2float(hz);
  if (isinf(u.s) || isinf(u.z)) u.flags |= KVQ_DEV_PARAM_OVERFLOW;
  if constexpr (BITS == 2) {
    constexpr uint16_t kInf = BF ? 0x7F80 : 0x7C00;
#pragma unroll
    for (int k = 0; k < 3; ++k)
      u.c[k] = u.s == 0.f ? kInf : threshold16<BF>((double)u.z + (k + 0.5) * (double)u.s, (k & 1) == 0);
  } else {
    u.inv = u.s > 0.f ? 1.f / u.s : 0.f;
    u.zinv = u.z * u.inv;
    const bool safe = ((double)u.z - dmn <= 0.5 * (double)u.s) && (dmx - (double)u.z <= (L + 0.5) * (double)u.s);
    u.thr = safe ? 0.5f - 2.384185791015625e-7f * (2.f * (float)L + 2.f + fabsf(u.zinv)) : -1.f;
  }
  return u;
}

template <bool BF> struct Pair16;
template <> struct Pair16<false> {
  using T = __half2;
  static __device__ __forceinline__ T of(uint32_t u) { return u32_as_h2(u); }
  static __device__ __forceinline__ float lo(T v) { return __low2float(v); }
  static __device__ __forceinline__ float hi(T v) { return __high2float(v); }
};
template <> struct Pair16<true> {
  using T = __nv_bfloat162;
  static __device__ __forceinline__ T of(uint32_t u) { return *reinterpret_cast<__nv_bfloat162*>(&u); }
  static __device__ __forceinline__ float lo(T v) { return __low2float(v); }
  static __device__ __forceinline__ float hi(T v) { return __high2float(v); }
};

// 2-bit: the two codes of a pair from three 16-bit threshold pairs.  The masks
// m0 >= m1 >= m2 (0xFFFF per passing half) are a thermometer code; its count in
// binary is b1 = m1, b0 = m0 ^ m1 ^ m2.  Pair j lands at bits (2j, 16 + 2j).
template <bool BF>
__device__ __forceinline__ uint32_t code_pair2(uint32_t x, uint32_t c0, uint32_t c1, uint32_t c2, int j) {
  using P = Pair16<BF>;
  const uint32_t m0 = __hge2_mask(P::of(x), P::of(c0));
  const uint32_t m1 = __hge2_mask(P::of(x), P::of(c1));
  const uint32_t m2 = __hge2_mask(P::of(x), P::of(c2));
  return ((m0 ^ m1 ^ m2) & (0x00010001u << (2 * j))) | (m1 & (0x00020002u << (2 * j)));
}

// 4-bit: fp32 estimates of the codes of a pair, accumulated as k * 16^j into
// the low bits of 2^23-offset floats; ok turns false when a code is undecided.
template <bool BF>
__device__ __forceinline__ void code_pair4(uint32_t x, float inv0, float zinv0, float inv1, float zinv1, float thr,
                                           float& acc0, float& acc1, bool& ok, int j) {
  using P = Pair16<BF>;
  constexpr float kRound = 12582912.f;   // 1.5 * 2^23: adding it rounds to an integer
  const float kPos = (float)(1 << (4 * j));
  const float x0 = P::lo(P::of(x)), x1 = P::hi(P::of(x));
  const float r0 = fmaf(x0, inv0, -zinv0), r1 = fmaf(x1, inv1, -zinv1);
  const float k0 = (r0 + kRound) - kRound, k1 = (r1 + kRound) - kRound;
  ok = ok && fabsf(r0 - k0) < thr && fabsf(r1 - k1) < thr;
  acc0 = fmaf(k0, kPos, acc0);
  acc1 = fmaf(k1, kPos, acc1);
}

// One 4-bit code of the fallback path: the estimate when it decides (thr as in
// code_pair4; thr < 0 decides nothing), else the exact decision with (s, z).
__device__ __forceinline__ uint32_t estimate_or_exact(float x, float inv, float zinv, float thr, float2 sz, int levels) {
  constexpr float kRound = 12582912.f;
  const float r = fmaf(x, inv, -zinv);
  const float k = (r + kRound) - kRound;
  return fabsf(r - k) < thr ? (uint32_t)k : code_exact(x, sz.y, sz.x, levels);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}

// One CTA quantizes one group record (G tokens of one row); BF: bf16 inputs
// (else fp16).
//
// 1. The key and value tiles are copied to shared memory (rows padded by 16
//    bytes, so the 8 rows of an 8x8 ldmatrix tile fall in distinct banks).
// 2. Parameters: the first half of the threads reduce key channel pairs over
//    the G tokens, the second half value tokens over d, with 16-bit min/max.
// 3. Codes: a thread builds whole 32-bit words of the packed format for its own
//    lane.  ldmatrix hands lane (gr, tc) exactly a word's pairs: a key tile
//    (tokens x channels) gives token gr, channels 2tc and 2tc + 1; the same
//    tile transposed gives channel gr, tokens 2tc and 2tc + 1 for the values.
//    The first half of the warps code keys (a thread keeps the thresholds of its
//    channels across token blocks), the rest values (its eight tokens').
// 4. The record, assembled in shared memory, is stored in 16-byte pieces.
template <int BITS, int D, int G, bool BF>
__global__ void __launch_bounds__(quant_threads<BITS, D, G>()) kivi_quantize_kernel(QuantArgs a) {
  constexpr int NT = quant_threads<BITS, D, G>();
  constexpr int KW = NT / 64;                   // key warps, then as many value warps
  constexpr int L = (1 << BITS) - 1;
  constexpr int NTB = G / kTB;
  constexpr int PAIRS = 16 / BITS;              // pairs per word
  constexpr int P = D * BITS / 32;              // words per lane per TB (keys or values)
  constexpr int WPT = D * BITS / 128;           // key words per (lane, 8-token block)
  constexpr int CPW = PAIRS / 4;                // 8-channel blocks per value word
  constexpr int TBB = kTB * D * BITS / 8;       // code bytes of one TB
  constexpr int REC = 2 * NTB * TBB + 4 * D + NTB * kTB * 4;
  constexpr int PITCH = D + 8;                  // staged row pitch (halves)
  constexpr int KS = NT / D;                    // key parameter threads per channel pair
  constexpr int VS = NT / 2 / G;                // value parameter threads per token
  static_assert(REC % 16 == 0 && PAIRS % 4 == 0 && (D / 2) * KS == NT / 2 && VS >= 1, "shape");
  static_assert(KS <= 2 && VS <= 2, "parameter threads per unit");
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* sk = reinterpret_cast<uint16_t*>(smem);           // [G][PITCH]
  uint16_t* sv = sk + G * PITCH;                              // [G][PITCH]
  unsigned char* srec = reinterpret_cast<unsigned char*>(sv + G * PITCH);   // record image
  // 2-bit: thresholds, 16-bit per unit, adjacent units share a word
  // 4-bit: (inv, zinv, thr, -) and (s, z) per unit
  __shared__ __align__(16) uint16_t kc[BITS == 2 ? 3 : 1][D], vc[BITS == 2 ? 3 : 1][G];
  __shared__ __align__(16) float4 kp[BITS == 4 ? D : 1], vp[BITS == 4 ? G : 1];
  __shared__ __align__(16) float2 ksz[BITS == 4 ? D : 1], vsz[BITS == 4 ? G : 1];
  __shared__ uint32_t s_flags;

  const int row = blockIdx.y;
  const int grp = blockIdx.x;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) s_flags = 0;

  // 1. stage
  {
    const uint16_t* gk = a.src_k + (int64_t)row * a.src_row_stride + (int64_t)grp * G * D;
    const uint16_t* gv = a.src_v + (int64_t)row * a.src_row_stride + (int64_t)grp * G * D;
#pragma unroll 4
    for (int i = tid; i < G * D / 8; i += NT) {
      const int t = i / (D / 8), c8 = i - t * (D / 8);
      cp_async16(sk + t * PITCH + 8 * c8, gk + 8 * i);
      cp_async16(sv + t * PITCH + 8 * c8, gv + 8 * i);
    }
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
  }
  __syncthreads();

  using PT = Pair16<BF>;
  using T2 = typename PT::T;
  uint32_t flags = 0;
  uint16_t* ksc = reinterpret_cast<uint16_t*>(srec + 2 * NTB * TBB);   // key scales, then zeros
  uint32_t* vmeta = reinterpret_cast<uint32_t*>(srec + 2 * NTB * TBB + 4 * D);
  auto put_key = [&](int c, const UnitOut<BITS, BF>& u) {
    const int kt = c >> 4, rho = (c >> 3) & 1, tc = (c >> 1) & 3, e = c & 1;
    const int pos = 8 * (4 * (kt >> 1) + tc) + 4 * (kt & 1) + 2 * rho + e;
    ksc[pos] = u.sb;
    ksc[D + pos] = u.zb;
    if constexpr (BITS == 2) {
#pragma unroll
      for (int k = 0; k < 3; ++k) kc[k][c] = u.c[k];
    } else {
      kp[c] = make_float4(u.inv, u.zinv, u.thr, 0.f);
      ksz[c] = make_float2(u.s, u.z);
    }
    flags |= u.flags;
  };
  auto put_value = [&](int t, const UnitOut<BITS, BF>& u) {
    const int tb = t / kTB, tt = t % kTB;
    const int kt = tt >> 4, rho = (tt >> 3) & 1, tc = (tt >> 1) & 3, e = tt & 1;
    vmeta[tb * kTB + 8 * tc + 4 * kt + 2 * rho + e] = (uint32_t)u.sb | ((uint32_t)u.zb << 16);
    if constexpr (BITS == 2) {
#pragma unroll
      for (int k = 0; k < 3; ++k) vc[k][t] = u.c[k];
    } else {
      vp[t] = make_float4(u.inv, u.zinv, u.thr, 0.f);
      vsz[t] = make_float2(u.s, u.z);
    }
    flags |= u.flags;
  };

  // 2. parameters
  if (tid < NT / 2) {
    // channel pair pc over tokens ks, ks + KS, ... (rows 1 apart: 4 banks apart)
    const int pc = tid / KS, ks = tid % KS;
    T2 mn = PT::of(BF ? 0x7F807F80u : 0x7C007C00u), mx = PT::of(BF ? 0xFF80FF80u : 0xFC00FC00u);
#pragma unroll 8
    for (int t = ks; t < G; t += KS) {
      const T2 x = PT::of(*reinterpret_cast<const uint32_t*>(sk + t * PITCH + 2 * pc));
      mn = __hmin2(mn, x);
      mx = __hmax2_nan(mx, x);
    }
    if (KS == 2) {
      uint32_t a0 = *reinterpret_cast<uint32_t*>(&mn), a1 = *reinterpret_cast<uint32_t*>(&mx);
      mn = __hmin2(mn, PT::of(__shfl_xor_sync(0xffffffffu, a0, 1)));
      mx = __hmax2_nan(mx, PT::of(__shfl_xor_sync(0xffffffffu, a1, 1)));
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (KS == 2 && e != ks) continue;
      const float fmn = e ? PT::hi(mn) : PT::lo(mn), fmx = e ? PT::hi(mx) : PT::lo(mx);
      put_key(2 * pc + e, unit_params<BITS, BF>(fmn, fmx));
    }
  } else {
    // token t over channel pairs [v D/(2 VS), (v + 1) D/(2 VS)), four at a time
    const int u = tid - NT / 2, t = u / VS, v = u % VS;
    constexpr int PPV = D / (2 * VS);
    T2 mn = PT::of(BF ? 0x7F807F80u : 0x7C007C00u), mx = PT::of(BF ? 0xFF80FF80u : 0xFC00FC00u);
#pragma unroll 4
    for (int p4 = 0; p4 < PPV / 4; ++p4) {
      const uint4 q = *reinterpret_cast<const uint4*>(sv + t * PITCH + 2 * (v * PPV + 4 * p4));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mn = __hmin2(mn, PT::of(w[i]));
        mx = __hmax2_nan(mx, PT::of(w[i]));
      }
    }
    float fmn = fminf(PT::lo(mn), PT::hi(mn));
    float fmx = PT::lo(mx), fmx1 = PT::hi(mx);
    fmx = (isnan(fmx) || isnan(fmx1)) ? __int_as_float(0x7fc00000) : fmaxf(fmx, fmx1);
    if (VS == 2) {
      const float omn = __shfl_xor_sync(0xffffffffu, fmn, 1), omx = __shfl_xor_sync(0xffffffffu, fmx, 1);
      fmn = fminf(fmn, omn);
      fmx = (isnan(fmx) || isnan(omx)) ? __int_as_float(0x7fc00000) : fmaxf(fmx, omx);
    }
    if (v == 0) put_value(t, unit_params<BITS, BF>(fmn, fmx));
  }
  // this half's parameters are in shared memory (with 256 threads a CTA-wide
  // barrier measured faster: 464 against 523 us on 8b4)
  if constexpr (NT == 128) half_bar_sync<NT>(tid >= NT / 2);
  else __syncthreads();

  // 3. codes
  const int tc = lane & 3;
  auto word_at = [&](bool is_v, int tb, int w) -> uint32_t* {
    return reinterpret_cast<uint32_t*>(srec + (is_v ? NTB + tb : tb) * TBB + 16 * (32 * (w >> 2) + lane) + 4 * (w & 3));
  };
  if (warp < KW) {
    // keys: word (nt, sub) of token 8 nt + gr holds channels 8 PAIRS sub + 8 j + 2 tc (+1);
    // a warp takes subs warp, warp + KW, ... of every 8-token block, or (fewer
    // subs than key warps) one sub of every (KW / WPT)-th block
    constexpr int SUBS_PER_WARP = WPT >= KW ? WPT / KW : 1;
    constexpr int IT_STEP = WPT >= KW ? 1 : KW / WPT;
    const int it0 = WPT >= KW ? 0 : warp / WPT;
    for (int si = 0; si < SUBS_PER_WARP; ++si) {
      const int sub = WPT >= KW ? KW * si + warp : warp % WPT;
      const int cbase = 8 * PAIRS * sub + 2 * tc;
      if constexpr (BITS == 2) {
        uint32_t c0[PAIRS], c1[PAIRS], c2[PAIRS];
#pragma unroll
        for (int j = 0; j < PAIRS; ++j) {
          c0[j] = *reinterpret_cast<const uint32_t*>(&kc[0][cbase + 8 * j]);
          c1[j] = *reinterpret_cast<const uint32_t*>(&kc[1][cbase + 8 * j]);
          c2[j] = *reinterpret_cast<const uint32_t*>(&kc[2][cbase + 8 * j]);
        }
#pragma unroll 1
        for (int it = it0; it < NTB * 4; it += IT_STEP) {
          const int tb = it >> 2, nt = it & 3;
          const uint16_t* rowp = sk + (tb * kTB + 8 * nt + (lane & 7)) * PITCH + 8 * PAIRS * sub + 8 * (lane >> 3);
          uint32_t x[PAIRS];
#pragma unroll
          for (int i = 0; i < PAIRS / 4; ++i) ldsm_x4(x + 4 * i, rowp + 32 * i);
          uint32_t wd = 0;
#pragma unroll
          for (int j = 0; j < PAIRS; ++j) wd |= code_pair2<BF>(x[j], c0[j], c1[j], c2[j], j);
          *word_at(false, tb, nt * WPT + sub) = wd;
        }
      } else {
        float inv[2 * PAIRS], zinv[2 * PAIRS], thr = 0.5f;
#pragma unroll
        for (int j = 0; j < PAIRS; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float4 q = kp[cbase + 8 * j + e];
            inv[2 * j + e] = q.x;
            zinv[2 * j + e] = q.y;
            thr = fminf(thr, q.z);
          }
#pragma unroll 1
        for (int it = it0; it < NTB * 4; it += IT_STEP) {
          const int tb = it >> 2, nt = it & 3;
          const uint16_t* rowp = sk + (tb * kTB + 8 * nt + (lane & 7)) * PITCH + 8 * PAIRS * sub + 8 * (lane >> 3);
          uint32_t x[PAIRS];
#pragma unroll
          for (int i = 0; i < PAIRS / 4; ++i) ldsm_x4(x + 4 * i, rowp + 32 * i);
          float acc0 = 8388608.f, acc1 = 8388608.f;
          bool ok = true;
#pragma unroll
          for (int j = 0; j < PAIRS; ++j)
            code_pair4<BF>(x[j], inv[2 * j], zinv[2 * j], inv[2 * j + 1], zinv[2 * j + 1], thr, acc0, acc1, ok, j);
          uint32_t wd = __byte_perm(__float_as_uint(acc0), __float_as_uint(acc1), 0x5410);
          if (!ok) {   // redo the word: the estimate where it decides, the exact decision elsewhere
            wd = 0;
            for (int j = 0; j < PAIRS; ++j)
              for (int e = 0; e < 2; ++e) {
                const int c = cbase + 8 * j + e;
                const float xv = e ? PT::hi(PT::of(x[j])) : PT::lo(PT::of(x[j]));
                wd |= estimate_or_exact(xv, inv[2 * j + e], zinv[2 * j + e], thr, ksz[c], L) << (16 * e + BITS * j);
              }
          }
          *word_at(false, tb, nt * WPT + sub) = wd;
        }
      }
    }
  } else {
    // values: word w holds channels 8 (CPW w + j / 4) + gr, tokens 8 (j % 4) + 2 tc (+1)
    const int vw = warp - KW;
    for (int tb = 0; tb < NTB; ++tb) {
      if constexpr (BITS == 2) {
        uint32_t c0[4], c1[4], c2[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int t = tb * kTB + 8 * m + 2 * tc;
          c0[m] = *reinterpret_cast<const uint32_t*>(&vc[0][t]);
          c1[m] = *reinterpret_cast<const uint32_t*>(&vc[1][t]);
          c2[m] = *reinterpret_cast<const uint32_t*>(&vc[2][t]);
        }
#pragma unroll 1
        for (int w = vw; w < P; w += KW) {
          uint32_t x[PAIRS];
#pragma unroll
          for (int i = 0; i < PAIRS / 4; ++i)
            ldsm_x4_t(x + 4 * i, sv + (tb * kTB + 8 * (lane >> 3) + (lane & 7)) * PITCH + 8 * (CPW * w + i));
          uint32_t wd = 0;
#pragma unroll
          for (int j = 0; j < PAIRS; ++j) wd |= code_pair2<BF>(x[j], c0[j & 3], c1[j & 3], c2[j & 3], j);
          *word_at(true, tb, w) = wd;
        }
      } else {
        float inv[8], zinv[8], thr = 0.5f;
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float4 q = vp[tb * kTB + 8 * m + 2 * tc + e];
            inv[2 * m + e] = q.x;
            zinv[2 * m + e] = q.y;
            thr = fminf(thr, q.z);
          }
#pragma unroll 1
        for (int w = vw; w < P; w += KW) {
          uint32_t x[PAIRS];
          ldsm_x4_t(x, sv + (tb * kTB + 8 * (lane >> 3) + (lane & 7)) * PITCH + 8 * w);
          float acc0 = 8388608.f, acc1 = 8388608.f;
          bool ok = true;
#pragma unroll
          for (int j = 0; j < PAIRS; ++j)
            code_pair4<BF>(x[j], inv[2 * j], zinv[2 * j], inv[2 * j + 1], zinv[2 * j + 1], thr, acc0, acc1, ok, j);
          uint32_t wd = __byte_perm(__float_as_uint(acc0), __float_as_uint(acc1), 0x5410);
          if (!ok) {   // redo the word: the estimate where it decides, the exact decision elsewhere
            wd = 0;
            for (int j = 0; j < PAIRS; ++j)
              for (int e = 0; e < 2; ++e) {
                const int t = tb * kTB + 8 * j + 2 * tc + e;
                const float xv = e ? PT::hi(PT::of(x[j])) : PT::lo(PT::of(x[j]));
                wd |= estimate_or_exact(xv, inv[2 * j + e], zinv[2 * j + e], thr, vsz[t], L) << (16 * e + BITS * j);
              }
          }
          *word_at(true, tb, w) = wd;
        }
      }
    }
  }

  if (flags) atomicOr(&s_flags, flags);
  __syncthreads();

  // 4. store the record
  char* rec = record_ptr(a.geom, row, a.dst_group0 + grp);
  if (rec != nullptr) {
    for (int i = tid; i < REC / 16; i += NT)
      reinterpret_cast<uint4*>(rec)[i] = reinterpret_cast<const uint4*>(srec)[i];
  } else if (tid == 0) {
    s_flags |= KVQ_DEV_BAD_PAGE;   // page outside the pool: nothing is written
  }
  if (tid == 0 && s_flags) flag_status(a.geom.status, s_flags);
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
  const size_t smem = (size_t)G * (D + 8) * 2 * 2 + (size_t)(2 * G * D * BITS / 8 + 4 * D + G * 4);
  auto kern = kivi_quantize_kernel<BITS, D, G, BF>;
  static bool attr_set = false;   // per template instance; the attribute is per device function
  if (!attr_set) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attr_set = true;
  }
  dim3 grid(a.n_groups, a.geom.B * a.geom.Hkv);
  kern<<<grid, quant_threads<BITS, D, G>(), smem, st>>>(a);
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

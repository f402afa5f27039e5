// KIVI decode attention straight from the packed cache.
//
// Every decode step reads the whole cache ("La compression du cache KV est une
// decision d'infrastructure...", section "... quand la HBM, pas les FLOPs, est
// votre plafond"), so the kernel is a streaming pass over the group records.
// The dequantization is fused into both contractions instead of materialising
// keys or values:
//   score_t = sum_c q_c (z_c + s_c code_tc) = beta + sum_c (q_c s_c) code_tc
//   o_c     = sum_t p_t (zv_t + sv_t code_tc) = sum_t p_t zv_t + sum_t (p_t sv_t) code_tc
// The per-group q~ = q (.) s and the per-token p~ = p (.) sv are split into fp16
// hi + lo parts that sit in the two 8-row halves of the m16 A operand, so each
// GQA group (up to 8 query heads) runs both contractions on mma.sync with
// exact small-integer fp16 codes as the B operand and ~22-bit weights.
//
// Split-K: each CTA covers a range of groups (or window tokens) of one row and
// writes a partial (m, l, o); a second kernel merges the partials with a
// log-sum-exp that normalises globally, as Minima-KV merges its per-format
// partial attention states ("KV-cache compresse et modeles 4-bit ...",
// section "Minima-KV : la compression sans eviction").
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kThreads = kWarpsAttn * 32;

__device__ __forceinline__ uint32_t in16x2_to_h2(uint32_t w, int dtype) {
  if (dtype == KVQ_FP16) return w;
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
  return h2_as_u32(__floats2half2_rn(lo, hi));
}

__device__ __forceinline__ float warp_max4(float x) {   // over the 4 lanes of a quad
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float warp_sum4(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// Writes the CTA's partial for `g` heads from per-warp states held in shared memory.
template <int D>
__device__ void cta_merge_write(const AttnArgs& a, const float* sm_m, const float* sm_l, const float* sm_o,
                                int row, int split, int n_split) {
  const int g = a.geom.g;
  for (int i = threadIdx.x; i < g * (D + 2); i += kThreads) {
    const int h = i / (D + 2), c = i - h * (D + 2);
    float M = -INFINITY;
    for (int w = 0; w < kWarpsAttn; ++w) M = fmaxf(M, sm_m[w * 8 + h]);
    float val;
    if (M == -INFINITY) {
      val = c == D ? -INFINITY : 0.0f;
    } else if (c < D) {
      val = 0.0f;
      for (int w = 0; w < kWarpsAttn; ++w) val += sm_o[(w * 8 + h) * D + c] * exp2f(sm_m[w * 8 + h] - M);
    } else if (c == D) {
      val = M;
    } else {
      val = 0.0f;
      for (int w = 0; w < kWarpsAttn; ++w) val += sm_l[w * 8 + h] * exp2f(sm_m[w * 8 + h] - M);
    }
    a.ws[(((int64_t)row * n_split + split) * g + h) * (D + 2) + c] = val;
  }
}

template <int BITS, int D, int G>
__global__ void __launch_bounds__(kThreads) kivi_attn_kernel(AttnArgs a) {
  constexpr int NTB = G / kTB;
  constexpr int P = D * BITS / 32;          // code words per lane per TB
  constexpr int J = BITS == 2 ? 4 : 2;      // pairs per half word
  constexpr int NKT = D / 16;               // channel k-tiles
  constexpr int NNT = D / 8;                // channel n-tiles (PV)
  constexpr int WPN = P / 4;                // key words per score n-tile
  constexpr int64_t TBC = kTB * D * BITS / 8;

  __shared__ float sm_m[kWarpsAttn * 8], sm_l[kWarpsAttn * 8];
  __shared__ __align__(16) float sm_o[kWarpsAttn * 8 * D];

  const Geom& gm = a.geom;
  const int row = blockIdx.y;
  const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
  const int split = blockIdx.x;
  const int n_split = a.nq + a.nw;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, tc = lane & 3;
  const bool head_ok = gr < gm.g;
  const uint16_t* qrow = a.q + ((int64_t)b * gm.Hq + (int64_t)hkv * gm.g + (head_ok ? gr : 0)) * D;

  if (split < a.nq) {
    // ---------------------------------------------------------------- quantized groups
    uint32_t qh[NKT][2];   // q of head gr at channels 16kt + 8rho + 2tc + {0, 1}, fp16x2
#pragma unroll
    for (int kt = 0; kt < NKT; ++kt)
#pragma unroll
      for (int rho = 0; rho < 2; ++rho)
        qh[kt][rho] = head_ok ? in16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow + 16 * kt + 8 * rho + 2 * tc),
                                             gm.dtype)
                              : 0u;
    float o[NNT][4];
#pragma unroll
    for (int i = 0; i < NNT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m = -INFINITY, l = 0.0f, wz = 0.0f;

    const int64_t g_lo = (int64_t)split * a.gps;
    const int64_t g_hi = min(g_lo + a.gps, a.n_groups);
    for (int64_t t_idx = g_lo * NTB + warp; t_idx < g_hi * NTB; t_idx += kWarpsAttn) {
      const int64_t gi = t_idx / NTB;
      const int tbg = (int)(t_idx - gi * NTB);
      const char* rec = record_ptr(gm, row, gi);
      uint4 kc[P / 4], vc[P / 4];
#pragma unroll
      for (int p = 0; p < P / 4; ++p) {
        kc[p] = ldg_nc_v4(rec + tbg * TBC + 16 * (32 * p + lane));
        vc[p] = ldg_nc_v4(rec + (NTB + tbg) * TBC + 16 * (32 * p + lane));
      }
      uint32_t ks[NKT][2], kz[NKT][2];
      {
        const uint4* psc = reinterpret_cast<const uint4*>(rec + rec_kscale_off(gm) + 2 * (tc * (D / 4)));
        const uint4* pz = reinterpret_cast<const uint4*>(rec + rec_kzero_off(gm) + 2 * (tc * (D / 4)));
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
          const uint4 s4 = ldg_nc_v4(psc + i), z4 = ldg_nc_v4(pz + i);
          ks[2 * i][0] = s4.x; ks[2 * i][1] = s4.y; ks[2 * i + 1][0] = s4.z; ks[2 * i + 1][1] = s4.w;
          kz[2 * i][0] = z4.x; kz[2 * i][1] = z4.y; kz[2 * i + 1][0] = z4.z; kz[2 * i + 1][1] = z4.w;
        }
      }
      uint32_t vm[8];
      {
        const uint4* pv = reinterpret_cast<const uint4*>(rec + rec_vmeta_off(gm) + 4 * (tbg * kTB + 8 * tc));
        const uint4 v0 = ldg_nc_v4(pv), v1 = ldg_nc_v4(pv + 1);
        vm[0] = v0.x; vm[1] = v0.y; vm[2] = v0.z; vm[3] = v0.w;
        vm[4] = v1.x; vm[5] = v1.y; vm[6] = v1.z; vm[7] = v1.w;
      }

      // beta = sum_c q_c z_c (z replicated over the 8 columns of B)
      float bacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kt = 0; kt < NKT; ++kt) {
        const uint32_t aq[4] = {qh[kt][0], 0u, qh[kt][1], 0u};
        mma_f16_16816(bacc, aq, kz[kt][0], kz[kt][1]);
      }
      const float beta = bacc[0];

      // q~ = q (.) s as hi + lo
      uint32_t aqs[NKT][4];
#pragma unroll
      for (int kt = 0; kt < NKT; ++kt)
#pragma unroll
        for (int rho = 0; rho < 2; ++rho) {
          const __half2 qv = u32_as_h2(qh[kt][rho]), sv = u32_as_h2(ks[kt][rho]);
          const __half2 hi = __hmul2(qv, sv);
          const __half2 lo = __hfma2(qv, sv, __hneg2(hi));
          aqs[kt][2 * rho] = h2_as_u32(hi);
          aqs[kt][2 * rho + 1] = h2_as_u32(lo);
        }

      // scores: rows gr (hi) and gr + 8 (lo) of head gr, columns = tokens
      float sc[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int wi = 0; wi < WPN; ++wi) {
          const int w = nt * WPN + wi;
          const uint4 pc = kc[w >> 2];
          const uint32_t word = (w & 3) == 0 ? pc.x : (w & 3) == 1 ? pc.y : (w & 3) == 2 ? pc.z : pc.w;
          uint32_t pr[2 * J];
          unpack_word<BITS>(word, pr);
#pragma unroll
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int m2 = 0; m2 < J / 2; ++m2) {
              const int kt = (J / 2) * (2 * wi + half) + m2;
              mma_f16_16816(sc[nt], aqs[kt], pr[half * J + 2 * m2], pr[half * J + 2 * m2 + 1]);
            }
        }
      }

      // online softmax (log2 domain) for head gr over this TB's 32 tokens
      float x[4][2];
      float mt = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          x[nt][e] = (sc[nt][e] + sc[nt][2 + e] + beta) * a.scale_log2;
          mt = fmaxf(mt, x[nt][e]);
        }
      mt = warp_max4(mt);
      if (mt > m) {
        const float alpha = exp2f(m - mt);
        l *= alpha;
        wz *= alpha;
#pragma unroll
        for (int i = 0; i < NNT; ++i) {
          o[i][0] *= alpha; o[i][1] *= alpha; o[i][2] *= alpha; o[i][3] *= alpha;
        }
        m = mt;
      }
      uint32_t apv[2][4];
#pragma unroll
      for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int nt = 2 * kt + rr;
          float pt[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float p = exp2f(x[nt][e] - m);
            const uint32_t meta = vm[2 * nt + e];
            const float svv = __half2float(__ushort_as_half((uint16_t)(meta & 0xFFFFu)));
            const float zv = __half2float(__ushort_as_half((uint16_t)(meta >> 16)));
            l += p;
            wz += p * zv;
            pt[e] = p * svv;
          }
          const __half2 hi = __floats2half2_rn(pt[0], pt[1]);
          const float2 hb = __half22float2(hi);
          const __half2 lo = __floats2half2_rn(pt[0] - hb.x, pt[1] - hb.y);
          apv[kt][2 * rr] = h2_as_u32(hi);
          apv[kt][2 * rr + 1] = h2_as_u32(lo);
        }

      // o += p~ . codes: rows gr (hi) and gr + 8 (lo), columns = channels
#pragma unroll
      for (int w = 0; w < P; ++w) {
        const uint4 pc = vc[w >> 2];
        const uint32_t word = (w & 3) == 0 ? pc.x : (w & 3) == 1 ? pc.y : (w & 3) == 2 ? pc.z : pc.w;
        uint32_t pr[2 * J];
        unpack_word<BITS>(word, pr);
        if (BITS == 2) {
#pragma unroll
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int kt = 0; kt < 2; ++kt)
              mma_f16_16816(o[2 * w + half], apv[kt], pr[half * 4 + 2 * kt], pr[half * 4 + 2 * kt + 1]);
        } else {
#pragma unroll
          for (int kt = 0; kt < 2; ++kt) mma_f16_16816(o[w], apv[kt], pr[2 * kt], pr[2 * kt + 1]);
        }
      }
    }

    // per-warp state -> shared memory
    l = warp_sum4(l);
    wz = warp_sum4(wz);
    if (tc == 0) {
      sm_m[warp * 8 + gr] = m;
      sm_l[warp * 8 + gr] = l;
    }
#pragma unroll
    for (int nt = 0; nt < NNT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) sm_o[(warp * 8 + gr) * D + 8 * nt + 2 * tc + e] = o[nt][e] + o[nt][2 + e] + wz;
  } else {
    // ---------------------------------------------------------------- window tokens (exact 16-bit)
    constexpr int CPL = D / 32;   // channels per lane in the PV step
    const int w0 = (split - a.nq) * kWindowChunk + warp * 32;
    const int i_tok = w0 + lane;
    const bool valid = i_tok < a.r;
    const int slot = (a.head + (valid ? i_tok : 0)) % gm.cap;
    const uint16_t* krow = ring_ptr(gm, row, 0) + (int64_t)slot * D;
    const uint16_t* qbase = a.q + ((int64_t)b * gm.Hq + (int64_t)hkv * gm.g) * D;
    float s[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) s[h] = 0.f;
    if (valid) {
      for (int c8 = 0; c8 < D; c8 += 8) {
        const uint4 kk = *reinterpret_cast<const uint4*>(krow + c8);
        const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w};
        float kf[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          kf[2 * i] = in16_to_float((uint16_t)(kw[i] & 0xFFFFu), gm.dtype);
          kf[2 * i + 1] = in16_to_float((uint16_t)(kw[i] >> 16), gm.dtype);
        }
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          if (h < gm.g) {
            const uint16_t* qh = qbase + (int64_t)h * D + c8;
#pragma unroll
            for (int i = 0; i < 8; ++i) s[h] += in16_to_float(qh[i], gm.dtype) * kf[i];
          }
        }
      }
    }
    float mh[8], p[8], lh[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float xv = valid ? s[h] * a.scale_log2 : -INFINITY;
      float mx = xv;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      mh[h] = mx;
      p[h] = (valid && mx != -INFINITY) ? exp2f(xv - mx) : 0.f;
      float sum = p[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      lh[h] = sum;
    }
    float ov[8][CPL];
#pragma unroll
    for (int h = 0; h < 8; ++h)
#pragma unroll
      for (int c = 0; c < CPL; ++c) ov[h][c] = 0.f;
    const int n_tok = min(32, a.r - w0);
    for (int j = 0; j < n_tok; ++j) {
      const int sl = (a.head + w0 + j) % gm.cap;
      const uint16_t* vrow = ring_ptr(gm, row, 1) + (int64_t)sl * D + lane * CPL;
      float vf[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) vf[c] = in16_to_float(vrow[c], gm.dtype);
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float pj = __shfl_sync(0xffffffffu, p[h], j);
#pragma unroll
        for (int c = 0; c < CPL; ++c) ov[h][c] += pj * vf[c];
      }
    }
    // every lane holds every head's warp-wide max and sum; lane h publishes head h
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (lane == h) {
        sm_m[warp * 8 + h] = (h < gm.g && n_tok > 0) ? mh[h] : -INFINITY;
        sm_l[warp * 8 + h] = (h < gm.g && n_tok > 0) ? lh[h] : 0.f;
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) sm_o[(warp * 8 + h) * D + lane * CPL + c] = ov[h][c];
    }
  }
  __syncthreads();
  cta_merge_write<D>(a, sm_m, sm_l, sm_o, row, split, n_split);
}

// One CTA per query head: log-sum-exp merge of the row's partials.
template <int D>
__global__ void lse_merge_kernel(AttnArgs a) {
  const int row = blockIdx.y, h = blockIdx.x;
  const Geom& gm = a.geom;
  const int n_split = a.nq + a.nw;
  const float* base = a.ws + ((int64_t)row * n_split * gm.g + h) * (D + 2);
  const int64_t stride = (int64_t)gm.g * (D + 2);
  float M = -INFINITY;
  for (int j = 0; j < n_split; ++j) M = fmaxf(M, base[j * stride + D]);
  float L = 0.f;
  for (int j = 0; j < n_split; ++j) L += base[j * stride + D + 1] * exp2f(base[j * stride + D] - M);
  const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
  float* out = a.out + ((int64_t)b * gm.Hq + (int64_t)hkv * gm.g + h) * D;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < n_split; ++j) acc += base[j * stride + c] * exp2f(base[j * stride + D] - M);
    out[c] = acc / L;
  }
}

template <int BITS, int D, int G>
void launch_attn(const AttnArgs& a, cudaStream_t st) {
  const int rows = a.geom.B * a.geom.Hkv;
  kivi_attn_kernel<BITS, D, G><<<dim3(a.nq + a.nw, rows), kThreads, 0, st>>>(a);
  lse_merge_kernel<D><<<dim3(a.geom.g, rows), D, 0, st>>>(a);
  count_launch(2);
}

}  // namespace

void launch_kivi_attention(const AttnArgs& a, cudaStream_t st) {
  const Geom& g = a.geom;
  if (g.bits == 2 && g.d == 128 && g.G == 32) launch_attn<2, 128, 32>(a, st);
  else if (g.bits == 2 && g.d == 64 && g.G == 32) launch_attn<2, 64, 32>(a, st);
  else if (g.bits == 4 && g.d == 128 && g.G == 64) launch_attn<4, 128, 64>(a, st);
  else if (g.bits == 4 && g.d == 128 && g.G == 32) launch_attn<4, 128, 32>(a, st);
  else if (g.bits == 2 && g.d == 128 && g.G == 64) launch_attn<2, 128, 64>(a, st);
  else if (g.bits == 4 && g.d == 64 && g.G == 32) launch_attn<4, 64, 32>(a, st);
  else if (g.bits == 2 && g.d == 64 && g.G == 64) launch_attn<2, 64, 64>(a, st);
  else if (g.bits == 4 && g.d == 64 && g.G == 64) launch_attn<4, 64, 64>(a, st);
}

}  // namespace kvq

// KIVI decode attention straight from the packed cache.
//
// Every decode step reads the whole cache ("La compression du cache KV est une
// decision d'infrastructure...", section "... quand la HBM, pas les FLOPs, est
// votre plafond"), so the kernel is one streaming pass over the group records
// and window tokens.  The dequantization is fused into both contractions:
//   score_t = sum_c q_c (z_c + s_c code_tc) = beta + sum_c (q_c s_c) code_tc
//   o_c     = sum_t p_t (zv_t + sv_t code_tc) = sum_t p_t zv_t + sum_t (p_t sv_t) code_tc
// q~ = q (.) s (per group) and p~ = p (.) sv (per token) are split into fp16
// hi + lo parts held in the two 8-row halves of the m16 A operand, so one GQA
// group of up to 8 query heads runs both contractions on mma.sync with exact
// small-integer fp16 codes as the B operand.
//
// Structure (one CTA per SM, one launch per decode step):
//   warp 0      producer: 1-D bulk copies (cp.async.bulk, no multicast) of whole
//               group records / window rows into a ring of shared-memory stages
//   warp 1      prep: the zero-point term beta = q . z for every group of a stage
//               in one batched mma (columns = groups)
//   warps 2..9  consumers: one 32-token block per warp per stage, online softmax
// Work: the (row, item) sequence -- a row's groups then its 32-token window
// chunks -- is cut into equal-byte ranges, one per CTA.  A CTA writes one
// partial (m, l, o) per row it touches; the last CTA to finish a row (atomic
// counter in the cache buffer, reset after use) merges that row's partials
// with a log-sum-exp that normalises globally, as Minima-KV merges its partial
// attention states ("KV-cache compresse et modeles 4-bit ...", section
// "Minima-KV : la compression sans eviction").
//
// Every mbarrier wait is bounded (about 1 s of SM cycles); on expiry the
// warp sets KVQ_DEV_WAIT_TIMEOUT, stops computing, keeps taking the same
// barriers as the other consumer warps, and the producer waits (bounded) for its
// copies in flight before the CTA exits.
#include <cuda_runtime.h>

#include <mutex>

#include <cuda_bf16.h>

#include "decode_common.cuh"

namespace kvq {

namespace {

constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 2) * 32;
constexpr int kWinTok = 32;                     // tokens per window item

__device__ __forceinline__ void consumer_bar() { named_bar_sync<kConsumers * 32>(); }

template <int BITS, int D, int G>
struct K {
  static constexpr int NTB = G / kTB;
  static constexpr int SG = kConsumers / NTB;                    // groups per stage
  static constexpr int REC = G * D * BITS / 4 + 4 * D + 4 * G;   // record bytes
  static constexpr int TBC = kTB * D * BITS / 8;                 // TB code bytes
  static constexpr int WROW = D * 2;                             // window row in shared memory
  static constexpr int WINB = kWinTok * WROW * 2;                 // window item bytes in a stage (K + V)
  static constexpr int STAGE = ((SG * REC > WINB ? SG * REC : WINB) + 127) / 128 * 128;
  static constexpr int NST = STAGE > 48 * 1024 ? 3 : 4;          // pipeline depth
  static constexpr int KSOFF = G * D * BITS / 4;
  static constexpr int KZOFF = KSOFF + 2 * D;
  static constexpr int VMOFF = KSOFF + 4 * D;
  // shared memory map (bytes)
  static constexpr int OFF_BETA = NST * STAGE;
  static constexpr int OFF_M = OFF_BETA + NST * SG * 8 * 4;
  static constexpr int OFF_L = OFF_M + kConsumers * 8 * 4;
  static constexpr int OFF_O = OFF_L + kConsumers * 8 * 4;
  static constexpr int OFF_Q = OFF_O + kConsumers * 8 * D * 4;   // q ring: 2 slots x raw 16-bit q of 8 heads
  static constexpr int OFF_BAR = OFF_Q + 2 * 8 * D * 2;
  static constexpr int OFF_FLAG = OFF_BAR + (3 * NST + 4) * 8;
  static constexpr int SMEM = OFF_FLAG + 16;
};

// ------------------------------------------------------------------ work partition
// Items of a row: groups 0..n_g-1, then window chunks of kWinTok tokens.  Item
// weights are the bytes they read; CTA c owns the items whose start byte lies in
// [c * W_tot / n, (c + 1) * W_tot / n).
struct Part {
  int64_t n_g, W_row, W_tot, rows;
  int n_items, n_wc, r, rec, tokb, n_cta;
  __device__ int64_t start_in_row(int k) const {
    return k < n_g ? (int64_t)k * rec : n_g * rec + (int64_t)(k - n_g) * kWinTok * tokb;
  }
  __device__ int64_t lo(int c) const { return (int64_t)c * W_tot / n_cta; }
  // first global item whose start byte is >= x
  __device__ int64_t first_item(int64_t x) const {
    const int64_t row = x / W_row;
    if (row >= rows) return rows * n_items;
    const int64_t off = x - row * W_row;
    int64_t k;
    if (off <= n_g * rec) {
      k = (off + rec - 1) / rec;
    } else {
      const int64_t wb = (int64_t)kWinTok * tokb;
      k = n_g + (off - n_g * rec + wb - 1) / wb;
    }
    return row * n_items + k;   // k == n_items rolls into the next row's item 0
  }
  __device__ int cta_of(int64_t item) const {
    const int64_t row = item / n_items;
    const int64_t st = row * W_row + start_in_row((int)(item - row * n_items));
    int c = (int)(st * n_cta / W_tot);
    if (c > n_cta - 1) c = n_cta - 1;
    while (c + 1 < n_cta && lo(c + 1) <= st) ++c;
    while (c > 0 && lo(c) > st) --c;
    return c;
  }
};

// Iterates the chunks of one CTA: calls f(stage_index, row, is_window, first, count)
// for quantized chunks (count groups from group `first`) and window chunks
// (count = 1, first = chunk index); calls seg(row, begin) at each segment start
// and seg_end(row) at its end.
template <int SG, class FC, class FS, class FE>
__device__ __forceinline__ void for_each_chunk(const Part& P, int64_t i0, int64_t i1, FC f, FS seg, FE seg_end) {
  int s = 0;
  if (i0 >= i1) return;
  for (int64_t row = i0 / P.n_items; row * P.n_items < i1; ++row) {
    const int64_t a = max(i0, row * P.n_items) - row * P.n_items;
    const int64_t b = min(i1, (row + 1) * P.n_items) - row * P.n_items;
    if (a >= b) continue;
    seg((int)row);
    for (int64_t k = a; k < min(b, P.n_g); k += SG) {
      const int cnt = (int)min((int64_t)SG, min(b, P.n_g) - k);
      f(s++, (int)row, false, k, cnt);
    }
    for (int64_t k = max(a, P.n_g); k < b; ++k) f(s++, (int)row, true, k - P.n_g, 1);
    seg_end((int)row);
  }
}

// ------------------------------------------------------------------ the kernel
template <int BITS, int D, int G>
__global__ void __launch_bounds__(kThreads, 1) kivi_decode_kernel(AttnArgs a) {
  using C = K<BITS, D, G>;
  constexpr int P = D * BITS / 32;
  constexpr int J = BITS == 2 ? 4 : 2;
  constexpr int NKT = D / 16;
  constexpr int NNT = D / 8;
  constexpr int WPN = P / 4;

  extern __shared__ __align__(128) unsigned char smem[];
  float* sm_beta = reinterpret_cast<float*>(smem + C::OFF_BETA);
  float* sm_m = reinterpret_cast<float*>(smem + C::OFF_M);
  float* sm_l = reinterpret_cast<float*>(smem + C::OFF_L);
  float* sm_o = reinterpret_cast<float*>(smem + C::OFF_O);
  uint16_t* sm_q = reinterpret_cast<uint16_t*>(smem + C::OFF_Q);
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_ready = bar_full + C::NST;
  uint64_t* bar_empty = bar_ready + C::NST;
  uint64_t* bar_qfull = bar_empty + C::NST;    // [2]
  uint64_t* bar_qempty = bar_qfull + 2;        // [2]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);
  volatile int* last_flag = abort_flag + 1;

  const Geom& gm = a.geom;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, tc = lane & 3;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_ready[i], 1);
      mbar_init(&bar_empty[i], kConsumers);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_qfull[i], 1);
      mbar_init(&bar_qempty[i], kConsumers + 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  }
  __syncthreads();

  Part Pt;
  Pt.n_g = a.n_groups;
  Pt.r = a.r;
  Pt.n_wc = (a.r + kWinTok - 1) / kWinTok;
  Pt.n_items = (int)(Pt.n_g + Pt.n_wc);
  Pt.rec = C::REC;
  Pt.tokb = 4 * D;
  Pt.W_row = Pt.n_g * C::REC + (int64_t)a.r * 4 * D;
  Pt.rows = (int64_t)gm.B * gm.Hkv;
  Pt.W_tot = Pt.rows * Pt.W_row;
  Pt.n_cta = gridDim.x;
  const int cta = blockIdx.x;
  const int64_t i0 = Pt.first_item(Pt.lo(cta));
  const int64_t i1 = Pt.first_item(Pt.lo(cta + 1));
  auto nop_seg = [](int) {};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0, qseg = 0;
      for_each_chunk<C::SG>(
          Pt, i0, i1,
          [&](int s, int row, bool win, int64_t first, int cnt) {
            if (*abort_flag) return;
            const int slot = s % C::NST;
            if (s >= C::NST && !mbar_wait(&bar_empty[slot], ((s / C::NST) - 1) & 1, abort_flag)) {
              atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
              *abort_flag = 1;
              return;
            }
            unsigned char* dst = smem + slot * C::STAGE;
            if (!win) {
              const uint32_t bytes = (uint32_t)cnt * C::REC;
              mbar_expect_tx(&bar_full[slot], bytes);
              bulk_g2s(dst, record_ptr(gm, row, first), bytes, &bar_full[slot]);
            } else {
              const int t0 = (int)first * kWinTok;
              const int n = min(kWinTok, a.r - t0);
              const int slot0 = (a.head + t0) % gm.cap;
              // two copies (key rows, value rows): a CTA's bulk copies complete
              // roughly one after another, so few large copies beat many small ones
              const uint32_t bytes = (uint32_t)n * D * 2;
              mbar_expect_tx(&bar_full[slot], 2 * bytes);
              bulk_g2s(dst, ring_ptr(gm, row, 0) + (int64_t)slot0 * D, bytes, &bar_full[slot]);
              bulk_g2s(dst + kWinTok * C::WROW, ring_ptr(gm, row, 1) + (int64_t)slot0 * D, bytes, &bar_full[slot]);
            }
            issued = s + 1;
          },
          [&](int row) {
            // q of the segment's row into ring slot k & 1
            if (*abort_flag) return;
            const int k = qseg++;
            const int qs = k & 1;
            if (k >= 2 && !mbar_wait(&bar_qempty[qs], ((k >> 1) - 1) & 1, abort_flag)) {
              atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
              *abort_flag = 1;
              return;
            }
            const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
            const uint32_t bytes = (uint32_t)gm.g * D * 2;
            mbar_expect_tx(&bar_qfull[qs], bytes);
            bulk_g2s(sm_q + qs * 8 * D, a.q + ((int64_t)b * gm.Hq + (int64_t)hkv * gm.g) * D, bytes, &bar_qfull[qs]);
          },
          nop_seg);
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        for (int s = max(0, issued - C::NST); s < issued; ++s) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&bar_full[s % C::NST], (s / C::NST) & 1) && clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
    return;
  }

  if (warp == 1) {
    // ------------------------------------------------------------ prep: beta for every group of a stage
    uint32_t qh[NKT][2];
    int qseg = 0;
    for_each_chunk<C::SG>(
        Pt, i0, i1,
        [&](int s, int row, bool win, int64_t first, int cnt) {
          const int slot = s % C::NST;
          // warp-uniform: every lane must take the mma below together
          const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_full[slot], (s / C::NST) & 1, abort_flag));
          if (!ok) {
            if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
          }
          if (ok && !win) {
            // columns of B = the stage's groups; rows of A = heads (q, exact in fp16)
            const unsigned char* st = smem + slot * C::STAGE;
            float bacc[4] = {0.f, 0.f, 0.f, 0.f};
            const int grp = gr < cnt ? gr : 0;
            const unsigned char* pz = st + grp * C::REC + C::KZOFF + 16 * tc;
#pragma unroll
            for (int i = 0; i < D / 32; ++i) {
              const uint4 z4 = lds128(pz + 64 * i);
              const uint32_t a0[4] = {qh[2 * i][0], 0u, qh[2 * i][1], 0u};
              const uint32_t a1[4] = {qh[2 * i + 1][0], 0u, qh[2 * i + 1][1], 0u};
              mma_f16_16816(bacc, a0, z4.x, z4.y);
              mma_f16_16816(bacc, a1, z4.z, z4.w);
            }
            float* bt = sm_beta + (slot * C::SG) * 8;
            // thread holds beta(head gr, groups 2tc, 2tc+1)
            if (2 * tc < cnt) bt[(2 * tc) * 8 + gr] = bacc[0];
            if (2 * tc + 1 < cnt) bt[(2 * tc + 1) * 8 + gr] = bacc[1];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_ready[slot]);
        },
        [&](int row) {
          (void)row;
          const int k = qseg++;
          const int qs = k & 1;
          const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_qfull[qs], (k >> 1) & 1, abort_flag));
          if (!ok) {
            if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
          }
          const bool hok = ok && gr < gm.g;
          const uint16_t* qrow = sm_q + qs * 8 * D + gr * D;
#pragma unroll
          for (int kt = 0; kt < NKT; ++kt)
#pragma unroll
            for (int rho = 0; rho < 2; ++rho)
              qh[kt][rho] =
                  hok ? in16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow + 16 * kt + 8 * rho + 2 * tc), gm.dtype)
                      : 0u;
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_qempty[qs]);
        },
        nop_seg);
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int cw = warp - 2;
  const bool head_ok = gr < gm.g;
  const uint32_t magic = kMagic;
  int qseg = 0;
  const uint16_t* sq = sm_q;   // ring slot of the current segment
  uint32_t qh[NKT][2];   // q of head gr at channels 16kt + 8rho + 2tc + {0, 1}, fp16x2
  float o[NNT][4];
  float m = -INFINITY, l = 0.f, wz = 0.f;
  int seg_row = 0;

  auto seg_begin = [&](int row) {
    seg_row = row;
    const int k = qseg++;
    const int qs = k & 1;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_qfull[qs], (k >> 1) & 1, abort_flag));
    if (!ok) {
      if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
    sq = sm_q + qs * 8 * D;
    const uint16_t* qrow = sq + gr * D;
    // q, pre-scaled by the position compensation of the key codes it meets:
    // pair position j' = (2kt + rho) & 3 for 2-bit, rho for 4-bit
#pragma unroll
    for (int kt = 0; kt < NKT; ++kt)
#pragma unroll
      for (int rho = 0; rho < 2; ++rho) {
        const uint32_t qv = (ok && head_ok)
                                ? in16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow + 16 * kt + 8 * rho + 2 * tc),
                                               gm.dtype)
                                : 0u;
        const int jp = BITS == 2 ? ((2 * kt + rho) & 3) : rho;
        qh[kt][rho] = h2_as_u32(__hmul2(u32_as_h2(qv), u32_as_h2(pos_comp(BITS, jp))));
      }
#pragma unroll
    for (int i = 0; i < NNT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    m = -INFINITY;
    l = 0.f;
    wz = 0.f;
  };

  // online-softmax update with this lane's scores x[] (head gr); returns nothing,
  // rescales the running state when the block max exceeds the running max
  auto rescale_to = [&](float mt) {
    // warp-uniform branch: lanes whose max did not grow scale by 1
    if (__any_sync(0xffffffffu, mt > m)) {
      const float mn = fmaxf(m, mt);
      const float alpha = fast_exp2(m - mn);
      l *= alpha;
      wz *= alpha;
#pragma unroll
      for (int i = 0; i < NNT; ++i) {
        o[i][0] *= alpha;
        o[i][1] *= alpha;
        o[i][2] *= alpha;
        o[i][3] *= alpha;
      }
      m = mn;
    }
  };

  auto chunk = [&](int s, int row, bool win, int64_t first, int cnt) {
    const int slot = s % C::NST;
    const uint32_t par = (s / C::NST) & 1;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_full[slot], par, abort_flag) &&
                                                mbar_wait(&bar_ready[slot], par, abort_flag));
    if (!ok) {
      if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
    const unsigned char* st = smem + slot * C::STAGE;
    if (ok && !win && cw < cnt * C::NTB) {
      // ---------------------------------------------------------- one quantized TB
      const int grp = cw / C::NTB, tbg = cw - grp * C::NTB;
      const unsigned char* rec = st + grp * C::REC;
      uint4 kc[P / 4];
#pragma unroll
      for (int p = 0; p < P / 4; ++p) kc[p] = lds128(rec + tbg * C::TBC + 16 * (32 * p + lane));
      const float beta = sm_beta[(slot * C::SG + grp) * 8 + gr];
      // this lane's key scales: 16 bytes per k-tile pair kt2 at 64 kt2 + 16 tc
      const unsigned char* psc = rec + C::KSOFF + 16 * tc;
      float sc[2][4][4];   // [k-tile parity][n-tile]: two independent chains per n-tile
#pragma unroll
      for (int par = 0; par < 2; ++par)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) sc[par][nt][0] = sc[par][nt][1] = sc[par][nt][2] = sc[par][nt][3] = 0.f;
#pragma unroll
      for (int wi = 0; wi < WPN; ++wi)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pr[4][J];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const int w = nt * WPN + wi;
            const uint4 pc = kc[w >> 2];
            const uint32_t word = (w & 3) == 0 ? pc.x : (w & 3) == 1 ? pc.y : (w & 3) == 2 ? pc.z : pc.w;
            unpack_half<BITS>(half ? word >> 8 : word, pr[nt], magic);
          }
#pragma unroll
          for (int m2 = 0; m2 < J / 2; ++m2) {
            const int kt = (J / 2) * (2 * wi + half) + m2;
            const uint2 s2 = *reinterpret_cast<const uint2*>(psc + 64 * (kt >> 1) + 8 * (kt & 1));
            const __half2 hi0 = __hmul2(u32_as_h2(qh[kt][0]), u32_as_h2(s2.x));
            const __half2 hi1 = __hmul2(u32_as_h2(qh[kt][1]), u32_as_h2(s2.y));
            const uint32_t aq[4] = {h2_as_u32(hi0), h2_as_u32(__hfma2(u32_as_h2(qh[kt][0]), u32_as_h2(s2.x), __hneg2(hi0))),
                                    h2_as_u32(hi1), h2_as_u32(__hfma2(u32_as_h2(qh[kt][1]), u32_as_h2(s2.y), __hneg2(hi1)))};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) mma_f16_16816(sc[kt & 1][nt], aq, pr[nt][2 * m2], pr[nt][2 * m2 + 1]);
          }
        }
      float x[4][2];
      float mt = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          x[nt][e] = ((sc[0][nt][e] + sc[1][nt][e]) + (sc[0][nt][2 + e] + sc[1][nt][2 + e]) + beta) * a.scale_log2;
          mt = fmaxf(mt, x[nt][e]);
        }
      rescale_to(quad_max(mt));
      uint32_t vm[8];
      {
        const uint4* pv = reinterpret_cast<const uint4*>(rec + C::VMOFF + 4 * (tbg * kTB + 8 * tc));
        const uint4 v0 = lds128(pv), v1 = lds128(pv + 1);
        vm[0] = v0.x; vm[1] = v0.y; vm[2] = v0.z; vm[3] = v0.w;
        vm[4] = v1.x; vm[5] = v1.y; vm[6] = v1.z; vm[7] = v1.w;
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
            const float p = fast_exp2(x[nt][e] - m);
            const uint32_t meta = vm[2 * nt + e];
            const float2 sz = __half22float2(u32_as_h2(meta));
            l += p;
            wz = fmaf(p, sz.y, wz);
            // value pair position j' = 2kt + rho (2-bit) or rho (4-bit)
            pt[e] = p * (sz.x * pos_comp_f(BITS, BITS == 2 ? 2 * kt + rr : rr));
          }
          const __half2 hi = __floats2half2_rn(pt[0], pt[1]);
          const float2 hb = __half22float2(hi);
          const __half2 lo = __floats2half2_rn(pt[0] - hb.x, pt[1] - hb.y);
          apv[kt][2 * rr] = h2_as_u32(hi);
          apv[kt][2 * rr + 1] = h2_as_u32(lo);
        }
      uint4 vc[P / 4];
#pragma unroll
      for (int p = 0; p < P / 4; ++p) vc[p] = lds128(rec + (C::NTB + tbg) * C::TBC + 16 * (32 * p + lane));
      // k-tile-major: every n-tile's kt = 0 mma before any kt = 1 mma, so the two
      // mma's into one accumulator are far apart (legacy mma.sync has a long latency)
#pragma unroll
      for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int w = 0; w < P; ++w) {
          const uint4 pc = vc[w >> 2];
          const uint32_t word = (w & 3) == 0 ? pc.x : (w & 3) == 1 ? pc.y : (w & 3) == 2 ? pc.z : pc.w;
          if (BITS == 2) {
            // pairs j' = 2kt, 2kt + 1 of both half words: n-tiles 2w (low half) and 2w + 1
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const uint32_t x = half ? word >> 8 : word;
              const uint32_t b0 = kt ? unpack_pair<2, 2>(x, magic) : unpack_pair<2, 0>(x, magic);
              const uint32_t b1 = kt ? unpack_pair<2, 3>(x, magic) : unpack_pair<2, 1>(x, magic);
              mma_f16_16816(o[2 * w + half], apv[kt], b0, b1);
            }
          } else {
            // 4-bit: half word = kt, pairs j' = 0, 1 = rho
            const uint32_t x = kt ? word >> 8 : word;
            mma_f16_16816(o[w], apv[kt], unpack_pair<4, 0>(x, magic), unpack_pair<4, 1>(x, magic));
          }
        }
    } else if (ok && win) {
      // ---------------------------------------------------------- window tokens 4cw..4cw+3 (exact 16-bit)
      // scores: rows = heads (q, exact in its own format), columns = the 8 tokens
      // from 4cw (the upper 4 belong to the next warp and are masked); P.V with
      // p split hi + lo in the same format, one 16-token k-tile of which only the
      // first 4 columns are non-zero
      const int n_tok = min(kWinTok, a.r - (int)first * kWinTok);
      const int t0 = 4 * cw;
      const unsigned char* kb = st;
      const unsigned char* vb = st + kWinTok * C::WROW;
      const bool bf = gm.dtype == KVQ_BF16;
      float sw[4] = {0.f, 0.f, 0.f, 0.f};
      const int mi = lane >> 3, ri = lane & 7;   // ldmatrix: matrix and row this lane addresses
      const int krow = min(t0 + ri, kWinTok - 1);
#pragma unroll
      for (int kt2 = 0; kt2 < NKT / 2; ++kt2) {
        uint32_t bk[4];
        ldsm_x4(bk, kb + krow * C::WROW + (16 * (2 * kt2 + (mi >> 1)) + 8 * (mi & 1)) * 2);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int kt = 2 * kt2 + h2;
          const uint32_t aq[4] = {head_ok ? *reinterpret_cast<const uint32_t*>(sq + gr * D + 16 * kt + 2 * tc) : 0u, 0u,
                                  head_ok ? *reinterpret_cast<const uint32_t*>(sq + gr * D + 16 * kt + 8 + 2 * tc) : 0u,
                                  0u};
          if (bf) mma_bf16_16816(sw, aq, bk[2 * h2], bk[2 * h2 + 1]);
          else mma_f16_16816(sw, aq, bk[2 * h2], bk[2 * h2 + 1]);
        }
      }
      float xv[2];
      float mt = -INFINITY;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = t0 + 2 * tc + e;
        const bool valid = head_ok && tc < 2 && t < n_tok;
        xv[e] = valid ? sw[e] * a.scale_log2 : -INFINITY;
        mt = fmaxf(mt, xv[e]);
      }
      rescale_to(quad_max(mt));
      float pw[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pw[e] = xv[e] == -INFINITY ? 0.f : fast_exp2(xv[e] - m);
        l += pw[e];
      }
      const uint32_t ph = pack2_in16(pw[0], pw[1], gm.dtype);
      const float2 pb = unpack2_in16(ph, gm.dtype);
      const uint32_t pl = pack2_in16(pw[0] - pb.x, pw[1] - pb.y, gm.dtype);
      const uint32_t apw[4] = {ph, pl, 0u, 0u};
      // value rows t0 + 2tc, t0 + 2tc + 1 of the k-tile: zero those past n_tok so
      // stale shared memory never meets the zero weights
      const uint32_t vmask = (t0 + 2 * tc < n_tok ? 0x0000FFFFu : 0u) | (t0 + 2 * tc + 1 < n_tok ? 0xFFFF0000u : 0u);
      const int vrow = min(t0 + ri, kWinTok - 1);
#pragma unroll
      for (int n4 = 0; n4 < NNT / 4; ++n4) {
        uint32_t bv[4];
        ldsm_x4_t(bv, vb + vrow * C::WROW + 8 * (4 * n4 + mi) * 2);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (bf) mma_bf16_16816(o[4 * n4 + j], apw, bv[j] & vmask, 0u);
          else mma_f16_16816(o[4 * n4 + j], apw, bv[j] & vmask, 0u);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_empty[slot]);
  };

  auto seg_end = [&](int row) {
    // warp states -> shared memory (consumer warps only)
    const float ls = quad_sum(l), wzs = quad_sum(wz);
    if (tc == 0) {
      sm_m[cw * 8 + gr] = m;
      sm_l[cw * 8 + gr] = ls;
    }
#pragma unroll
    for (int nt = 0; nt < NNT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) sm_o[(cw * 8 + gr) * D + 8 * nt + 2 * tc + e] = o[nt][e] + o[nt][2 + e] + wzs;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_qempty[(qseg - 1) & 1]);   // this warp is done with the segment's q
    consumer_bar();
    const int ct = threadIdx.x - 64;
    const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
    const int64_t first_it = (int64_t)row * Pt.n_items;
    const int c_first = Pt.cta_of(first_it), c_last = Pt.cta_of(first_it + Pt.n_items - 1);
    const int expected = c_last - c_first + 1;
    float* out_row = a.out + ((int64_t)b * gm.Hq + (int64_t)hkv * gm.g) * D;
    if (expected == 1) {
      for (int i = ct; i < gm.g * D; i += kConsumers * 32) {
        const int h = i / D, c = i - h * D;
        float M = -INFINITY;
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, sm_m[w * 8 + h]);
        float O = 0.f, L = 0.f;
        for (int w = 0; w < kConsumers; ++w) {
          const float f = M == -INFINITY ? 0.f : exp2f(sm_m[w * 8 + h] - M);
          O += sm_o[(w * 8 + h) * D + c] * f;
          L += sm_l[w * 8 + h] * f;
        }
        if (!*abort_flag) out_row[i] = O / L;
      }
    } else {
      float* part = a.ws + ((int64_t)(cta + row) * gm.g) * (D + 2);
      for (int i = ct; i < gm.g * (D + 2); i += kConsumers * 32) {
        const int h = i / (D + 2), c = i - h * (D + 2);
        float M = -INFINITY;
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, sm_m[w * 8 + h]);
        float val;
        if (c == D) {
          val = M;
        } else {
          val = 0.f;
          for (int w = 0; w < kConsumers; ++w) {
            const float f = M == -INFINITY ? 0.f : exp2f(sm_m[w * 8 + h] - M);
            val += (c < D ? sm_o[(w * 8 + h) * D + c] : sm_l[w * 8 + h]) * f;
          }
        }
        part[i] = val;
      }
      // The CTA barrier orders every thread's partial stores before thread 0's
      // gpu-scope acq_rel atomic (release is cumulative), so one fenced atomic
      // publishes the whole partial; the last arriver's acquire plus the next
      // barrier make every partial visible to all its threads.
      consumer_bar();
      if (ct == 0) {
        int last = 0;
        if (!*abort_flag) {
          unsigned old;
          asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;\n" : "=r"(old) : "l"(a.counters + row) : "memory");
          last = old == (unsigned)(expected - 1);
        }
        *last_flag = last;
      }
      consumer_bar();
      if (*last_flag) {
        // last CTA of the row: merge its np partials.  All loads of a step are
        // independent and issued together; the per-partial weights
        // 2^(m_j - M) / L go through shared memory (the warp-state area).
        const int np = c_last - c_first + 1;
        const int g = gm.g;
        float* pm = sm_o;                  // [np][g]
        float* pw = sm_o + np * g;         // [np][g]
        float* pl = sm_o + 2 * np * g;     // [np][g]
        float* hm = sm_o + 3 * np * g;     // [g] max, then [g] 1/L
        const float* ws_row = a.ws + (int64_t)(c_first + row) * g * (D + 2);
        for (int i = ct; i < np * g; i += kConsumers * 32) {
          pm[i] = __ldcg(ws_row + (int64_t)i * (D + 2) + D);
          pl[i] = __ldcg(ws_row + (int64_t)i * (D + 2) + D + 1);
        }
        consumer_bar();
        for (int h = ct; h < g; h += kConsumers * 32) {
          float M = -INFINITY;
          for (int j = 0; j < np; ++j) M = fmaxf(M, pm[j * g + h]);
          float L = 0.f;
          for (int j = 0; j < np; ++j) L += pm[j * g + h] == -INFINITY ? 0.f : pl[j * g + h] * exp2f(pm[j * g + h] - M);
          hm[h] = M;
          hm[g + h] = 1.f / L;
        }
        consumer_bar();
        for (int i = ct; i < np * g; i += kConsumers * 32) {
          const int h = i % g;
          pw[i] = pm[i] == -INFINITY ? 0.f : exp2f(pm[i] - hm[h]) * hm[g + h];
        }
        consumer_bar();
        for (int e = ct; e < g * D; e += kConsumers * 32) {
          const int h = e / D, c = e - h * D;
          const float* col = ws_row + (int64_t)h * (D + 2) + c;
          float acc = 0.f;
          int j = 0;
          for (; j + 8 <= np; j += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldcg(col + (int64_t)(j + u) * g * (D + 2));
#pragma unroll
            for (int u = 0; u < 8; ++u) acc = fmaf(v[u], pw[(j + u) * g + h], acc);
          }
          for (; j < np; ++j) acc = fmaf(__ldcg(col + (int64_t)j * g * (D + 2)), pw[j * g + h], acc);
          out_row[e] = acc;
        }
        if (ct == 0) a.counters[row] = 0u;
      }
    }
    consumer_bar();
  };

  for_each_chunk<C::SG>(Pt, i0, i1, chunk, seg_begin, seg_end);
}

template <int BITS, int D, int G>
void launch_decode(const AttnArgs& a, cudaStream_t st) {
  using C = K<BITS, D, G>;
  auto kern = kivi_decode_kernel<BITS, D, G>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    attr_set = true;
  }
  kern<<<a.n_cta, kThreads, C::SMEM, st>>>(a);
  count_launch(1);
}

}  // namespace

int decode_stage_bytes(int bits, int d, int G) {
  if (bits == 2 && d == 128 && G == 32) return K<2, 128, 32>::STAGE;
  if (bits == 2 && d == 64 && G == 32) return K<2, 64, 32>::STAGE;
  if (bits == 4 && d == 128 && G == 64) return K<4, 128, 64>::STAGE;
  if (bits == 4 && d == 128 && G == 32) return K<4, 128, 32>::STAGE;
  if (bits == 2 && d == 128 && G == 64) return K<2, 128, 64>::STAGE;
  if (bits == 4 && d == 64 && G == 32) return K<4, 64, 32>::STAGE;
  if (bits == 2 && d == 64 && G == 64) return K<2, 64, 64>::STAGE;
  if (bits == 4 && d == 64 && G == 64) return K<4, 64, 64>::STAGE;
  return 0;
}

void launch_kivi_attention(const AttnArgs& a, cudaStream_t st) {
  const Geom& g = a.geom;
  if (g.bits == 2 && g.d == 128 && g.G == 32) launch_decode<2, 128, 32>(a, st);
  else if (g.bits == 2 && g.d == 64 && g.G == 32) launch_decode<2, 64, 32>(a, st);
  else if (g.bits == 4 && g.d == 128 && g.G == 64) launch_decode<4, 128, 64>(a, st);
  else if (g.bits == 4 && g.d == 128 && g.G == 32) launch_decode<4, 128, 32>(a, st);
  else if (g.bits == 2 && g.d == 128 && g.G == 64) launch_decode<2, 128, 64>(a, st);
  else if (g.bits == 4 && g.d == 64 && g.G == 32) launch_decode<4, 64, 32>(a, st);
  else if (g.bits == 2 && g.d == 64 && g.G == 64) launch_decode<2, 64, 64>(a, st);
  else if (g.bits == 4 && g.d == 64 && g.G == 64) launch_decode<4, 64, 64>(a, st);
}

}  // namespace kvq

// ------------------------------------------------------------------ decode attention without caller scratch
// For callers that cannot allocate device memory (see kvq_decode_attention_static
// in kvq.h): the split-K partial states go to this fixed array instead of a
// caller workspace.  The counters the kernel needs are in the cache buffer, so
// nothing here has to start at zero.
namespace kvq {
static __device__ __align__(256) unsigned char g_static_ws[KVQ_STATIC_WORKSPACE_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mutex;
void* g_static_ws_addr[kMaxDevices] = {};

// Device address of g_static_ws on the current device.  The host-side name
// g_static_ws is only a stand-in; the address is looked up once per device,
// with that device current.
kvq_status static_ws_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  if (g_static_ws_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_static_ws) != cudaSuccess || ptr == nullptr) return KVQ_ERR_CUDA;
    g_static_ws_addr[dev] = ptr;
  }
  *out = g_static_ws_addr[dev];
  return KVQ_OK;
}
}  // namespace
}  // namespace kvq

extern "C" kvq_status kvq_decode_attention_static(const kvq_cache* cache, const void* q, float* out,
                                                  float softmax_scale, void* stream) {
  if (!cache) return KVQ_ERR_INVALID_ARG;
  const size_t need = kvq::cache_workspace_bytes(cache);
  if (need == 0) return KVQ_ERR_INVALID_ARG;
  if (need > KVQ_STATIC_WORKSPACE_BYTES) return KVQ_ERR_CAPACITY;
  void* ws = nullptr;
  const kvq_status st = kvq::static_ws_address(&ws);
  if (st != KVQ_OK) return st;
  return kvq_decode_attention(cache, q, out, softmax_scale, ws, KVQ_STATIC_WORKSPACE_BYTES, stream);
}

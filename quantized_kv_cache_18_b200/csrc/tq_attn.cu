// TurboQuant-style decode attention straight from the packed cache.
//
// Scores and values of a quantized token come from its codes c_hat, norms and
// sketch ("Quantification du KV-Cache : TurboQuant et l'etat de l'art en
// 2026", "TurboQuant : les cinq innovations", items 1-3; zubnet.ai survey,
// "Famille deux ..."):
//   score_t = n_t <Pi q, c_hat_t> + gamma_t sqrt(pi/2)/m <S Pi q, sign_t>
//   o       = Pi^T sum_t p_t n_t c_hat_t  +  sum_{window} p_t v_t
// The second score term is the 1-bit QJL estimate of n_t <Pi q, e_t>; sign_t
// is in {-1, +1}.  Pi q and S Pi q arrive pre-split into fp16 hi + lo parts
// (tq_query_prep_kernel) and sit in the two 8-row halves of the m16 A operand;
// the B operands are exact fp16: codebook levels from a 64-entry pair table in
// shared memory, and +-1 built from the sign bits with one LOP3.
//
// Structure as the KIVI decode kernel: one CTA per SM, a producer warp feeding
// a ring of shared-memory stages with 1-D bulk copies (no multicast), eleven
// consumer warps each taking one 32-token block of a stage.  A row's items are
// its token blocks, then its 32-token window chunks; the two kinds form
// separate segments because their partial outputs live in different bases
// (rotated, original).  At the end of a rotated segment the CTA applies Pi^T
// to its merged partial (Pi is copied into shared memory once per CTA), so
// every partial state (m, l, o) is in the original basis and the last CTA to
// finish a row merges them with a globally normalised log-sum-exp, as
// Minima-KV merges partial attention states ("KV-cache compresse et modeles
// 4-bit ...", section "Minima-KV : la compression sans eviction").
//
// Every wait is bounded; on expiry the CTA sets KVQ_DEV_WAIT_TIMEOUT and stops
// computing, and the producer waits (bounded) for its copies in flight.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "decode_common.cuh"

namespace kvq {

namespace {

constexpr int kTqConsumers = kTqDecodeConsumers;
constexpr int kTqThreads = (kTqConsumers + 1) * 32;
constexpr int kTqWin = kDecodeWinTok;

struct TL {
  static constexpr int D = kTqD;
  static constexpr int NKT = D / 16;
  static constexpr int NNT = D / 8;
  static constexpr int SG = kTqConsumers;                          // token blocks per stage
  static constexpr int WROW = D * 2;
  static constexpr int WINB = kTqWin * WROW * 2;
  static constexpr int STAGE = ((SG * kTqTbBytes > WINB ? SG * kTqTbBytes : WINB) + 127) / 128 * 128;
  static constexpr int NST = 2;
  static constexpr int QRAW = 8 * D * 2;                          // raw 16-bit q of up to 8 heads
  static constexpr int QSLOT = kTqQPrepBytes + QRAW;
  static constexpr int OFF_PI = NST * STAGE;                      // float [D][D], Pi[j][c]
  static constexpr int OFF_LUT = OFF_PI + D * D * 4;              // uint32 [64][32]: pair table per lane
  static constexpr int OFF_M = OFF_LUT + 64 * 32 * 4;
  static constexpr int OFF_L = OFF_M + kTqConsumers * 8 * 4;
  static constexpr int OFF_HM = OFF_L + kTqConsumers * 8 * 4;    // merged m, l per head [2][8]
  static constexpr int OFF_O = OFF_HM + 2 * 8 * 4;
  static constexpr int OFF_Q = OFF_O + kTqConsumers * 8 * D * 4;
  static constexpr int OFF_BAR = OFF_Q + 2 * QSLOT;
  static constexpr int N_BAR = 2 * NST + 5;
  static constexpr int OFF_FLAG = OFF_BAR + N_BAR * 8;
  static constexpr int OFF_ZERO = (OFF_FLAG + 16 + 15) / 16 * 16;   // a zero 16-bit row (FP8 chunks)
  static constexpr int SMEM = OFF_ZERO + WROW;
  // FP8 window / anchor chunk in a stage: K rows [32][144], V rows [32][144],
  // then each consumer warp's fp16 rows of its 4 tokens (K 1 KB, V 1 KB)
  static constexpr int FP8_SCR = 2 * kTqWin * kFp8RowBytes;
  static_assert(FP8_SCR + kTqConsumers * 2048 <= STAGE, "FP8 chunk scratch exceeds a stage");
};
static_assert(TL::SMEM <= 227 * 1024, "TurboQuant decode kernel exceeds shared memory");

__device__ __forceinline__ void tq_consumer_bar() { named_bar_sync<kTqConsumers * 32>(); }

// byte offset (index * 128) into the per-lane pair table of field f of a code word
template <int F>
__device__ __forceinline__ uint32_t lut_off(uint32_t w) {
  if constexpr (6 * F >= 7) return (w >> (6 * F - 7)) & 0x1F80u;
  else return (w << (7 - 6 * F)) & 0x1F80u;
}
template <int SLOT>
__device__ __forceinline__ uint32_t lut_pair(const uint32_t* words, const unsigned char* lut_lane) {
  return *reinterpret_cast<const uint32_t*>(lut_lane + lut_off<SLOT % 5>(words[SLOT / 5]));
}
// fp16x2 (+-1, +-1) from sign bits Q (low half) and 16 + Q (high half) of w
template <int Q>
__device__ __forceinline__ uint32_t sign_pair(uint32_t w) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;\n" : "=r"(r) : "r"(w << (15 - Q)), "n"(0x80008000u), "n"(0xBC00BC00u));
  return r;   // ((w << (15 - Q)) & 0x80008000) ^ 0xBC00BC00: bit 1 -> +1.0, bit 0 -> -1.0
}

// Work partition: items of a row are n_tb token blocks then n_wc window-type
// chunks; the host cuts the (row, item) sequence into stage-balanced CTA ranges
// (item0 in the launch arguments, read from the grid-constant parameter space).
struct TPart {
  int n_tb, n_items, n_wc, n_cta;
  const int32_t* item0;   // [n_cta + 1]
  __device__ int row_of(int item) const { return item / n_items; }
  // CTA owning an item: the largest c with item0[c] <= item
  __device__ int cta_of(int item) const {
    int lo = 0, hi = n_cta - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (item0[mid] <= item) lo = mid;
      else hi = mid - 1;
    }
    return lo;
  }
};

// f(stage, row, is_window, first, count) per chunk; seg(row, part) before and
// seg_end(row, part) after the token blocks (part 0) and the window chunks
// (part 1) a CTA owns in a row.
template <class FC, class FS, class FE>
__device__ __forceinline__ void tq_for_each_chunk(const TPart& P, int i0, int i1, FC f, FS seg, FE seg_end) {
  int s = 0;
  if (i0 >= i1) return;
  for (int row = P.row_of(i0); row * P.n_items < i1; ++row) {
    const int a = max(i0, row * P.n_items) - row * P.n_items;
    const int b = min(i1, (row + 1) * P.n_items) - row * P.n_items;
    if (a >= b) continue;
    if (a < P.n_tb) {
      seg(row, 0);
      for (int k = a; k < min(b, P.n_tb); k += TL::SG) {
        const int cnt = min(TL::SG, min(b, P.n_tb) - k);
        f(s++, row, false, (int64_t)k, cnt);
      }
      seg_end(row, 0);
    }
    if (b > P.n_tb) {
      seg(row, 1);
      for (int k = max(a, P.n_tb); k < b; ++k) f(s++, row, true, (int64_t)(k - P.n_tb), 1);
      seg_end(row, 1);
    }
  }
}

__global__ void __launch_bounds__(kTqThreads, 1) tq_decode_kernel(const __grid_constant__ AttnArgs a) {
  using C = TL;
  constexpr int D = C::D, NKT = C::NKT, NNT = C::NNT;

  extern __shared__ __align__(128) unsigned char smem[];
  float* sm_pi = reinterpret_cast<float*>(smem + C::OFF_PI);
  uint32_t* sm_lut = reinterpret_cast<uint32_t*>(smem + C::OFF_LUT);
  float* sm_m = reinterpret_cast<float*>(smem + C::OFF_M);
  float* sm_l = reinterpret_cast<float*>(smem + C::OFF_L);
  float* sm_hm = reinterpret_cast<float*>(smem + C::OFF_HM);
  float* sm_o = reinterpret_cast<float*>(smem + C::OFF_O);
  unsigned char* sm_q = smem + C::OFF_Q;
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_empty = bar_full + C::NST;
  uint64_t* bar_qfull = bar_empty + C::NST;    // [2]
  uint64_t* bar_qempty = bar_qfull + 2;        // [2]
  uint64_t* bar_pi = bar_qempty + 2;           // [1]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);
  volatile int* last_flag = abort_flag + 1;

  const Geom& gm = a.geom;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, tc = lane & 3;
  const long long wl = a.wait_cycles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], kTqConsumers);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_qfull[i], 1);
      mbar_init(&bar_qempty[i], kTqConsumers);
    }
    mbar_init(bar_pi, 1);
    *abort_flag = 0;
    for (int i = 0; i < C::WROW / 16; ++i) reinterpret_cast<uint4*>(smem + C::OFF_ZERO)[i] = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  }
  __syncthreads();

  TPart Pt;
  Pt.n_tb = (int)a.n_groups;
  // window-type items: the window's chunks, then (mixed cache) the anchors' chunks
  Pt.n_items = a.n_items;
  Pt.n_wc = a.n_items - Pt.n_tb;
  Pt.n_cta = a.n_cta;
  Pt.item0 = a.item0;
  const int n_wcw = (a.r + kTqWin - 1) / kTqWin;   // window chunks (the anchors' chunks follow)
  const int cta = blockIdx.x;
  const int i0 = a.item0[cta];
  const int i1 = a.item0[cta + 1];
  auto nop_seg = [](int, int) {};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(bar_pi, D * D * 4);
      bulk_g2s(sm_pi, gm.params + kTqPi, D * D * 4, bar_pi);
      int issued = 0, qseg = 0, qissued = 0, withheld = -1;
      tq_for_each_chunk(
          Pt, i0, i1,
          [&](int s, int row, bool win, int64_t first, int cnt) {
            if (*abort_flag) return;
            const int slot = s % C::NST;
            // a paged stage's page ids load while the producer waits for the slot
            // (a contiguous cache skips all page bookkeeping: this thread's
            // per-stage work is on the critical path)
            const bool paged = !win && gm.page_table != nullptr;
            RecordPages pages;
            if (paged) record_pages(gm, row, first, cnt, pages);
            if (s >= C::NST && !mbar_wait(&bar_empty[slot], ((s / C::NST) - 1) & 1, abort_flag, wl)) {
              atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
              *abort_flag = 1;
              return;
            }
            // consumers that gave up on this slot's previous copy set the flag
            // before releasing the slot: that copy may still be in flight
            if (*abort_flag) return;
            if (s == 0 && cta == 0 && a.withhold_first_stage) {
              withheld = 0;   // test hook: a stage whose wait nothing completes
              issued = 1;
              return;
            }
            unsigned char* dst = smem + slot * C::STAGE;
            if (!win && !paged) {
              const uint32_t bytes = (uint32_t)cnt * kTqTbBytes;
              mbar_expect_tx(&bar_full[slot], bytes);
              bulk_g2s(dst, record_ptr(gm, row, first), bytes, &bar_full[slot]);
            } else if (!win) {
              if (!pages_valid(gm, pages)) {
                atomicOr(gm.status, KVQ_DEV_BAD_PAGE);
                *abort_flag = 1;
                return;
              }
              copy_records(gm, row, first, cnt, kTqTbBytes, pages, dst, &bar_full[slot]);
            } else if (gm.fp8) {
              // FP8 token rows of a window chunk (ring) or an anchor chunk
              const int j = (int)first;
              const unsigned char *srck, *srcv;
              int n;
              if (j < n_wcw) {
                const int t0 = j * kTqWin;
                n = min(kTqWin, a.r - t0);
                const int slot0 = (a.head + t0) % gm.cap;
                srck = reinterpret_cast<const unsigned char*>(gm.window) +
                       ((int64_t)row * 2 * gm.cap + slot0) * kFp8RowBytes;
                srcv = srck + (int64_t)gm.cap * kFp8RowBytes;
              } else {
                const int t0 = (j - n_wcw) * kTqWin;
                n = kTqWin;
                srck = gm.anchors + ((int64_t)row * 2 * gm.anchor + t0) * kFp8RowBytes;
                srcv = srck + (int64_t)gm.anchor * kFp8RowBytes;
              }
              const uint32_t bytes = (uint32_t)n * kFp8RowBytes;
              mbar_expect_tx(&bar_full[slot], 2 * bytes);
              bulk_g2s(dst, srck, bytes, &bar_full[slot]);
              bulk_g2s(dst + kTqWin * kFp8RowBytes, srcv, bytes, &bar_full[slot]);
            } else {
              const int t0 = (int)first * kTqWin;
              const int n = min(kTqWin, a.r - t0);
              const int slot0 = (a.head + t0) % gm.cap;
              // with a fused append the chunk's last token comes from k_new / v_new
              const bool fused = a.k_new != nullptr && t0 + n == a.r;
              const int n_ring = fused ? n - 1 : n;
              mbar_expect_tx(&bar_full[slot], 2u * (uint32_t)n * D * 2);
              if (n_ring > 0) {
                const uint32_t bytes = (uint32_t)n_ring * D * 2;
                bulk_g2s(dst, ring_ptr(gm, row, 0) + (int64_t)slot0 * D, bytes, &bar_full[slot]);
                bulk_g2s(dst + kTqWin * C::WROW, ring_ptr(gm, row, 1) + (int64_t)slot0 * D, bytes, &bar_full[slot]);
              }
              if (fused) {
                bulk_g2s(dst + n_ring * C::WROW, a.k_new + (int64_t)row * D, D * 2, &bar_full[slot]);
                bulk_g2s(dst + (kTqWin + n_ring) * C::WROW, a.v_new + (int64_t)row * D, D * 2, &bar_full[slot]);
              }
            }
            issued = s + 1;
          },
          [&](int row, int part) {
            // the segment's query data into ring slot k & 1: rotated fragments
            // for token blocks, raw q for window chunks
            if (*abort_flag) return;
            const int k = qseg++;
            const int qs = k & 1;
            if (k >= 2 && !mbar_wait(&bar_qempty[qs], ((k >> 1) - 1) & 1, abort_flag, wl)) {
              atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
              *abort_flag = 1;
              return;
            }
            if (*abort_flag) return;
            qissued = k + 1;
            unsigned char* dq = sm_q + qs * C::QSLOT;
            if (part == 0) {
              mbar_expect_tx(&bar_qfull[qs], kTqQPrepBytes);
              bulk_g2s(dq, a.qprep + (int64_t)row * kTqQPrepBytes, kTqQPrepBytes, &bar_qfull[qs]);
            } else {
              const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
              const uint32_t bytes = (uint32_t)gm.g * D * 2;
              mbar_expect_tx(&bar_qfull[qs], bytes);
              bulk_g2s(dq + kTqQPrepBytes, a.q + ((int64_t)b * gm.Hq + (int64_t)hkv * gm.g) * D, bytes,
                       &bar_qfull[qs]);
            }
          },
          nop_seg);
      // Every copy issued lands before this warp exits (only the last NST
      // stages, the last two query slots and the Pi copy can still be in
      // flight), so none can write shared memory after the CTA is gone, even
      // when its consumers gave up waiting.
      for (int s = max(0, issued - C::NST); s < issued; ++s)
        if (s != withheld) mbar_drain(&bar_full[s % C::NST], (s / C::NST) & 1);
      for (int k = max(0, qissued - 2); k < qissued; ++k) mbar_drain(&bar_qfull[k & 1], (k >> 1) & 1);
      mbar_drain(bar_pi, 0);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int cw = warp - 1;
  const int ct = threadIdx.x - 32;
  const bool head_ok = gr < gm.g;
  // GQA groups of up to 4 heads run the token blocks in the token-major
  // formulation (codes as the A operand, the heads' hi | lo parts as the 8
  // columns of B): half the mma's of the head-major form, whose 8 hi | lo rows
  // such a group only half fills.  Window chunks stay head-major.
  const bool tr = gm.g <= 4;
  {
    // per-lane copy of the pair table: entry idx of lane L at [idx][L]
    const uint32_t* lut_g = reinterpret_cast<const uint32_t*>(gm.params + kTqLut);
    for (int e = ct; e < 64 * 32; e += kTqConsumers * 32) sm_lut[e] = __ldg(lut_g + (e >> 5));
  }
  tq_consumer_bar();
  const unsigned char* lut_lane = reinterpret_cast<const unsigned char*>(sm_lut + lane);
  bool pi_ready = false;
  int qseg = 0;
  const unsigned char* sq = sm_q;   // ring slot of the current segment
  uint32_t qa[NKT][4];              // Pi q fragments (hi, lo) of k-tile kt
  float o[NNT][4];
  float m = -INFINITY, l = 0.f;

  auto seg_begin = [&](int row, int part) {
    (void)row;
    const int k = qseg++;
    const int qs = k & 1;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_qfull[qs], (k >> 1) & 1, abort_flag, wl));
    if (!ok) {
      if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
    sq = sm_q + qs * C::QSLOT;
    if (part == 0) {
#pragma unroll
      for (int kt = 0; kt < NKT; ++kt) {
        const uint4 v = ok ? lds128(sq + (kt * 32 + lane) * 16) : make_uint4(0u, 0u, 0u, 0u);
        qa[kt][0] = v.x;
        qa[kt][1] = v.y;
        qa[kt][2] = v.z;
        qa[kt][3] = v.w;
      }
      if (tr) {
        // token-major: B operands, column n = head n >> 1, part n & 1 (hi | lo),
        // taken from the A fragments (rows = heads hi | lo) of lane (n >> 1, tc):
        // qa[kt][0..1] = Pi q, qa[kt][2..3] = S Pi q
        const int src = (gr >> 1) * 4 + tc;
        const bool lo = (gr & 1) != 0;
#pragma unroll
        for (int kt = 0; kt < NKT; ++kt) {
          const uint4 w = ok ? lds128(sq + ((NKT + kt) * 32 + lane) * 16) : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t s0 = __shfl_sync(0xffffffffu, qa[kt][0], src), s1 = __shfl_sync(0xffffffffu, qa[kt][1], src);
          const uint32_t s2 = __shfl_sync(0xffffffffu, qa[kt][2], src), s3 = __shfl_sync(0xffffffffu, qa[kt][3], src);
          const uint32_t t0 = __shfl_sync(0xffffffffu, w.x, src), t1 = __shfl_sync(0xffffffffu, w.y, src);
          const uint32_t t2 = __shfl_sync(0xffffffffu, w.z, src), t3 = __shfl_sync(0xffffffffu, w.w, src);
          qa[kt][0] = lo ? s1 : s0;
          qa[kt][1] = lo ? s3 : s2;
          qa[kt][2] = lo ? t1 : t0;
          qa[kt][3] = lo ? t3 : t2;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NNT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    m = -INFINITY;
    l = 0.f;
  };

  auto rescale_to = [&](float mt) {
    if (__any_sync(0xffffffffu, mt > m)) {
      const float mn = fmaxf(m, mt);
      const float alpha = fast_exp2(m - mn);
      l *= alpha;
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
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_full[slot], par, abort_flag, wl));
    if (!ok) {
      if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
    const unsigned char* st = smem + slot * C::STAGE;
    if (ok && win && a.k_new != nullptr && cw == kTqConsumers - 1) {
      // fused append: the new token of this row (the chunk's last) into its ring slot
      const int t0 = (int)first * kTqWin;
      const int n = min(kTqWin, a.r - t0);
      if (t0 + n == a.r) {
        const int slot_new = (a.head + a.r - 1) % gm.cap;
        constexpr int CH = D * 2 / 16;   // 16-byte chunks per row
        if (lane < 2 * CH) {
          const int part = lane / CH, ci = lane - part * CH;
          const uint4 v = lds128(st + (part * kTqWin + n - 1) * C::WROW + 16 * ci);
          reinterpret_cast<uint4*>(ring_ptr(gm, row, part) + (int64_t)slot_new * D)[ci] = v;
        }
      }
    }
    if (ok && !win && cw < cnt && tr) {
      // ---------------------------------------------------------- one token block, token-major
      // A fragment of token m-tile MT = the B fragments of token n-tiles 2MT,
      // 2MT + 1 of the packed format; lane (gr, tc) gets the scores of head tc,
      // tokens gr + 8i, and the output of head tc, channels 16MT + gr (+8).
      const unsigned char* tb = st + cw * kTqTbBytes;
      float sc[2][4], ss[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[mt][e] = ss[mt][e] = 0.f;
      {
        uint32_t kw[13];
        const uint4 w0 = lds128(tb + kTqKCodes + 16 * lane), w1 = lds128(tb + kTqKCodes + 512 + 16 * lane),
                    w2 = lds128(tb + kTqKCodes + 1024 + 16 * lane);
        kw[0] = w0.x; kw[1] = w0.y; kw[2] = w0.z; kw[3] = w0.w;
        kw[4] = w1.x; kw[5] = w1.y; kw[6] = w1.z; kw[7] = w1.w;
        kw[8] = w2.x; kw[9] = w2.y; kw[10] = w2.z; kw[11] = w2.w;
        kw[12] = *reinterpret_cast<const uint32_t*>(tb + kTqKCodes + 1536 + 4 * lane);
        // <Pi q, c_hat>: key pair slot 16 nt + 2 kt + rho of token n-tile nt
#define TQ_TR_KEY(KT)                                                                                \
  {                                                                                                  \
    const uint32_t a0[4] = {lut_pair<2 * KT>(kw, lut_lane), lut_pair<16 + 2 * KT>(kw, lut_lane),     \
                            lut_pair<1 + 2 * KT>(kw, lut_lane), lut_pair<17 + 2 * KT>(kw, lut_lane)}; \
    mma_f16_16816(sc[0], a0, qa[KT][0], qa[KT][1]);                                                  \
    const uint32_t a1[4] = {lut_pair<32 + 2 * KT>(kw, lut_lane), lut_pair<48 + 2 * KT>(kw, lut_lane), \
                            lut_pair<33 + 2 * KT>(kw, lut_lane), lut_pair<49 + 2 * KT>(kw, lut_lane)}; \
    mma_f16_16816(sc[1], a1, qa[KT][0], qa[KT][1]);                                                  \
  }
        TQ_TR_KEY(0) TQ_TR_KEY(1) TQ_TR_KEY(2) TQ_TR_KEY(3) TQ_TR_KEY(4) TQ_TR_KEY(5) TQ_TR_KEY(6) TQ_TR_KEY(7)
#undef TQ_TR_KEY
      }
      {
        // <S Pi q, sign>: sign word nt of the lane, bits 2 kt + rho and 16 + 2 kt + rho
        const uint4 swv = lds128(tb + kTqSigns + 16 * lane);
        const uint32_t sw[4] = {swv.x, swv.y, swv.z, swv.w};
#define TQ_TR_SGN(KT)                                                                                 \
  {                                                                                                   \
    const uint32_t a0[4] = {sign_pair<2 * KT>(sw[0]), sign_pair<2 * KT>(sw[1]), sign_pair<2 * KT + 1>(sw[0]), \
                            sign_pair<2 * KT + 1>(sw[1])};                                            \
    mma_f16_16816(ss[0], a0, qa[KT][2], qa[KT][3]);                                                   \
    const uint32_t a1[4] = {sign_pair<2 * KT>(sw[2]), sign_pair<2 * KT>(sw[3]), sign_pair<2 * KT + 1>(sw[2]), \
                            sign_pair<2 * KT + 1>(sw[3])};                                            \
    mma_f16_16816(ss[1], a1, qa[KT][2], qa[KT][3]);                                                   \
  }
        TQ_TR_SGN(0) TQ_TR_SGN(1) TQ_TR_SGN(2) TQ_TR_SGN(3) TQ_TR_SGN(4) TQ_TR_SGN(5) TQ_TR_SGN(6) TQ_TR_SGN(7)
#undef TQ_TR_SGN
      }
      // meta of token gr + 8i: entry 8 (gr >> 1) + 2i + (gr & 1) (key: n, gamma; value: n)
      const int e0 = 8 * (gr >> 1) + (gr & 1);
      const uint32_t* kmw = reinterpret_cast<const uint32_t*>(tb + kTqKMeta);
      const uint16_t* vnw = reinterpret_cast<const uint16_t*>(tb + kTqVMeta);
      float x[4];
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int mt = i >> 1, e2 = i & 1;
        const float2 ng = __half22float2(u32_as_h2(kmw[e0 + 2 * i]));
        const float main = sc[mt][2 * e2] + sc[mt][2 * e2 + 1];
        const float corr = ss[mt][2 * e2] + ss[mt][2 * e2 + 1];
        x[i] = fmaf(ng.x, main, ng.y * a.qjl_c * corr) * a.scale_log2;
        mx = fmaxf(mx, x[i]);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      rescale_to(mx);
      uint32_t pp[4];   // (hi, lo) of p~ = p n_v, head tc, token gr + 8i
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float p = fast_exp2(x[i] - m);
        l += p;
        const float pt = p * __half2float(__ushort_as_half(vnw[e0 + 2 * i]));
        const __half hi = __float2half_rn(pt);
        const __half lo = __float2half_rn(pt - __half2float(hi));
        pp[i] = h2_as_u32(__halves2half2(hi, lo));
      }
      // B fragments of P.V (k = tokens 16 kt + 2 tc (+1, +8, +9), column gr =
      // head gr >> 1, hi | lo) from the lanes holding those tokens
      const int la = 8 * tc + (gr >> 1), lb = la + 4;
      const uint32_t psel = (gr & 1) ? 0x7632u : 0x5410u;
      uint32_t bp[2][2];
#pragma unroll
      for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t xa = __shfl_sync(0xffffffffu, pp[2 * kt + h], la);
          const uint32_t xb = __shfl_sync(0xffffffffu, pp[2 * kt + h], lb);
          bp[kt][h] = __byte_perm(xa, xb, psel);
        }
      {
        uint32_t vw[13];
        const uint4 w0 = lds128(tb + kTqVCodes + 16 * lane), w1 = lds128(tb + kTqVCodes + 512 + 16 * lane),
                    w2 = lds128(tb + kTqVCodes + 1024 + 16 * lane);
        vw[0] = w0.x; vw[1] = w0.y; vw[2] = w0.z; vw[3] = w0.w;
        vw[4] = w1.x; vw[5] = w1.y; vw[6] = w1.z; vw[7] = w1.w;
        vw[8] = w2.x; vw[9] = w2.y; vw[10] = w2.z; vw[11] = w2.w;
        vw[12] = *reinterpret_cast<const uint32_t*>(tb + kTqVCodes + 1536 + 4 * lane);
        // value pair slot 32 kt + 2 nt + rho of channel n-tile nt; A of channel
        // m-tile MT = n-tiles 2MT, 2MT + 1
#define TQ_TR_PV(KT, MT)                                                                                      \
  {                                                                                                           \
    const uint32_t av[4] = {lut_pair<32 * KT + 4 * MT>(vw, lut_lane), lut_pair<32 * KT + 4 * MT + 2>(vw, lut_lane), \
                            lut_pair<32 * KT + 4 * MT + 1>(vw, lut_lane), lut_pair<32 * KT + 4 * MT + 3>(vw, lut_lane)}; \
    mma_f16_16816(o[MT], av, bp[KT][0], bp[KT][1]);                                                          \
  }
#define TQ_TR_PV_KT(KT) \
  TQ_TR_PV(KT, 0) TQ_TR_PV(KT, 1) TQ_TR_PV(KT, 2) TQ_TR_PV(KT, 3) TQ_TR_PV(KT, 4) TQ_TR_PV(KT, 5) TQ_TR_PV(KT, 6) TQ_TR_PV(KT, 7)
        TQ_TR_PV_KT(0) TQ_TR_PV_KT(1)
#undef TQ_TR_PV_KT
#undef TQ_TR_PV
      }
    } else if (ok && !win && cw < cnt) {
      // ---------------------------------------------------------- one token block, head-major
      const unsigned char* tb = st + cw * kTqTbBytes;
      float sc[4][4], ss[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = ss[nt][e] = 0.f;
      {
        uint32_t kw[13];
        const uint4 w0 = lds128(tb + kTqKCodes + 16 * lane), w1 = lds128(tb + kTqKCodes + 512 + 16 * lane),
                    w2 = lds128(tb + kTqKCodes + 1024 + 16 * lane);
        kw[0] = w0.x; kw[1] = w0.y; kw[2] = w0.z; kw[3] = w0.w;
        kw[4] = w1.x; kw[5] = w1.y; kw[6] = w1.z; kw[7] = w1.w;
        kw[8] = w2.x; kw[9] = w2.y; kw[10] = w2.z; kw[11] = w2.w;
        kw[12] = *reinterpret_cast<const uint32_t*>(tb + kTqKCodes + 1536 + 4 * lane);
        // <Pi q, c_hat>: key pair slot 16 nt + 2 kt + rho
#define TQ_KEY_KT(KT)                                                                                     \
  mma_f16_16816(sc[0], qa[KT], lut_pair<0 + 2 * KT>(kw, lut_lane), lut_pair<1 + 2 * KT>(kw, lut_lane));   \
  mma_f16_16816(sc[1], qa[KT], lut_pair<16 + 2 * KT>(kw, lut_lane), lut_pair<17 + 2 * KT>(kw, lut_lane)); \
  mma_f16_16816(sc[2], qa[KT], lut_pair<32 + 2 * KT>(kw, lut_lane), lut_pair<33 + 2 * KT>(kw, lut_lane)); \
  mma_f16_16816(sc[3], qa[KT], lut_pair<48 + 2 * KT>(kw, lut_lane), lut_pair<49 + 2 * KT>(kw, lut_lane));
        TQ_KEY_KT(0) TQ_KEY_KT(1) TQ_KEY_KT(2) TQ_KEY_KT(3) TQ_KEY_KT(4) TQ_KEY_KT(5) TQ_KEY_KT(6) TQ_KEY_KT(7)
#undef TQ_KEY_KT
      }
      {
        // <S Pi q, sign>: sign word nt of the lane, bits 2 kt + rho and 16 + 2 kt + rho
        const uint4 swv = lds128(tb + kTqSigns + 16 * lane);
        const uint32_t sw[4] = {swv.x, swv.y, swv.z, swv.w};
#define TQ_SGN_KT(KT)                                                                     \
  {                                                                                       \
    const uint4 qv = lds128(sq + ((NKT + KT) * 32 + lane) * 16);                          \
    const uint32_t aq[4] = {qv.x, qv.y, qv.z, qv.w};                                      \
    _Pragma("unroll") for (int nt = 0; nt < 4; ++nt)                                      \
        mma_f16_16816(ss[nt], aq, sign_pair<2 * KT>(sw[nt]), sign_pair<2 * KT + 1>(sw[nt])); \
  }
        TQ_SGN_KT(0) TQ_SGN_KT(1) TQ_SGN_KT(2) TQ_SGN_KT(3) TQ_SGN_KT(4) TQ_SGN_KT(5) TQ_SGN_KT(6) TQ_SGN_KT(7)
#undef TQ_SGN_KT
      }
      // key meta of tokens 8 nt + 2 tc + e: entries 8 tc + 2 nt + e
      uint32_t km[8];
      {
        const uint4 m0 = lds128(tb + kTqKMeta + 32 * tc), m1 = lds128(tb + kTqKMeta + 32 * tc + 16);
        km[0] = m0.x; km[1] = m0.y; km[2] = m0.z; km[3] = m0.w;
        km[4] = m1.x; km[5] = m1.y; km[6] = m1.z; km[7] = m1.w;
      }
      float x[4][2];
      float mt = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float2 ng = __half22float2(u32_as_h2(km[2 * nt + e]));
          const float main = sc[nt][e] + sc[nt][2 + e];
          const float corr = ss[nt][e] + ss[nt][2 + e];
          x[nt][e] = fmaf(ng.x, main, ng.y * a.qjl_c * corr) * a.scale_log2;
          mt = fmaxf(mt, x[nt][e]);
        }
      rescale_to(quad_max(mt));
      // value norms of the same tokens: fp16 entries 8 tc + 2 nt + e
      const uint4 vnv = lds128(tb + kTqVMeta + 16 * tc);
      const uint32_t vn[4] = {vnv.x, vnv.y, vnv.z, vnv.w};
      uint32_t apv[2][4];
#pragma unroll
      for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int nt = 2 * kt + rr;
          const float2 nv = __half22float2(u32_as_h2(vn[nt]));
          const float p0 = fast_exp2(x[nt][0] - m), p1 = fast_exp2(x[nt][1] - m);
          l += p0 + p1;
          const float pt0 = p0 * nv.x, pt1 = p1 * nv.y;
          const __half2 hi = __floats2half2_rn(pt0, pt1);
          const float2 hb = __half22float2(hi);
          const __half2 lo = __floats2half2_rn(pt0 - hb.x, pt1 - hb.y);
          apv[kt][2 * rr] = h2_as_u32(hi);
          apv[kt][2 * rr + 1] = h2_as_u32(lo);
        }
      {
        uint32_t vw[13];
        const uint4 w0 = lds128(tb + kTqVCodes + 16 * lane), w1 = lds128(tb + kTqVCodes + 512 + 16 * lane),
                    w2 = lds128(tb + kTqVCodes + 1024 + 16 * lane);
        vw[0] = w0.x; vw[1] = w0.y; vw[2] = w0.z; vw[3] = w0.w;
        vw[4] = w1.x; vw[5] = w1.y; vw[6] = w1.z; vw[7] = w1.w;
        vw[8] = w2.x; vw[9] = w2.y; vw[10] = w2.z; vw[11] = w2.w;
        vw[12] = *reinterpret_cast<const uint32_t*>(tb + kTqVCodes + 1536 + 4 * lane);
        // sum_t p~_t c_hat_t: value pair slot 32 kt + 2 nt + rho, k-tile-major
#define TQ_PV(KT, NT) \
  mma_f16_16816(o[NT], apv[KT], lut_pair<32 * KT + 2 * NT>(vw, lut_lane), lut_pair<32 * KT + 2 * NT + 1>(vw, lut_lane));
#define TQ_PV_KT(KT)                                                                                          \
  TQ_PV(KT, 0) TQ_PV(KT, 1) TQ_PV(KT, 2) TQ_PV(KT, 3) TQ_PV(KT, 4) TQ_PV(KT, 5) TQ_PV(KT, 6) TQ_PV(KT, 7) \
  TQ_PV(KT, 8) TQ_PV(KT, 9) TQ_PV(KT, 10) TQ_PV(KT, 11) TQ_PV(KT, 12) TQ_PV(KT, 13) TQ_PV(KT, 14) TQ_PV(KT, 15)
        TQ_PV_KT(0) TQ_PV_KT(1)
#undef TQ_PV_KT
#undef TQ_PV
      }
    } else if (ok && win && gm.fp8) {
      // ---------------------------------------------------------- FP8 window / anchor tokens 4cw..4cw+3
      // The warp turns its 4 tokens' E4M3 codes into exact fp16 rows of its own
      // scratch (its other ldmatrix rows read the zero row); the per-token
      // scales multiply the scores and p in fp32.  q goes to fp16 for the mma.
      const uint16_t* qraw = reinterpret_cast<const uint16_t*>(sq + kTqQPrepBytes);
      const int j = (int)first;
      const int n_tok = j < n_wcw ? min(kTqWin, a.r - j * kTqWin) : kTqWin;
      const int t0 = 4 * cw;
      const unsigned char* kb8 = st;
      const unsigned char* vb8 = st + kTqWin * kFp8RowBytes;
      unsigned char* scr = smem + slot * C::STAGE + C::FP8_SCR + cw * 2048;   // K rows 0..3, then V rows 0..3
      {
        const int tt = lane >> 3, c0 = 16 * (lane & 7);
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
          const uint4 w = lds128((kv ? vb8 : kb8) + (t0 + tt) * kFp8RowBytes + c0);
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
          uint32_t hv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2(
                (__nv_fp8x2_storage_t)((wv[e >> 1] >> (16 * (e & 1))) & 0xFFFFu), __NV_E4M3);
            hv[e] = (uint32_t)h2.x | ((uint32_t)h2.y << 16);
          }
          uint4* outp = reinterpret_cast<uint4*>(scr + kv * 1024 + tt * C::WROW + c0 * 2);
          outp[0] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          outp[1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
        }
      }
      __syncwarp();
      const unsigned char* zero = smem + C::OFF_ZERO;
      float sw[4] = {0.f, 0.f, 0.f, 0.f};
      const int mi = lane >> 3, ri = lane & 7;
      const unsigned char* krowp = ri < 4 ? scr + ri * C::WROW : zero;
#pragma unroll
      for (int kt2 = 0; kt2 < NKT / 2; ++kt2) {
        uint32_t bk[4];
        ldsm_x4(bk, krowp + (16 * (2 * kt2 + (mi >> 1)) + 8 * (mi & 1)) * 2);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int kt = 2 * kt2 + h2;
          const uint32_t aq[4] = {
              head_ok ? in16x2_to_h2(*reinterpret_cast<const uint32_t*>(qraw + gr * D + 16 * kt + 2 * tc), gm.dtype)
                      : 0u,
              0u,
              head_ok ? in16x2_to_h2(*reinterpret_cast<const uint32_t*>(qraw + gr * D + 16 * kt + 8 + 2 * tc),
                                     gm.dtype)
                      : 0u,
              0u};
          mma_f16_16816(sw, aq, bk[2 * h2], bk[2 * h2 + 1]);
        }
      }
      float xv[2], vsc[2];
      float mt = -INFINITY;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = t0 + 2 * tc + e;
        const bool valid = head_ok && tc < 2 && t < n_tok;
        const int tr = min(t, kTqWin - 1);
        const float ks = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(kb8 + tr * kFp8RowBytes + D)));
        vsc[e] = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(vb8 + tr * kFp8RowBytes + D)));
        xv[e] = valid ? sw[e] * ks * a.scale_log2 : -INFINITY;
        mt = fmaxf(mt, xv[e]);
      }
      rescale_to(quad_max(mt));
      float pw[2], pt[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pw[e] = xv[e] == -INFINITY ? 0.f : fast_exp2(xv[e] - m);
        l += pw[e];
        pt[e] = xv[e] == -INFINITY ? 0.f : pw[e] * vsc[e];   // a masked token's scale may be stale bytes
      }
      const __half2 hi = __floats2half2_rn(pt[0], pt[1]);
      const float2 hb = __half22float2(hi);
      const __half2 lo = __floats2half2_rn(pt[0] - hb.x, pt[1] - hb.y);
      const uint32_t apw[4] = {h2_as_u32(hi), h2_as_u32(lo), 0u, 0u};
      const uint32_t vmask = (t0 + 2 * tc < n_tok ? 0x0000FFFFu : 0u) | (t0 + 2 * tc + 1 < n_tok ? 0xFFFF0000u : 0u);
      const unsigned char* vrowp = ri < 4 ? scr + 1024 + ri * C::WROW : zero;
#pragma unroll
      for (int n4 = 0; n4 < NNT / 4; ++n4) {
        uint32_t bv[4];
        ldsm_x4_t(bv, vrowp + 8 * (4 * n4 + mi) * 2);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) mma_f16_16816(o[4 * n4 + jj], apw, bv[jj] & vmask, 0u);
      }
      // the scratch's generic writes come before the copy that will reuse this
      // stage (async proxy), which the empty barrier alone does not order
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      __syncwarp();
    } else if (ok && win) {
      // ---------------------------------------------------------- window tokens 4cw..4cw+3 (exact 16-bit)
      const uint16_t* qraw = reinterpret_cast<const uint16_t*>(sq + kTqQPrepBytes);
      const int n_tok = min(kTqWin, a.r - (int)first * kTqWin);
      const int t0 = 4 * cw;
      const unsigned char* kb = st;
      const unsigned char* vb = st + kTqWin * C::WROW;
      const bool bf = gm.dtype == KVQ_BF16;
      float sw[4] = {0.f, 0.f, 0.f, 0.f};
      const int mi = lane >> 3, ri = lane & 7;
      const int krow = min(t0 + ri, kTqWin - 1);
#pragma unroll
      for (int kt2 = 0; kt2 < NKT / 2; ++kt2) {
        uint32_t bk[4];
        ldsm_x4(bk, kb + krow * C::WROW + (16 * (2 * kt2 + (mi >> 1)) + 8 * (mi & 1)) * 2);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int kt = 2 * kt2 + h2;
          const uint32_t aq[4] = {head_ok ? *reinterpret_cast<const uint32_t*>(qraw + gr * D + 16 * kt + 2 * tc) : 0u,
                                  0u,
                                  head_ok ? *reinterpret_cast<const uint32_t*>(qraw + gr * D + 16 * kt + 8 + 2 * tc)
                                          : 0u,
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
      const uint32_t vmask = (t0 + 2 * tc < n_tok ? 0x0000FFFFu : 0u) | (t0 + 2 * tc + 1 < n_tok ? 0xFFFF0000u : 0u);
      const int vrow = min(t0 + ri, kTqWin - 1);
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

  auto seg_end = [&](int row, int part) {
    if (tr && part == 0) {
      // token-major state: head tc, l summed over the 8 lanes gr
      float ls = l;
      ls += __shfl_xor_sync(0xffffffffu, ls, 4);
      ls += __shfl_xor_sync(0xffffffffu, ls, 8);
      ls += __shfl_xor_sync(0xffffffffu, ls, 16);
      if (gr == 0) {
        sm_m[cw * 8 + tc] = m;
        sm_l[cw * 8 + tc] = ls;
      }
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        sm_o[(cw * 8 + tc) * D + 16 * mt + gr] = o[mt][0] + o[mt][1];
        sm_o[(cw * 8 + tc) * D + 16 * mt + 8 + gr] = o[mt][2] + o[mt][3];
      }
    } else {
      const float ls = quad_sum(l);
      if (tc == 0) {
        sm_m[cw * 8 + gr] = m;
        sm_l[cw * 8 + gr] = ls;
      }
#pragma unroll
      for (int nt = 0; nt < NNT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) sm_o[(cw * 8 + gr) * D + 8 * nt + 2 * tc + e] = o[nt][e] + o[nt][2 + e];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_qempty[(qseg - 1) & 1]);
    tq_consumer_bar();
    const int g = gm.g;
    // 1. merge the warps: O[h][c] relative to the head's max M, into warp 0's slice
    for (int i = ct; i < g * D; i += kTqConsumers * 32) {
      const int h = i / D, c = i - h * D;
      float M = -INFINITY;
      for (int w = 0; w < kTqConsumers; ++w) M = fmaxf(M, sm_m[w * 8 + h]);
      float O = 0.f, L = 0.f;
      for (int w = 0; w < kTqConsumers; ++w) {
        const float f = M == -INFINITY ? 0.f : exp2f(sm_m[w * 8 + h] - M);
        O += sm_o[(w * 8 + h) * D + c] * f;
        L += sm_l[w * 8 + h] * f;
      }
      sm_o[h * D + c] = O;
      if (c == 0) {
        sm_hm[h] = M;
        sm_hm[8 + h] = L;
      }
    }
    tq_consumer_bar();
    // 2. token blocks: back to the original basis, y_c = sum_j Pi[j][c] O_j (into warp 1's slice)
    const float* fin = sm_o;
    if (part == 0) {
      if (!pi_ready) {
        const bool ok = mbar_wait(bar_pi, 0, abort_flag, wl);
        if (!ok && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
        if (!ok) *abort_flag = 1;
        pi_ready = true;
      }
      float* y = sm_o + 8 * D;
      for (int i = ct; i < g * D; i += kTqConsumers * 32) {
        const int h = i / D, c = i - h * D;
        const float* oh = sm_o + h * D;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
        for (int j = 0; j < D; j += 2) {
          acc0 = fmaf(sm_pi[j * D + c], oh[j], acc0);
          acc1 = fmaf(sm_pi[(j + 1) * D + c], oh[j + 1], acc1);
        }
        y[i] = acc0 + acc1;
      }
      tq_consumer_bar();
      fin = y;
    }
    const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
    const int it0 = row * Pt.n_items;
    const int np0 = Pt.n_tb > 0 ? Pt.cta_of(it0 + Pt.n_tb - 1) - Pt.cta_of(it0) + 1 : 0;
    const int c_f1 = Pt.n_wc > 0 ? Pt.cta_of(it0 + Pt.n_tb) : 0;
    const int np1 = Pt.n_wc > 0 ? Pt.cta_of(it0 + Pt.n_items - 1) - c_f1 + 1 : 0;
    const int c_f0 = Pt.n_tb > 0 ? Pt.cta_of(it0) : 0;
    const int expected = np0 + np1;
    float* out_row = a.out + ((int64_t)b * gm.Hq + (int64_t)hkv * g) * D;
    if (expected == 1) {
      for (int i = ct; i < g * D; i += kTqConsumers * 32) {
        const int h = i / D;
        if (!*abort_flag) out_row[i] = fin[i] / sm_hm[8 + h];
      }
    } else {
      // partial slot cta + 2 row + part
      float* pslot = a.ws + ((int64_t)(cta + 2 * row + part) * g) * (D + 2);
      for (int i = ct; i < g * (D + 2); i += kTqConsumers * 32) {
        const int h = i / (D + 2), c = i - h * (D + 2);
        pslot[i] = c < D ? fin[h * D + c] : sm_hm[(c - D) * 8 + h];
      }
      tq_consumer_bar();
      // An aborted CTA arrives as well (its partial is then unspecified), so
      // the last arriver always resets the counter for the next launch; an
      // aborted last arriver writes no output.
      if (ct == 0) {
        unsigned old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;\n" : "=r"(old) : "l"(a.counters + row) : "memory");
        *last_flag = old == (unsigned)(expected - 1);
      }
      tq_consumer_bar();
      if (*last_flag) {
        // last segment of the row: merge its partials (slots c_f0 + 2 row ... for
        // the token blocks, c_f1 + 2 row + 1 ... for the window)
        const int np = expected;
        float* pm = sm_o;                  // [np][g]
        float* pw = sm_o + np * g;         // [np][g]
        float* pl = sm_o + 2 * np * g;     // [np][g]
        float* hm = sm_o + 3 * np * g;     // [g] max, then [g] 1/L
        auto slot_of = [&](int j) -> int64_t {
          return j < np0 ? (int64_t)(c_f0 + 2 * row + j) : (int64_t)(c_f1 + 2 * row + 1 + (j - np0));
        };
        for (int i = ct; i < np * g; i += kTqConsumers * 32) {
          const int j = i / g, h = i - j * g;
          const float* ps = a.ws + (slot_of(j) * g + h) * (D + 2);
          pm[i] = __ldcg(ps + D);
          pl[i] = __ldcg(ps + D + 1);
        }
        tq_consumer_bar();
        for (int h = ct; h < g; h += kTqConsumers * 32) {
          float M = -INFINITY;
          for (int j = 0; j < np; ++j) M = fmaxf(M, pm[j * g + h]);
          float L = 0.f;
          for (int j = 0; j < np; ++j) L += pm[j * g + h] == -INFINITY ? 0.f : pl[j * g + h] * exp2f(pm[j * g + h] - M);
          hm[h] = M;
          hm[g + h] = 1.f / L;
        }
        tq_consumer_bar();
        for (int i = ct; i < np * g; i += kTqConsumers * 32) {
          const int h = i % g;
          pw[i] = pm[i] == -INFINITY ? 0.f : exp2f(pm[i] - hm[h]) * hm[g + h];
        }
        tq_consumer_bar();
        for (int e = ct; e < g * D && !*abort_flag; e += kTqConsumers * 32) {
          const int h = e / D, c = e - h * D;
          float acc = 0.f;
          for (int j = 0; j < np; ++j) acc = fmaf(__ldcg(a.ws + (slot_of(j) * g + h) * (D + 2) + c), pw[j * g + h], acc);
          out_row[e] = acc;
        }
        if (ct == 0) a.counters[row] = 0u;
      }
    }
    tq_consumer_bar();
  };

  tq_for_each_chunk(Pt, i0, i1, chunk, seg_begin, seg_end);
}

}  // namespace

void launch_tq_attention(const AttnArgs& a, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(tq_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TL::SMEM);
    attr_set = true;
  }
  tq_decode_kernel<<<a.n_cta, kTqThreads, TL::SMEM, st>>>(a);
  count_launch(1);
}

}  // namespace kvq

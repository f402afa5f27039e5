// KIVI decode attention straight from the packed cache.
//
// Every decode step reads the whole cache ("La compression du cache KV est une
// decision d'infrastructure...", section "... quand la HBM, pas les FLOPs, est
// votre plafond"), so the kernel is one streaming pass over the group records
// and window tokens.  The dequantization is fused into both contractions:
//   score_t = sum_c q_c (z_c + s_c code_tc) = beta + sum_c (q_c s_c) code_tc
//   o_c     = sum_t p_t (zv_t + sv_t code_tc) = sum_t p_t zv_t + sum_t (p_t sv_t) code_tc
// q~ = q (.) s (per group) and p~ = p (.) sv (per token) are split into fp16
// hi + lo parts, and both contractions run on mma.sync with the exact
// small-integer fp16 codes as the other operand.  Two formulations:
//   hybrid (GQA groups of 8 heads): scores head-major -- the heads' hi | lo
//     parts are the two 8-row halves of the m16 A operand and the key codes
//     are the B operand -- and P.V token-major -- the value codes are the A
//     operand and p~ of the 8 heads the B operand, its hi and lo parts
//     accumulated into one tile;
//   token-major (groups of 1..4 heads): the codes are the A operand of both
//     contractions (tokens, resp. channels, are M) and the heads' hi | lo
//     parts are the 8 columns of B, half the mma's of the hybrid form for
//     such groups.
//
// Structure (one CTA per SM, one launch per decode step):
//   warp 0      producer: 1-D bulk copies (cp.async.bulk, no multicast) of whole
//               group records / window rows into a ring of shared-memory stages
//   warp 1      prep: the zero-point term beta = q . z for every group of a stage
//               in batched mma's (columns = groups)
//   warp 2      merge: the warp states of every segment but the CTA's last
//   warps 3..   12 consumers: one 32-token block per warp per stage, online
//               softmax
// Work: the (row, item) sequence -- a row's groups then its 32-token window
// chunks -- is cut on the host into ranges of equal stage count, one per CTA
// (a window chunk's stage weighs 1.5 group stages).  A CTA writes one
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

constexpr int kWinTok = kDecodeWinTok;                     // tokens per window item

// Code operands as fp16 subnormals: (x & field) is the fp16 bit pattern of
// code * 2^(b j') * 2^-24 (exponent field zero), one LOP3 per pair instead of
// LOP3 + HSUB2.  The mma.sync products of such operands keep about 2^-17 of
// the sum of |products| (measured against exact sums; normal operands keep
// about 2^-21), well inside the attention tolerance.  The 2^24 goes back in
// fp32: into the score scale, and into the output at the end of a segment.
constexpr float kSubScale = 16777216.f;   // 2^24
template <int BITS, int JP>
__device__ __forceinline__ uint32_t code_pair(uint32_t x) {
  constexpr uint32_t M = (BITS == 2 ? 0x00030003u : 0x000F000Fu) << (BITS * JP);
  return x & M;
}
template <int BITS>
__device__ __forceinline__ void code_half(uint32_t x, uint32_t* out) {
  out[0] = code_pair<BITS, 0>(x);
  out[1] = code_pair<BITS, 1>(x);
  if (BITS == 2) {
    out[2] = code_pair<BITS, 2>(x);
    out[3] = code_pair<BITS, 3>(x);
  }
}

template <int NC>
__device__ __forceinline__ void consumer_bar() { named_bar_sync<NC * 32>(); }

// NC consumer warps; TR selects the token-major formulation (GQA groups of up
// to 4 heads, see the kernel comment), which runs 12 consumers.
template <int BITS, int D, int G, bool TR>
struct K {
  static constexpr int NC = TR ? kKiviConsumersTM : kKiviConsumersHM;   // consumer warps
  static constexpr int THREADS = (NC + 3) * 32;                  // + producer, prep, merge warps
  static constexpr int HS = TR ? 4 : 8;                          // heads per warp state
  static constexpr int DP = D + 4;                               // partial row (o[D], m, l, pad): 16-byte multiple
  static constexpr int NTB = G / kTB;
  static constexpr int SG = NC / NTB;                            // groups per stage
  static constexpr int REC = G * D * BITS / 4 + 4 * D + 4 * G;   // record bytes
  static constexpr int TBC = kTB * D * BITS / 8;                 // TB code bytes
  static constexpr int WROW = D * 2;                             // window row in shared memory
  static constexpr int WINB = kWinTok * WROW * 2;                 // window item bytes in a stage (K + V)
  static constexpr int STAGE = ((SG * REC > WINB ? SG * REC : WINB) + 127) / 128 * 128;
  // warp-state buffer (floats): m[NC][HS], l[NC][HS], a flag word and padding,
  // then o[NC][HS][D]
  static constexpr int SO = (2 * NC * HS + 1 + 3) / 4 * 4;
  static constexpr int SBUF_F = SO + NC * HS * D;
  // warp-state buffers: two let the merge warp merge one segment while the
  // consumers fill the next; the hybrid formulation's 8-head states are twice
  // as large, so it keeps one and spends the room on a deeper stage ring
  static constexpr int NSB = TR ? 2 : 1;
  static constexpr int FIXED = NSB * SBUF_F * 4 + (TR ? NC * 512 : 0) + 2 * 8 * D * 2 + 8 * 8 + 16;
  static constexpr int NST_FIT = (227 * 1024 - FIXED) / (STAGE + SG * 8 * 4 + 3 * 8);
  static constexpr int NST = (STAGE > 48 * 1024 ? 3 : 4) < NST_FIT ? (STAGE > 48 * 1024 ? 3 : 4) : NST_FIT;
  static constexpr int KSOFF = G * D * BITS / 4;
  static constexpr int KZOFF = KSOFF + 2 * D;
  static constexpr int VMOFF = KSOFF + 4 * D;
  // shared memory map (bytes)
  static constexpr int OFF_BETA = NST * STAGE;
  static constexpr int OFF_S = OFF_BETA + NST * SG * 8 * 4;      // two warp-state buffers
  static constexpr int OFF_PW = OFF_S + NSB * SBUF_F * 4;        // per-warp P tile (TR): 32 tokens x 8 fp16
  static constexpr int OFF_Q = OFF_PW + (TR ? NC * 512 : 0);     // q ring: 2 slots x raw 16-bit q of 8 heads
  static constexpr int OFF_BAR = OFF_Q + 2 * 8 * D * 2;
  static constexpr int OFF_FLAG = OFF_BAR + (3 * NST + 9) * 8;
  static constexpr int SMEM = OFF_FLAG + 16;
  static_assert(NST >= 2, "decode pipeline needs two stages");
  static_assert(SG <= 16, "a stage copies at most 16 records");
  static_assert(SMEM <= 227 * 1024, "decode kernel shared memory exceeds the per-block limit");
};

// ------------------------------------------------------------------ work partition
// Items of a row: groups 0..n_g-1, then window chunks of kWinTok tokens.  The
// host cuts the (row, item) sequence into stage-balanced CTA ranges (item0 in
// the launch arguments, read from the grid-constant parameter space).
struct Part {
  int n_g, n_items, n_cta;
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

// Iterates the chunks of one CTA: calls f(stage_index, row, is_window, first, count)
// for quantized chunks (count groups from group `first`) and window chunks
// (count = 1, first = chunk index); calls seg(row, begin) at each segment start
// and seg_end(row) at its end.
template <int SG, class FC, class FS, class FE>
__device__ __forceinline__ void for_each_chunk(const Part& P, int i0, int i1, FC f, FS seg, FE seg_end) {
  int s = 0;
  if (i0 >= i1) return;
  for (int row = P.row_of(i0); row * P.n_items < i1; ++row) {
    const int a = max(i0, row * P.n_items) - row * P.n_items;
    const int b = min(i1, (row + 1) * P.n_items) - row * P.n_items;
    if (a >= b) continue;
    seg(row);
    for (int k = a; k < min(b, P.n_g); k += SG) {
      const int cnt = min(SG, min(b, P.n_g) - k);
      f(s++, row, false, (int64_t)k, cnt);
    }
    for (int k = max(a, P.n_g); k < b; ++k) f(s++, row, true, (int64_t)(k - P.n_g), 1);
    seg_end(row);
  }
}

// ------------------------------------------------------------------ the kernel
// Both formulations run 15 warps.  Declaring 512 threads caps them at 128
// registers, so that the four warps one SM sub-partition holds fit its
// 16,384-entry register file.
template <int BITS, int D, int G, bool TR>
__global__ void __launch_bounds__(512, 1) kivi_decode_kernel(const __grid_constant__ AttnArgs a) {
  using C = K<BITS, D, G, TR>;
  constexpr int P = D * BITS / 32;
  constexpr int J = BITS == 2 ? 4 : 2;
  constexpr int NKT = D / 16;
  constexpr int WPN = P / 4;

  extern __shared__ __align__(128) unsigned char smem[];
  float* sm_beta = reinterpret_cast<float*>(smem + C::OFF_BETA);
  float* sm_state = reinterpret_cast<float*>(smem + C::OFF_S);   // [NSB][SBUF_F]
  uint16_t* sm_q = reinterpret_cast<uint16_t*>(smem + C::OFF_Q);
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_ready = bar_full + C::NST;
  uint64_t* bar_empty = bar_ready + C::NST;
  uint64_t* bar_qfull = bar_empty + C::NST;    // [2]
  uint64_t* bar_qempty = bar_qfull + 2;        // [2]
  uint64_t* bar_sfull = bar_qempty + 2;        // [2] warp states of a segment written
  uint64_t* bar_sfree = bar_sfull + 2;         // [2] merge warp done with a state buffer
  uint64_t* bar_merge = bar_sfree + 2;         // [1] partials of the final row merge copied in
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);

  const Geom& gm = a.geom;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, tc = lane & 3;
  const long long wl = a.wait_cycles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_ready[i], 1);
      mbar_init(&bar_empty[i], C::NC);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_qfull[i], 1);
      mbar_init(&bar_qempty[i], C::NC + 1);
      mbar_init(&bar_sfull[i], C::NC);
      mbar_init(&bar_sfree[i], 1);
    }
    mbar_init(bar_merge, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  }
  __syncthreads();

  Part Pt;
  Pt.n_g = (int)a.n_groups;
  Pt.n_items = a.n_items;
  Pt.n_cta = a.n_cta;
  Pt.item0 = a.item0;
  const int cta = blockIdx.x;
  const int i0 = a.item0[cta];
  const int i1 = a.item0[cta + 1];
  auto nop_seg = [](int) {};
  const int last_row = i1 > i0 ? Pt.row_of(i1 - 1) : -1;

  // Merges the warp states of one segment (state buffer sb) and writes the
  // row's output when this CTA covers the whole row, else the CTA's partial
  // (o[D], m, l) of the row; the last CTA to finish a row then merges the row's
  // partials with a log-sum-exp.  tid / nth: this thread's rank among the nth
  // threads running it together; sync(): their barrier.  A thread handles four
  // channels of one head at a time and derives that head's merge factors
  // itself, so only the publication of a partial needs barriers.
  // c_first, np: the first CTA of the row and the number of CTAs with a partial
  // of it.  The consumer warps (nth > 32) merge the CTA's last segment after
  // the loop, when the stage ring is idle: their row merge copies the partials
  // there with bulk copies instead of loading them (one round trip per chunk).
  auto merge_segment = [&](int row, float* sb, int tid, int nth, auto sync, int c_first, int np) {
    constexpr int NC = C::NC, HS = C::HS, DP = C::DP;
    const float* s_m = sb;
    const float* s_l = sb + NC * HS;
    volatile int* s_last = reinterpret_cast<volatile int*>(sb + 2 * NC * HS);
    const float* s_o = sb + C::SO;
    const int g = gm.g;
    const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
    float* out_row = a.out + ((int64_t)b * gm.Hq + (int64_t)hkv * g) * D;
    float* part = a.ws + ((int64_t)(cta + row) * g) * DP;
    // warp states -> this CTA's (o, M, L) of the row, four channels per step
    for (int e4 = tid; e4 < g * D / 4; e4 += nth) {
      const int h = e4 / (D / 4), c = 4 * (e4 - h * (D / 4));
      float M = -INFINITY;
      for (int w = 0; w < NC; ++w) M = fmaxf(M, s_m[w * HS + h]);
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
      float L = 0.f;
#pragma unroll 4
      for (int w = 0; w < NC; ++w) {
        const float f = M == -INFINITY ? 0.f : exp2f(s_m[w * HS + h] - M);
        const float4 v = *reinterpret_cast<const float4*>(s_o + (w * HS + h) * D + c);
        O.x = fmaf(v.x, f, O.x);
        O.y = fmaf(v.y, f, O.y);
        O.z = fmaf(v.z, f, O.z);
        O.w = fmaf(v.w, f, O.w);
        L = fmaf(s_l[w * HS + h], f, L);
      }
      if (np == 1) {
        if (!*abort_flag) {
          const float r = 1.f / L;
          *reinterpret_cast<float4*>(out_row + h * D + c) = make_float4(O.x * r, O.y * r, O.z * r, O.w * r);
        }
      } else {
        *reinterpret_cast<float4*>(part + h * DP + c) = O;
        if (c == 0) *reinterpret_cast<float4*>(part + h * DP + D) = make_float4(M, L, 0.f, 0.f);
      }
    }
    if (np == 1) return;
    // The barrier orders every thread's partial stores before thread 0's
    // gpu-scope acq_rel atomic (release is cumulative), so one fenced atomic
    // publishes the whole partial; the last arriver's acquire plus the next
    // barrier make every partial visible to all the merging threads.
    // An aborted CTA arrives as well (its partial is then unspecified), so the
    // last arriver always resets the counter for the next launch; an aborted
    // last arriver writes no output.
    sync();
    if (tid == 0) {
      unsigned old;
      asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;\n" : "=r"(old) : "l"(a.counters + row) : "memory");
      *s_last = old == (unsigned)(np - 1);
    }
    sync();
    if (!*s_last) return;
    const float* ws_row = a.ws + (int64_t)(c_first + row) * g * DP;
    if (nth > 32) {
      // Last CTA of the row, consumer warps: the np partials (consecutive
      // slots) are bulk-copied into the idle stage ring, KP at a time, and
      // merged from there with an online log-sum-exp.
      const int PB = g * DP * 4;
      const int KP = (C::NST * C::STAGE) / PB;
      const float* buf = reinterpret_cast<const float*>(smem);
      float M[2], L[2];
      float4 acc[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        M[i] = -INFINITY;
        L[i] = 0.f;
        acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      for (int j0 = 0, k = 0; j0 < np; j0 += KP, ++k) {
        const int nj = min(KP, np - j0);
        bool issued = false;
        if (tid == 0 && !*abort_flag) {
          // the partials are generic-proxy stores of this and other CTAs, seen
          // through the acquire above; order them before the async-proxy copy
          asm volatile("fence.proxy.async.global;\n" ::: "memory");
          mbar_expect_tx(bar_merge, (uint32_t)(nj * PB));
          bulk_g2s(smem, ws_row + (int64_t)j0 * g * DP, (uint32_t)(nj * PB), bar_merge);
          issued = true;
        }
        const bool ok = !*abort_flag && mbar_wait(bar_merge, k & 1, abort_flag, wl);
        if (!ok && !*abort_flag) {
          atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
          *abort_flag = 1;
        }
        if (issued && !ok) mbar_drain(bar_merge, k & 1);   // the copy lands before the CTA can exit
        if (ok) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int e4 = tid + i * nth;
            if (e4 < g * D / 4) {
              const int h = e4 / (D / 4), c = 4 * (e4 - h * (D / 4));
              float Mb = M[i];
              for (int u = 0; u < nj; ++u) Mb = fmaxf(Mb, buf[(u * g + h) * DP + D]);
              const float r = M[i] == -INFINITY ? 0.f : exp2f(M[i] - Mb);
              L[i] *= r;
              acc[i].x *= r;
              acc[i].y *= r;
              acc[i].z *= r;
              acc[i].w *= r;
              for (int u = 0; u < nj; ++u) {
                const float* pu = buf + (u * g + h) * DP;
                const float mu = pu[D];
                const float f = mu == -INFINITY ? 0.f : exp2f(mu - Mb);
                const float4 v = *reinterpret_cast<const float4*>(pu + c);
                L[i] = fmaf(pu[D + 1], f, L[i]);
                acc[i].x = fmaf(v.x, f, acc[i].x);
                acc[i].y = fmaf(v.y, f, acc[i].y);
                acc[i].z = fmaf(v.z, f, acc[i].z);
                acc[i].w = fmaf(v.w, f, acc[i].w);
              }
              M[i] = Mb;
            }
          }
        }
        sync();   // every thread is done with the chunk before the next copy
      }
      if (!*abort_flag) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int e4 = tid + i * nth;
          if (e4 < g * D / 4) {
            const int h = e4 / (D / 4), c = 4 * (e4 - h * (D / 4));
            const float r = 1.f / L[i];
            *reinterpret_cast<float4*>(out_row + h * D + c) =
                make_float4(acc[i].x * r, acc[i].y * r, acc[i].z * r, acc[i].w * r);
          }
        }
      }
      if (tid == 0) a.counters[row] = 0u;
      return;
    }
    // Last CTA of the row, merge warp: online log-sum-exp over the np partials,
    // the loads of up to kMB partials (o, m, l) in flight together.
    constexpr int kMB = 8;
    for (int e4 = tid; e4 < g * D / 4 && !*abort_flag; e4 += nth) {
      const int h = e4 / (D / 4), c = 4 * (e4 - h * (D / 4));
      const float* col = ws_row + (int64_t)h * DP;
      float M = -INFINITY, L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j0 = 0; j0 < np; j0 += kMB) {
        const int nj = min(kMB, np - j0);
        float4 v[kMB];
        float2 ml[kMB];
#pragma unroll
        for (int u = 0; u < kMB; ++u) {
          if (u < nj) {
            const float* pj = col + (int64_t)(j0 + u) * g * DP;
            v[u] = __ldcg(reinterpret_cast<const float4*>(pj + c));
            ml[u] = __ldcg(reinterpret_cast<const float2*>(pj + D));
          }
        }
        float Mb = M;
#pragma unroll
        for (int u = 0; u < kMB; ++u)
          if (u < nj) Mb = fmaxf(Mb, ml[u].x);
        const float r = M == -INFINITY ? 0.f : exp2f(M - Mb);
        L *= r;
        acc.x *= r;
        acc.y *= r;
        acc.z *= r;
        acc.w *= r;
#pragma unroll
        for (int u = 0; u < kMB; ++u) {
          if (u < nj) {
            const float f = ml[u].x == -INFINITY ? 0.f : exp2f(ml[u].x - Mb);
            L = fmaf(ml[u].y, f, L);
            acc.x = fmaf(v[u].x, f, acc.x);
            acc.y = fmaf(v[u].y, f, acc.y);
            acc.z = fmaf(v[u].z, f, acc.z);
            acc.w = fmaf(v[u].w, f, acc.w);
          }
        }
        M = Mb;
      }
      const float r = 1.f / L;
      *reinterpret_cast<float4*>(out_row + h * D + c) = make_float4(acc.x * r, acc.y * r, acc.z * r, acc.w * r);
    }
    if (tid == 0) a.counters[row] = 0u;
  };

  if (warp == 2) {
    // ------------------------------------------------------------ merge: every segment but the CTA's last
    int k = 0;
    for_each_chunk<C::SG>(
        Pt, i0, i1, [](int, int, bool, int64_t, int) {}, nop_seg,
        [&](int row) {
          const int sbi = k % C::NSB;
          const uint32_t par = (k / C::NSB) & 1;
          ++k;
          if (row == last_row) return;   // the consumer warps merge the CTA's last segment
          const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_sfull[sbi], par, abort_flag, wl));
          if (!ok) {
            if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
          } else {
            const int first_it = row * Pt.n_items;
            const int c_first = Pt.cta_of(first_it);
            merge_segment(row, sm_state + sbi * C::SBUF_F, lane, 32, [] { __syncwarp(); }, c_first,
                          Pt.cta_of(first_it + Pt.n_items - 1) - c_first + 1);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_sfree[sbi]);
        });
    return;
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0, qseg = 0, qissued = 0, withheld = -1;
      for_each_chunk<C::SG>(
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
              const uint32_t bytes = (uint32_t)cnt * C::REC;
              mbar_expect_tx(&bar_full[slot], bytes);
              bulk_g2s(dst, record_ptr(gm, row, first), bytes, &bar_full[slot]);
            } else if (!win) {
              if (!pages_valid(gm, pages)) {
                atomicOr(gm.status, KVQ_DEV_BAD_PAGE);
                *abort_flag = 1;
                return;
              }
              copy_records(gm, row, first, cnt, C::REC, pages, dst, &bar_full[slot]);
            } else {
              const int t0 = (int)first * kWinTok;
              const int n = min(kWinTok, a.r - t0);
              const int slot0 = (a.head + t0) % gm.cap;
              // two copies (key rows, value rows): a CTA's bulk copies complete
              // roughly one after another, so few large copies beat many small ones;
              // with a fused append the chunk's last token comes from k_new / v_new
              const bool fused = a.k_new != nullptr && t0 + n == a.r;
              const int n_ring = fused ? n - 1 : n;
              mbar_expect_tx(&bar_full[slot], 2u * (uint32_t)n * D * 2);
              if (n_ring > 0) {
                const uint32_t bytes = (uint32_t)n_ring * D * 2;
                bulk_g2s(dst, ring_ptr(gm, row, 0) + (int64_t)slot0 * D, bytes, &bar_full[slot]);
                bulk_g2s(dst + kWinTok * C::WROW, ring_ptr(gm, row, 1) + (int64_t)slot0 * D, bytes, &bar_full[slot]);
              }
              if (fused) {
                bulk_g2s(dst + n_ring * C::WROW, a.k_new + (int64_t)row * D, D * 2, &bar_full[slot]);
                bulk_g2s(dst + (kWinTok + n_ring) * C::WROW, a.v_new + (int64_t)row * D, D * 2, &bar_full[slot]);
              }
            }
            issued = s + 1;
          },
          [&](int row) {
            // q of the segment's row into ring slot k & 1
            if (*abort_flag) return;
            const int k = qseg++;
            const int qs = k & 1;
            if (k >= 2 && !mbar_wait(&bar_qempty[qs], ((k >> 1) - 1) & 1, abort_flag, wl)) {
              atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
              *abort_flag = 1;
              return;
            }
            if (*abort_flag) return;
            const int b = row / gm.Hkv, hkv = row - b * gm.Hkv;
            const uint32_t bytes = (uint32_t)gm.g * D * 2;
            mbar_expect_tx(&bar_qfull[qs], bytes);
            bulk_g2s(sm_q + qs * 8 * D, a.q + ((int64_t)b * gm.Hq + (int64_t)hkv * gm.g) * D, bytes, &bar_qfull[qs]);
            qissued = k + 1;
          },
          nop_seg);
      // Every copy issued lands before this warp exits (only the last NST
      // stages and the last two q slots can still be in flight), so none can
      // write shared memory after the CTA is gone, even when its consumers
      // gave up waiting.
      for (int s = max(0, issued - C::NST); s < issued; ++s)
        if (s != withheld) mbar_drain(&bar_full[s % C::NST], (s / C::NST) & 1);
      for (int k = max(0, qissued - 2); k < qissued; ++k) mbar_drain(&bar_qfull[k & 1], (k >> 1) & 1);
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
          const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_full[slot], (s / C::NST) & 1, abort_flag, wl));
          if (!ok) {
            if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
          }
          if (ok && !win) {
            // columns of B = the stage's groups; rows of A = heads (q, exact in fp16)
            const unsigned char* st = smem + slot * C::STAGE;
            float* bt = sm_beta + (slot * C::SG) * 8;
            for (int g0 = 0; g0 < cnt; g0 += 8) {   // columns: groups g0 .. g0 + 7
              float bacc[4] = {0.f, 0.f, 0.f, 0.f};
              const int grp = g0 + gr < cnt ? g0 + gr : g0;
              const unsigned char* pz = st + grp * C::REC + C::KZOFF + 16 * tc;
#pragma unroll
              for (int i = 0; i < D / 32; ++i) {
                const uint4 z4 = lds128(pz + 64 * i);
                const uint32_t a0[4] = {qh[2 * i][0], 0u, qh[2 * i][1], 0u};
                const uint32_t a1[4] = {qh[2 * i + 1][0], 0u, qh[2 * i + 1][1], 0u};
                mma_f16_16816(bacc, a0, z4.x, z4.y);
                mma_f16_16816(bacc, a1, z4.z, z4.w);
              }
              // thread holds beta(head gr, groups g0 + 2tc, g0 + 2tc + 1)
              if (g0 + 2 * tc < cnt) bt[(g0 + 2 * tc) * 8 + gr] = bacc[0];
              if (g0 + 2 * tc + 1 < cnt) bt[(g0 + 2 * tc + 1) * 8 + gr] = bacc[1];
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_ready[slot]);
        },
        [&](int row) {
          (void)row;
          const int k = qseg++;
          const int qs = k & 1;
          const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_qfull[qs], (k >> 1) & 1, abort_flag, wl));
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
  const int cw = warp - 3;
  // Head whose q this lane feeds to the score contraction: gr in the
  // hybrid formulation; gr >> 1 in the token-major one, where column gr of
  // the q~ operand is the hi (even gr) or lo (odd gr) part of head gr >> 1.
  const int qhead = TR ? gr >> 1 : gr;
  const bool head_ok = qhead < gm.g;
  int qseg = 0;
  const uint16_t* sq = sm_q;   // ring slot of the current segment
  uint32_t qh[NKT][2];   // q of head qhead at channels 16kt + 8rho + 2tc + {0, 1}, fp16x2
  // Output accumulators, m16n8 tiles with rows = 16 channels.  Hybrid:
  // columns = the 8 heads (hi and lo parts of p~ accumulate into the same
  // tile).  Token-major: columns = heads x {hi, lo}; this lane then holds
  // head tc only.
  constexpr int NO = D / 16;
  float o[NO][4];
  float m = -INFINITY, l = 0.f, wz = 0.f;
  int seg_row = 0;
  // The code contractions accumulate 2^-24 of their value (subnormal code
  // operands); o_sub: o is still on that scale (the segment's window chunks,
  // which come after its quantized blocks, bring it to 1 first).
  const float sl_code = a.scale_log2 * kSubScale;
  bool o_sub = true;
  auto o_to_unit = [&]() {
    if (o_sub) {
#pragma unroll
      for (int i = 0; i < NO; ++i) {
        o[i][0] *= kSubScale;
        o[i][1] *= kSubScale;
        o[i][2] *= kSubScale;
        o[i][3] *= kSubScale;
      }
      o_sub = false;
    }
  };

  auto seg_begin = [&](int row) {
    seg_row = row;
    const int k = qseg++;
    const int qs = k & 1;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_qfull[qs], (k >> 1) & 1, abort_flag, wl));
    if (!ok) {
      if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
    sq = sm_q + qs * 8 * D;
    const uint16_t* qrow = sq + qhead * D;
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
    for (int i = 0; i < NO; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    o_sub = true;
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
      for (int i = 0; i < NO; ++i) {
        o[i][0] *= alpha;
        o[i][1] *= alpha;
        o[i][2] *= alpha;
        o[i][3] *= alpha;
      }
      m = mn;
    }
  };

  // ---------------------------------------------------------------- token-major formulation
  // Tokens are the M dimension of both contractions, so the K and V codes are
  // the A operand (one A fragment = the B fragments of two adjacent 8-token
  // or 8-channel tiles of the packed format) and the N = 8 columns are the
  // heads' hi and lo parts: column 2h + {0, 1} = head h, hi | lo.  A GQA group
  // of up to 4 heads then fills the tile, with half the mma's of the
  // head-major formulation and half its accumulators.  Lane (gr, tc) holds
  // the scores of head tc for tokens gr + 8i and the output of head tc.
  uint32_t* sm_pw = reinterpret_cast<uint32_t*>(smem + C::OFF_PW) + cw * 128;   // [32 tokens][4 words]
  auto tr_head_max = [&](float x) {
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
    return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
  };
  auto tr_block = [&](const unsigned char* st, int slot) {
    const int grp = cw / C::NTB, tbg = cw - grp * C::NTB;
    const unsigned char* rec = st + grp * C::REC;
    uint4 kc[P / 4];
#pragma unroll
    for (int p = 0; p < P / 4; ++p) kc[p] = lds128(rec + tbg * C::TBC + 16 * (32 * p + lane));
    const float bs = sm_beta[(slot * C::SG + grp) * 8 + tc] * a.scale_log2;
    const unsigned char* psc = rec + C::KSOFF + 16 * tc;
    // fp16x2 (-1, -1) on lo lanes, (0, 0) on hi lanes: q~ column = fma(q, s, sel * round(q s))
    const uint32_t sel = (gr & 1) ? 0xBC00BC00u : 0u;
    float sc[2][2][4];   // [k-tile parity][token m-tile]: two independent chains per m-tile
#pragma unroll
    for (int par = 0; par < 2; ++par)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) sc[par][mt][0] = sc[par][mt][1] = sc[par][mt][2] = sc[par][mt][3] = 0.f;
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
          code_half<BITS>(half ? word >> 8 : word, pr[nt]);
        }
#pragma unroll
        for (int m2 = 0; m2 < J / 2; ++m2) {
          const int kt = (J / 2) * (2 * wi + half) + m2;
          const uint2 s2 = *reinterpret_cast<const uint2*>(psc + 64 * (kt >> 1) + 8 * (kt & 1));
          const __half2 h0 = __hmul2(u32_as_h2(qh[kt][0]), u32_as_h2(s2.x));
          const __half2 h1 = __hmul2(u32_as_h2(qh[kt][1]), u32_as_h2(s2.y));
          const uint32_t b0 = h2_as_u32(__hfma2(u32_as_h2(qh[kt][0]), u32_as_h2(s2.x), __hmul2(h0, u32_as_h2(sel))));
          const uint32_t b1 = h2_as_u32(__hfma2(u32_as_h2(qh[kt][1]), u32_as_h2(s2.y), __hmul2(h1, u32_as_h2(sel))));
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const uint32_t ak[4] = {pr[2 * mt][2 * m2], pr[2 * mt + 1][2 * m2], pr[2 * mt][2 * m2 + 1],
                                    pr[2 * mt + 1][2 * m2 + 1]};
            mma_f16_16816(sc[kt & 1][mt], ak, b0, b1);
          }
        }
      }
    // scores of head tc, tokens gr + 8i (i = 2 mt + e2)
    float x[4];
    float mx = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        const int i = 2 * mt + e2;
        x[i] = fmaf((sc[0][mt][2 * e2] + sc[1][mt][2 * e2]) + (sc[0][mt][2 * e2 + 1] + sc[1][mt][2 * e2 + 1]),
                    sl_code, bs);
        mx = fmaxf(mx, x[i]);
      }
    rescale_to(tr_head_max(mx));
    // value meta of token gr + 8i sits at entry 8 (gr >> 1) + 2i + (gr & 1) of the TB
    const unsigned char* pvm = rec + C::VMOFF + 4 * (tbg * kTB + 8 * (gr >> 1) + (gr & 1));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = fast_exp2(x[i] - m);
      const float2 sz = __half22float2(u32_as_h2(*reinterpret_cast<const uint32_t*>(pvm + 8 * i)));
      l += p;
      wz = fmaf(p, sz.y, wz);
      // value pair position j' of token gr + 8i: i (2-bit), i & 1 (4-bit)
      const float ps = p * (sz.x * pos_comp_f(BITS, BITS == 2 ? i : (i & 1)));
      const __half hi = __float2half_rn(ps);
      const __half lo = __float2half_rn(ps - __half2float(hi));
      sm_pw[(gr + 8 * i) * 4 + tc] = h2_as_u32(__halves2half2(hi, lo));
    }
    __syncwarp();
    uint32_t bp[4];   // k-tile kt: b0 = bp[2kt], b1 = bp[2kt + 1]
    ldsm_x4_t(bp, sm_pw + 4 * lane);
    uint4 vc[P / 4];
#pragma unroll
    for (int p = 0; p < P / 4; ++p) vc[p] = lds128(rec + (C::NTB + tbg) * C::TBC + 16 * (32 * p + lane));
    auto vword = [&](int w) {
      const uint4 pc = vc[w >> 2];
      return (w & 3) == 0 ? pc.x : (w & 3) == 1 ? pc.y : (w & 3) == 2 ? pc.z : pc.w;
    };
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t av[4];
        if (BITS == 2) {
          // channels 16mt + gr (low byte of each half word) and 16mt + 8 + gr (high byte)
          const uint32_t w = vword(mt);
          av[0] = kt ? code_pair<2, 2>(w) : code_pair<2, 0>(w);
          av[1] = kt ? code_pair<2, 2>(w >> 8) : code_pair<2, 0>(w >> 8);
          av[2] = kt ? code_pair<2, 3>(w) : code_pair<2, 1>(w);
          av[3] = kt ? code_pair<2, 3>(w >> 8) : code_pair<2, 1>(w >> 8);
        } else {
          // words 2mt (channel 16mt + gr) and 2mt + 1 (16mt + 8 + gr); half word = kt
          const uint32_t w0 = kt ? vword(2 * mt) >> 8 : vword(2 * mt);
          const uint32_t w1 = kt ? vword(2 * mt + 1) >> 8 : vword(2 * mt + 1);
          av[0] = code_pair<4, 0>(w0);
          av[1] = code_pair<4, 0>(w1);
          av[2] = code_pair<4, 1>(w0);
          av[3] = code_pair<4, 1>(w1);
        }
        mma_f16_16816(o[mt], av, bp[2 * kt], bp[2 * kt + 1]);
      }
    __syncwarp();   // the P tile is rewritten by this warp's next block
  };
  // Window chunk: warps 0 and 1 take tokens 16cw .. 16cw + 15 (exact 16-bit
  // operands; p split hi + lo in the input's format).
  auto tr_window = [&](const unsigned char* st, int64_t first) {
    const int n_tok = min(kWinTok, a.r - (int)first * kWinTok);
    const int t0 = 16 * cw;
    if (cw >= kWinTok / 16 || t0 >= n_tok) return;
    o_to_unit();
    const unsigned char* kb = st;
    const unsigned char* vb = st + kWinTok * C::WROW;
    const bool bf = gm.dtype == KVQ_BF16;
    const int mi = lane >> 3, ri = lane & 7;   // ldmatrix: matrix and row this lane addresses
    // scores: A = key rows t0 .. t0 + 15 (matrix mi: rows + 8 (mi & 1), channels + 8 (mi >> 1));
    // B = q, column gr = head gr >> 1 on even gr, zero on odd gr
    const int krow = min(t0 + 8 * (mi & 1) + ri, kWinTok - 1);
    const bool qcol = !(gr & 1) && (gr >> 1) < gm.g;
    const uint16_t* qr = sq + (gr >> 1) * D;
    float sw[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kt = 0; kt < NKT; ++kt) {
      uint32_t ak[4];
      ldsm_x4(ak, kb + krow * C::WROW + (16 * kt + 8 * (mi >> 1)) * 2);
      const uint32_t b0 = qcol ? *reinterpret_cast<const uint32_t*>(qr + 16 * kt + 2 * tc) : 0u;
      const uint32_t b1 = qcol ? *reinterpret_cast<const uint32_t*>(qr + 16 * kt + 8 + 2 * tc) : 0u;
      if (bf) mma_bf16_16816(sw[kt & 1], ak, b0, b1);
      else mma_f16_16816(sw[kt & 1], ak, b0, b1);
    }
    float xv[2];
    float mx = -INFINITY;
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const bool valid = t0 + gr + 8 * e2 < n_tok;
      xv[e2] = valid ? (sw[0][2 * e2] + sw[1][2 * e2]) * a.scale_log2 : -INFINITY;
      mx = fmaxf(mx, xv[e2]);
    }
    rescale_to(tr_head_max(mx));
    float pw[2];
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      pw[e2] = xv[e2] == -INFINITY ? 0.f : fast_exp2(xv[e2] - m);
      l += pw[e2];
    }
    // P tile rows = tokens gr, gr + 8; word tc = (hi, lo) of head tc
    const uint32_t ph = pack2_in16(pw[0], pw[1], gm.dtype);
    const float2 pb = unpack2_in16(ph, gm.dtype);
    const uint32_t pl = pack2_in16(pw[0] - pb.x, pw[1] - pb.y, gm.dtype);
    sm_pw[gr * 4 + tc] = (ph & 0xFFFFu) | (pl << 16);
    sm_pw[(gr + 8) * 4 + tc] = (ph >> 16) | (pl & 0xFFFF0000u);
    __syncwarp();
    uint32_t bp[2];
    ldsm_x2_t(bp, sm_pw + 4 * (lane & 15));
    // P.V: A = value rows transposed (matrix mi: tokens + 8 (mi >> 1), channels + 8 (mi & 1));
    // rows past n_tok are zeroed so stale shared memory never meets the zero weights
    const int vrow = min(t0 + 8 * (mi >> 1) + ri, kWinTok - 1);
    const uint32_t m01 = (t0 + 2 * tc < n_tok ? 0x0000FFFFu : 0u) | (t0 + 2 * tc + 1 < n_tok ? 0xFFFF0000u : 0u);
    const uint32_t m23 =
        (t0 + 8 + 2 * tc < n_tok ? 0x0000FFFFu : 0u) | (t0 + 8 + 2 * tc + 1 < n_tok ? 0xFFFF0000u : 0u);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t av[4];
      ldsm_x4_t(av, vb + vrow * C::WROW + (16 * mt + 8 * (mi & 1)) * 2);
      av[0] &= m01;
      av[1] &= m01;
      av[2] &= m23;
      av[3] &= m23;
      if (bf) mma_bf16_16816(o[mt], av, bp[0], bp[1]);
      else mma_f16_16816(o[mt], av, bp[0], bp[1]);
    }
    __syncwarp();
  };

  // ---------------------------------------------------------------- hybrid formulation (GQA groups of 8)
  // Scores head-major: A = q~ of the 8 heads, hi parts in rows 0-7 and lo
  // parts in rows 8-15; B = key codes (k16 channels x n8 tokens of the packed
  // format).  Lane (gr, tc) then holds the scores of head gr for tokens
  // 8 nt + 2 tc + {0, 1} -- which is exactly the B fragment of a token-major
  // P.V (k16 tokens x n8 heads), so p~ never leaves registers.  P.V: A = value
  // codes (m16 channels x k16 tokens: the B fragments of two adjacent 8-channel
  // tiles of the packed format), B = p~ of the 8 heads, split hi + lo, both
  // accumulated into one C tile [16 channels x 8 heads].  The output
  // accumulators are then 32 registers (64 in a purely head-major P.V, whose
  // lo rows are dead accumulator space), which leaves room for 12 consumer
  // warps.  Lane (gr, tc) holds the softmax state of head gr and the output of
  // heads 2 tc, 2 tc + 1.
  auto hx_rescale = [&](float mt) {
    // warp-uniform branch: lanes whose max did not grow scale by 1
    if (__any_sync(0xffffffffu, mt > m)) {
      const float mn = fmaxf(m, mt);
      const float alpha = m == -INFINITY ? 0.f : fast_exp2(m - mn);
      l *= alpha;
      wz *= alpha;
      m = mn;
      // the output columns are heads 2 tc and 2 tc + 1: their factors come
      // from quad 2 tc and quad 2 tc + 1
      const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * tc);
      const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * tc + 4);
#pragma unroll
      for (int i = 0; i < NO; ++i) {
        o[i][0] *= a0;
        o[i][1] *= a1;
        o[i][2] *= a0;
        o[i][3] *= a1;
      }
    }
  };
  // scores of one block (log2 domain, zero-point term included) -> x
  auto hx_qk = [&](const unsigned char* rec, int tbg, int slot, int grp, float (&x)[4][2]) {
    uint4 kc[P / 4];
#pragma unroll
    for (int p = 0; p < P / 4; ++p) kc[p] = lds128(rec + tbg * C::TBC + 16 * (32 * p + lane));
    const float bs = sm_beta[(slot * C::SG + grp) * 8 + gr] * a.scale_log2;
    // this lane's key scales: 16 bytes per k-tile pair kt2 at 64 kt2 + 16 tc
    const unsigned char* psc = rec + C::KSOFF + 16 * tc;
    float sc[4][4];   // [n-tile]
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
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
          code_half<BITS>(half ? word >> 8 : word, pr[nt]);
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
          for (int nt = 0; nt < 4; ++nt) mma_f16_16816(sc[nt], aq, pr[nt][2 * m2], pr[nt][2 * m2 + 1]);
        }
      }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) x[nt][e] = fmaf(sc[nt][e] + sc[nt][2 + e], sl_code, bs);
  };
  // online softmax and P.V of a block whose scores are x (record rec, token block tbg)
  auto hx_finish = [&](const unsigned char* rec, int tbg, const float (&x)[4][2]) {
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) mx = fmaxf(mx, fmaxf(x[nt][0], x[nt][1]));
    hx_rescale(quad_max(mx));
    uint32_t vm[8];
    {
      const uint4* pv = reinterpret_cast<const uint4*>(rec + C::VMOFF + 4 * (tbg * kTB + 8 * tc));
      const uint4 v0 = lds128(pv), v1 = lds128(pv + 1);
      vm[0] = v0.x; vm[1] = v0.y; vm[2] = v0.z; vm[3] = v0.w;
      vm[4] = v1.x; vm[5] = v1.y; vm[6] = v1.z; vm[7] = v1.w;
    }
    // B fragments of P.V: k-tile kt, b0 = tokens 16 kt + 2 tc + {0, 1} (n-tile
    // 2 kt), b1 = tokens 16 kt + 8 + 2 tc + {0, 1} (n-tile 2 kt + 1); column gr
    uint32_t bh[2][2], bl[2][2];
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int nt = 2 * kt + rr;
        float pt[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float p = fast_exp2(x[nt][e] - m);
          const float2 sz = __half22float2(u32_as_h2(vm[2 * nt + e]));
          l += p;
          wz = fmaf(p, sz.y, wz);
          // value pair position j' of token 8 nt + 2 tc + e: nt (2-bit), nt & 1 (4-bit)
          pt[e] = p * (sz.x * pos_comp_f(BITS, BITS == 2 ? nt : (nt & 1)));
        }
        const __half2 hi = __floats2half2_rn(pt[0], pt[1]);
        const float2 hb = __half22float2(hi);
        bh[kt][rr] = h2_as_u32(hi);
        bl[kt][rr] = h2_as_u32(__floats2half2_rn(pt[0] - hb.x, pt[1] - hb.y));
      }
    uint4 vc[P / 4];
#pragma unroll
    for (int p = 0; p < P / 4; ++p) vc[p] = lds128(rec + (C::NTB + tbg) * C::TBC + 16 * (32 * p + lane));
    auto vword = [&](int w) {
      const uint4 pc = vc[w >> 2];
      return (w & 3) == 0 ? pc.x : (w & 3) == 1 ? pc.y : (w & 3) == 2 ? pc.z : pc.w;
    };
    // k-tile-major: every m-tile's kt = 0 mma's before any kt = 1 mma, so the
    // mma's into one accumulator are far apart (legacy mma.sync has a long latency)
#pragma unroll
    for (int kt = 0; kt < 2; ++kt)
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t av[4];
        if (BITS == 2) {
          // channels 16mt + gr (low byte of each half word) and 16mt + 8 + gr (high byte)
          const uint32_t w = vword(mt);
          av[0] = kt ? code_pair<2, 2>(w) : code_pair<2, 0>(w);
          av[1] = kt ? code_pair<2, 2>(w >> 8) : code_pair<2, 0>(w >> 8);
          av[2] = kt ? code_pair<2, 3>(w) : code_pair<2, 1>(w);
          av[3] = kt ? code_pair<2, 3>(w >> 8) : code_pair<2, 1>(w >> 8);
        } else {
          // words 2mt (channel 16mt + gr) and 2mt + 1 (16mt + 8 + gr); half word = kt
          const uint32_t w0 = kt ? vword(2 * mt) >> 8 : vword(2 * mt);
          const uint32_t w1 = kt ? vword(2 * mt + 1) >> 8 : vword(2 * mt + 1);
          av[0] = code_pair<4, 0>(w0);
          av[1] = code_pair<4, 0>(w1);
          av[2] = code_pair<4, 1>(w0);
          av[3] = code_pair<4, 1>(w1);
        }
        mma_f16_16816(o[mt], av, bh[kt][0], bh[kt][1]);
        mma_f16_16816(o[mt], av, bl[kt][0], bl[kt][1]);
      }
  };
  // Window chunk: warps 0 and 1 take tokens 16 cw .. 16 cw + 15 (exact 16-bit
  // operands).  Scores head-major (A = q rows of the 8 heads, rows 8-15 zero;
  // B = key rows by ldmatrix), P.V token-major (A = value rows transposed by
  // ldmatrix; B = p split hi + lo in the input's format).
  auto hx_window = [&](const unsigned char* st, int64_t first) {
    const int n_tok = min(kWinTok, a.r - (int)first * kWinTok);
    const int t0 = 16 * cw;
    if (cw >= kWinTok / 16 || t0 >= n_tok) return;
    o_to_unit();
    const unsigned char* kb = st;
    const unsigned char* vb = st + kWinTok * C::WROW;
    const bool bf = gm.dtype == KVQ_BF16;
    const int mi = lane >> 3, ri = lane & 7;   // ldmatrix: matrix and row this lane addresses
    const uint16_t* qr = sq + gr * D;
    float sw[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int krow = min(t0 + 8 * nt + ri, kWinTok - 1);
#pragma unroll
      for (int kt2 = 0; kt2 < NKT / 2; ++kt2) {
        uint32_t bk[4];
        ldsm_x4(bk, kb + krow * C::WROW + (16 * (2 * kt2 + (mi >> 1)) + 8 * (mi & 1)) * 2);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int kt = 2 * kt2 + h2;
          const uint32_t aq[4] = {*reinterpret_cast<const uint32_t*>(qr + 16 * kt + 2 * tc), 0u,
                                  *reinterpret_cast<const uint32_t*>(qr + 16 * kt + 8 + 2 * tc), 0u};
          if (bf) mma_bf16_16816(sw[nt], aq, bk[2 * h2], bk[2 * h2 + 1]);
          else mma_f16_16816(sw[nt], aq, bk[2 * h2], bk[2 * h2 + 1]);
        }
      }
    }
    float xv[2][2];
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool valid = t0 + 8 * nt + 2 * tc + e < n_tok;
        xv[nt][e] = valid ? sw[nt][e] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, xv[nt][e]);
      }
    hx_rescale(quad_max(mx));
    uint32_t ph[2], pl[2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float pw[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pw[e] = xv[nt][e] == -INFINITY ? 0.f : fast_exp2(xv[nt][e] - m);
        l += pw[e];
      }
      ph[nt] = pack2_in16(pw[0], pw[1], gm.dtype);
      const float2 pb = unpack2_in16(ph[nt], gm.dtype);
      pl[nt] = pack2_in16(pw[0] - pb.x, pw[1] - pb.y, gm.dtype);
    }
    // rows past n_tok are zeroed so stale shared memory never meets the zero weights
    const int vrow = min(t0 + 8 * (mi >> 1) + ri, kWinTok - 1);
    const uint32_t m01 = (t0 + 2 * tc < n_tok ? 0x0000FFFFu : 0u) | (t0 + 2 * tc + 1 < n_tok ? 0xFFFF0000u : 0u);
    const uint32_t m23 =
        (t0 + 8 + 2 * tc < n_tok ? 0x0000FFFFu : 0u) | (t0 + 8 + 2 * tc + 1 < n_tok ? 0xFFFF0000u : 0u);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t av[4];
      ldsm_x4_t(av, vb + vrow * C::WROW + (16 * mt + 8 * (mi & 1)) * 2);
      av[0] &= m01;
      av[1] &= m01;
      av[2] &= m23;
      av[3] &= m23;
      if (bf) {
        mma_bf16_16816(o[mt], av, ph[0], ph[1]);
        mma_bf16_16816(o[mt], av, pl[0], pl[1]);
      } else {
        mma_f16_16816(o[mt], av, ph[0], ph[1]);
        mma_f16_16816(o[mt], av, pl[0], pl[1]);
      }
    }
  };

  auto chunk = [&](int s, int row, bool win, int64_t first, int cnt) {
    const int slot = s % C::NST;
    const uint32_t par = (s / C::NST) & 1;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_full[slot], par, abort_flag, wl) &&
                                                mbar_wait(&bar_ready[slot], par, abort_flag, wl));
    if (!ok) {
      if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
    if (TR && s == 0 && cw >= 4) {
      // Token-major formulation: the consumer warps of one SM sub-partition
      // (cw, cw + 4, cw + 8) start a fraction of a block apart, so that one's
      // softmax overlaps another's mma's instead of all of them alternating in
      // step.  (In the hybrid formulation the warps drift into the same phase
      // whatever the start offsets; measured on 70b, no offset was fastest.)
      const long long t0 = clock64();
      const long long d = (cw >> 2) * 800;
      while (clock64() - t0 < d) {
      }
    }
    const unsigned char* st = smem + slot * C::STAGE;
    if (ok && win && a.k_new != nullptr && cw == C::NC - 1) {
      // fused append: the new token of this row (the chunk's last) into its ring slot
      const int t0 = (int)first * kWinTok;
      const int n = min(kWinTok, a.r - t0);
      if (t0 + n == a.r) {
        const int slot_new = (a.head + a.r - 1) % gm.cap;
        constexpr int CH = D * 2 / 16;   // 16-byte chunks per row
        if (lane < 2 * CH) {
          const int part = lane / CH, ci = lane - part * CH;
          const uint4 v = lds128(st + (part * kWinTok + n - 1) * C::WROW + 16 * ci);
          reinterpret_cast<uint4*>(ring_ptr(gm, row, part) + (int64_t)slot_new * D)[ci] = v;
        }
      }
    }
    if constexpr (TR) {
      if (ok && !win && cw < cnt * C::NTB) tr_block(st, slot);
      else if (ok && win) tr_window(st, first);
    } else if (ok && !win && cw < cnt * C::NTB) {
      const int grp = cw / C::NTB, tbg = cw - grp * C::NTB;
      const unsigned char* rec = st + grp * C::REC;
      float x[4][2];
      hx_qk(rec, tbg, slot, grp, x);
      hx_finish(rec, tbg, x);
    } else if (ok && win) {
      hx_window(st, first);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_empty[slot]);
  };

  int final_row = -1;
  float* final_sb = nullptr;
  auto seg_end = [&](int row) {
    // warp state -> state buffer k % NSB, once the merge warp is done with segment k - NSB
    const int k = qseg - 1;
    const int sbi = k % C::NSB;
    float* sb = sm_state + sbi * C::SBUF_F;
    if (k >= C::NSB) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_sfree[sbi], ((k / C::NSB) - 1) & 1, abort_flag, wl));
      if (!ok) {
        if (lane == 0 && !*abort_flag) atomicOr(gm.status, KVQ_DEV_WAIT_TIMEOUT);
        *abort_flag = 1;
      }
    }
    o_to_unit();
    float* s_m = sb;
    float* s_l = sb + C::NC * C::HS;
    float* s_o = sb + C::SO;
    if constexpr (TR) {
      // head tc: l and wz summed over the 8 lanes gr
      float ls = l, wzs = wz;
#pragma unroll
      for (int x = 4; x < 32; x <<= 1) {
        ls += __shfl_xor_sync(0xffffffffu, ls, x);
        wzs += __shfl_xor_sync(0xffffffffu, wzs, x);
      }
      if (gr == 0) {
        s_m[cw * C::HS + tc] = m;
        s_l[cw * C::HS + tc] = ls;
      }
#pragma unroll
      for (int mt = 0; mt < NO; ++mt) {
        s_o[(cw * C::HS + tc) * D + 16 * mt + gr] = o[mt][0] + o[mt][1] + wzs;
        s_o[(cw * C::HS + tc) * D + 16 * mt + 8 + gr] = o[mt][2] + o[mt][3] + wzs;
      }
    } else {
      // softmax state of head gr; output columns heads 2 tc, 2 tc + 1
      const float ls = quad_sum(l), wzs = quad_sum(wz);
      if (tc == 0) {
        s_m[cw * C::HS + gr] = m;
        s_l[cw * C::HS + gr] = ls;
      }
      const float wz0 = __shfl_sync(0xffffffffu, wzs, 8 * tc), wz1 = __shfl_sync(0xffffffffu, wzs, 8 * tc + 4);
      float* o0 = s_o + (cw * C::HS + 2 * tc) * D;
      float* o1 = o0 + D;
#pragma unroll
      for (int mt = 0; mt < NO; ++mt) {
        o0[16 * mt + gr] = o[mt][0] + wz0;
        o1[16 * mt + gr] = o[mt][1] + wz1;
        o0[16 * mt + 8 + gr] = o[mt][2] + wz0;
        o1[16 * mt + 8 + gr] = o[mt][3] + wz1;
      }
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&bar_qempty[k & 1]);   // this warp is done with the segment's q
      mbar_arrive(&bar_sfull[sbi]);
    }
    if (row == last_row) {   // the CTA's last segment: merged by all consumer warps after the loop
      final_row = row;
      final_sb = sb;
    }
  };

  // the CTA range of the last segment's row, computed while the first stage loads
  int fin_c0 = 0, fin_np = 1;
  if (last_row >= 0) {
    const int it = last_row * Pt.n_items;
    fin_c0 = Pt.cta_of(it);
    fin_np = Pt.cta_of(it + Pt.n_items - 1) - fin_c0 + 1;
    asm volatile("" ::"r"(fin_c0), "r"(fin_np));
  }
  for_each_chunk<C::SG>(Pt, i0, i1, chunk, seg_begin, seg_end);
  if (final_row >= 0) {
    consumer_bar<C::NC>();   // every consumer warp's state of the segment is written
    merge_segment(final_row, final_sb, threadIdx.x - 96, C::NC * 32, [] { consumer_bar<C::NC>(); }, fin_c0, fin_np);
  }
}

template <int BITS, int D, int G, bool TR>
void launch_decode(const AttnArgs& a, cudaStream_t st) {
  using C = K<BITS, D, G, TR>;
  auto kern = kivi_decode_kernel<BITS, D, G, TR>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    attr_set = true;
  }
  kern<<<a.n_cta, C::THREADS, C::SMEM, st>>>(a);
  count_launch(1);
}

template <int BITS, int D, int G>
void launch_decode(const AttnArgs& a, cudaStream_t st) {
  if (a.geom.g <= 4) launch_decode<BITS, D, G, true>(a, st);
  else launch_decode<BITS, D, G, false>(a, st);
}

}  // namespace

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

// TurboQuant-style quantization on the 5th-generation tensor cores (16-bit
// sources; either rotation, Pi taken as its dense table).  The arithmetic and the readings are those of
// tq_quantize_kernel in tq_quant.cu ("Quantification du KV-Cache : TurboQuant
// et l'etat de l'art en 2026", "TurboQuant : les cinq innovations", items 1-3):
// n = ||x|| (fp64 sum), y = Pi x / n to about fp32 precision, the 3-bit
// Lloyd-Max cell of each coordinate of y (a coordinate equal to a threshold
// goes to the lower cell), the residual e = y - c_hat in rotated coordinates,
// the signs of S e (exactly 0 gives bit 1) and gamma = n ||e||.
//
// A tile is 128 tokens: four 32-token blocks (tasks) in task order.  Each
// product is one chain of tcgen05.mma over the whole tile (M = 128 tokens,
// N = 128 outputs, K = 128 summed coordinates in 8 steps of 16), in the
// input's 16-bit type with fp32 accumulation:
//   16 Pi x = x (16 Pi hi) + x (16 Pi lo): the input x is exact in its own type,
//      so A needs no split and y = (16 Pi x) / (16 n) is divided out in the
//      thresholds and the residual (per-token constants);
//   64 S e = eh Sh + eh Sl + el Sh with (64 e) split into hi + lo (the dropped
//      lo*lo term is below 2^-16 of each product in bf16, 2^-22 in fp16).
//   A  x, or the split 64 e, in tensor memory, one lane per token, written by
//      the thread that owns the token;
//   B  images of 16 Pi and S split hi + lo in the input's type, from the
//      parameter block, kept in shared memory for the whole launch;
//   D  fp32 in tensor memory.
// The scalings keep the lo parts clear of fp16 subnormals.
//
// Warp roles (544 threads, one persistent CTA per SM):
//   warps 0-15  token warps: warp w serves the tensor-memory lane quadrant
//               q = w % 4, so thread (w, l) owns token 32 q + l of the tile,
//               and r = w / 4 picks keys (r < 2) or values and the half of
//               the 128 coordinates it handles (r % 2).  The two halves of a
//               token meet in shared memory for its norm, ||e||^2 and sign
//               words (a 64-thread named barrier per kind and quadrant).
//   warp 16     lane 0 issues the mma chains and commits them to mbarriers
// Keys: norm and x into A; after y the codes, e, ||e||^2 and split e; after
// S e the sign bits and (n, gamma).  Values: norm, x into A, codes, n.
// Tensor memory (512 columns): keys D 0-127, A hi 128-191, A lo 192-255 (e
// reuses A, S e reuses D); values D 256-383, A hi 384-447, A lo 448-511.  The
// value chain runs while the key warps code y, the S e chain while the value
// warps code theirs.  Key threads write their 6-bit pair indices in record
// slot order; value threads combine their codes with the next token's (the
// next lane) into pair indices.  The key warps and the value warps (256
// threads each) then run as two groups: each packs the words of its own kind
// from its own index tile.  The values pack while the keys wait for S e; the
// keys run the next tile's A stage before packing, so that its y chain runs
// meanwhile (the value warps run theirs after packing).
// Every wait is bounded and idles with a short sleep instead of spinning; a
// wait that gives up sets KVQ_DEV_WAIT_TIMEOUT and the CTA stops at the next
// tile boundary, after its issued chains complete.
#include <cuda_runtime.h>

#include "kvq_internal.cuh"
#include "tc_common.cuh"

namespace kvq {

namespace {

constexpr int kTcTok = 128;
constexpr int kTokWarps = 16;
constexpr int kTokThreads = kTokWarps * 32;
constexpr int kTcThreads = kTokThreads + 32;
constexpr int kTcCols = 512;

struct TcSmem {
  static constexpr int B = 0;                          // 16 Pi hi, 16 Pi lo, S hi, S lo
  static constexpr int IK = B + 4 * kTqBImgBytes;      // uint8 [4 blocks][32 lanes][kIKRow] key pair indices (64 slots)
  static constexpr int IV = IK + 4 * 32 * 72;          // uint8 [64 token pairs][kIVRow] value pair indices (128 coordinates)
  static constexpr int NP = IV + 64 * 144;             // double [2 kinds][2 halves][128] partial sums of squares
  static constexpr int EP = NP + 2 * 2 * 128 * 8;      // float [128] partial ||64 e||^2 of the low half
  static constexpr int SW = EP + 128 * 4;              // uint32 [128][4] sign words of the low half
  static constexpr int XS = SW + 128 * 16;             // [2 kinds][128 tokens][kXRow] staged input rows
  static constexpr int BYTES = XS + 2 * 128 * 272;
};
constexpr int kXRow = 272;   // staged row pitch: 256 bytes + 16, so 8 consecutive rows fall 4 banks apart
// index tile pitches, padded so that the lanes of a packing or index-writing
// warp spread over the banks instead of hitting one column
constexpr int kIKRow = 72;
constexpr int kIVRow = 144;
static_assert(TcSmem::BYTES <= 227 * 1024, "TurboQuant tensor-core quantizer exceeds shared memory");

template <bool BF>
__device__ __forceinline__ float in16f(uint32_t bits16) {
  return BF ? __uint_as_float(bits16 << 16) : __half2float(__ushort_as_half((uint16_t)bits16));
}

// hi + lo split of two fp32 values in the 16-bit type (fp16, or bf16), packed as pairs
template <bool BF>
__device__ __forceinline__ void split_pair(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  if constexpr (BF) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
  } else {
    const __half2 h = __floats2half2_rn(v0, v1);
    const float2 hf = __half22float2(h);
    hi = h2_as_u32(h);
    lo = h2_as_u32(__floats2half2_rn(v0 - hf.x, v1 - hf.y));
  }
}

// Bounded wait that sleeps between polls (the waits here last microseconds;
// polling would take issue slots from the warps that work meanwhile).
__device__ __forceinline__ bool mbar_wait_nap(uint64_t* b, uint32_t parity, volatile int* abort_flag, long long limit) {
  if (mbar_try_wait(b, parity)) return true;
  const long long t0 = clock64();
  uint32_t ns = 32;
  for (;;) {
    __nanosleep(ns);
    if (mbar_try_wait(b, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) return false;
    if (ns < 256) ns <<= 1;
  }
}

__device__ __forceinline__ void bar_pair(int id) { asm volatile("bar.sync %0, 64;\n" ::"r"(id) : "memory"); }
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}

// The chain D = A_hi B_hi + A_hi B_lo (+ A_lo B_hi when SPLIT_A) over K = 128.
template <bool BF, bool SPLIT_A>
__device__ __forceinline__ void issue_product(uint32_t d, uint32_t a_hi, uint32_t a_lo, const unsigned char* b_hi,
                                              const unsigned char* b_lo) {
  constexpr uint32_t idesc = umma_idesc_f16(kTcTok, kTqD, BF);
#pragma unroll
  for (int kk = 0; kk < kTqD / 16; ++kk) {
    const uint64_t bh = umma_sdesc(b_hi + kk * 4096, 2048, 128);
    const uint64_t bl = umma_sdesc(b_lo + kk * 4096, 2048, 128);
    umma_ts(d, a_hi + 8 * kk, bh, idesc, kk > 0);
    umma_ts(d, a_hi + 8 * kk, bl, idesc, true);
    if (SPLIT_A) umma_ts(d, a_lo + 8 * kk, bh, idesc, true);
  }
}

__device__ __forceinline__ uint32_t gt_mask(float a, float b) {   // 0xFFFFFFFF if a > b, else 0
  uint32_t r;
  asm("set.gt.u32.f32 %0, %1, %2;\n" : "=r"(r) : "f"(a), "f"(b));
  return r;
}
// 3-bit cell of a coordinate from d = 16 n y and the thresholds T4 < T5 < T6
// of the positive half scaled the same way.  The deployed codebook is
// symmetric (T_{6-k} = -T_k, T3 = 0; the setup makes it so), so the cell is
// 4 + #{T_k < d} for d > 0 and 3 - #{T_k < |d|} otherwise.  (A negative d
// exactly on a threshold would take the upper of the two cells; such a d lies
// within the rounding error of the exact coordinate, where either is accepted.)
__device__ __forceinline__ uint32_t cell_sym(float d, float t4, float t5, float t6) {
  const float ad = fabsf(d);
  const uint32_t s = gt_mask(ad, t4) + gt_mask(ad, t5) + gt_mask(ad, t6);   // minus the count
  return d > 0.f ? 4u - s : 3u + s;
}

template <bool BF>
__global__ void __launch_bounds__(kTcThreads, 1) tq_quantize_tc_kernel(QuantArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar_b, bar_fin, bar_a[2], bar_d[2];
  __shared__ uint32_t s_tmem, s_flags;
  __shared__ int s_abort;
  __shared__ float s_t256[8], s_lv64[8];
  __shared__ uint32_t* s_rec[2][2][4];   // [kind][tile parity]: records of a tile's four tasks (null: none or outside the pool)

  const Geom& gm = a.geom;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned char* sB = smem + TcSmem::B;
  uint8_t* sIK = smem + TcSmem::IK;
  uint8_t* sIV = smem + TcSmem::IV;
  double* sNP = reinterpret_cast<double*>(smem + TcSmem::NP);
  float* sEP = reinterpret_cast<float*>(smem + TcSmem::EP);
  uint32_t* sSW = reinterpret_cast<uint32_t*>(smem + TcSmem::SW);

  if (tid == 0) {
    mbar_init(&bar_b, 1);
    mbar_init(&bar_fin, 1);
    mbar_init(&bar_a[0], 256);
    mbar_init(&bar_a[1], 256);
    mbar_init(&bar_d[0], 1);
    mbar_init(&bar_d[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    s_flags = 0;
    s_abort = 0;
  }
  if (tid < 8) {
    const float* P = reinterpret_cast<const float*>(gm.params);
    s_t256[tid] = P[kTqThr / 4 + tid] * 256.f;
    s_lv64[tid] = P[kTqLevels / 4 + tid] * 64.f;
  }
  if (warp == 0) tmem_alloc(&s_tmem, kTcCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = s_tmem;

  const int64_t n_tasks = (int64_t)gm.B * gm.Hkv * a.n_groups;
  const int64_t n_tiles = (n_tasks + 3) / 4;
  uint32_t flags = 0;

  if (warp == kTokWarps) {
    // ------------------------------------------------------------ mma issue
    if (lane == 0) {
      // (test hook: CTA 0 may withhold the copy, so that the wait below runs out)
      const bool withheld = a.withhold_first_stage && blockIdx.x == 0;
      if (!withheld) {
        mbar_expect_tx(&bar_b, 4 * kTqBImgBytes);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          bulk_g2s(sB + i * kTqBImgBytes, gm.params + kTqBImg + (BF ? kTqBImgSet : 0) + i * kTqBImgBytes, kTqBImgBytes,
                   &bar_b);
      }
      bool ok = mbar_wait_nap(&bar_b, 0, &s_abort, a.wait_cycles);
      if (!ok && !withheld) mbar_drain(&bar_b, 0);   // the copy in flight lands before the CTA exits
      const unsigned char *pi_hi = sB, *pi_lo = sB + kTqBImgBytes;
      const unsigned char *s_hi = sB + 2 * kTqBImgBytes, *s_lo = sB + 3 * kTqBImgBytes;
      int64_t it = 0;
      for (int64_t tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++it) {
        if (!(ok = mbar_wait_nap(&bar_a[0], 0, &s_abort, a.wait_cycles))) break;
        tc_fence_after();
        issue_product<BF, false>(tbase, tbase + 128, tbase + 192, pi_hi, pi_lo);
        umma_commit(&bar_d[0]);
        if (!(ok = mbar_wait_nap(&bar_a[1], (uint32_t)(it & 1), &s_abort, a.wait_cycles))) break;
        tc_fence_after();
        issue_product<BF, false>(tbase + 256, tbase + 384, tbase + 448, pi_hi, pi_lo);
        umma_commit(&bar_d[1]);
        if (!(ok = mbar_wait_nap(&bar_a[0], 1, &s_abort, a.wait_cycles))) break;
        tc_fence_after();
        issue_product<BF, true>(tbase, tbase + 128, tbase + 192, s_hi, s_lo);
        umma_commit(&bar_d[0]);
      }
      if (!ok) {
        flags |= KVQ_DEV_WAIT_TIMEOUT;
        s_abort = 1;
      }
      // every chain issued so far has completed before the CTA frees tensor memory
      umma_commit(&bar_fin);
      mbar_drain(&bar_fin, 0);
    }
  } else {
    // ------------------------------------------------------------ token warps
    const int q = warp & 3, r = warp >> 2;
    const int kind = r >> 1, h = r & 1;           // kind 0 keys, 1 values; coordinate half h
    const int m = 32 * q + lane;                  // token row of the tile
    const int tt = m & 31, tbm = m >> 5;          // token of its block, block of the tile
    const int pair_bar = 1 + 4 * kind + q;        // the two halves of these 32 tokens
    const uint32_t t_d = tbase + ((uint32_t)(32 * q) << 16) + (kind ? 256u : 0u);
    const uint32_t t_hi = t_d + 128, t_lo = t_d + 192;
    const float t4 = s_t256[4], t5 = s_t256[5], t6 = s_t256[6];   // thresholds x 256 (positive half)
    const int entry = 8 * ((tt >> 1) & 3) + 4 * (tt >> 4) + 2 * ((tt >> 3) & 1) + (tt & 1);
    const double rng = recip(a.n_groups);
    // The thread's half row of a tile is staged with cp.async one tile ahead,
    // into a shared-memory region only this thread reads.
    unsigned char* xs = smem + TcSmem::XS + (kind * 128 + m) * kXRow + 128 * h;
    auto stage_rows = [&](int64_t t) {
      const int64_t tk = t * 4 + tbm;
      if (t < n_tiles && tk < n_tasks) {
        const int rw = (int)div_floor(tk, a.n_groups, rng);
        const int64_t bk = tk - (int64_t)rw * a.n_groups;
        const uint16_t* g = (kind ? a.src_v : a.src_k) + (int64_t)rw * a.src_row_stride + (bk * kTB + tt) * kTqD + 64 * h;
#pragma unroll
        for (int i = 0; i < 8; ++i) cp_async16(xs + 16 * i, g + 8 * i);
      }
      asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
    // The A stage of a tile: its records, the norm, x into the A operand, the
    // per-token constants; then the next tile's rows are staged and the A
    // operand is signalled.  It runs for tile i + 1 before tile i's words are
    // packed, so the tensor core computes the next y while the warps pack.
    bool valid = false;
    unsigned char* dst = nullptr;
    double ss = 0.0;
    float T4 = 0.f, T5 = 0.f, T6 = 0.f, c4 = 0.f;
    auto stage_a = [&](int64_t t, int par) {
      const int64_t task = t * 4 + tbm;
      valid = task < n_tasks;
      int row = 0;
      int64_t blk = 0;
      if (valid) {
        row = (int)div_floor(task, a.n_groups, rng);
        blk = task - (int64_t)row * a.n_groups;
      }
      dst = valid ? reinterpret_cast<unsigned char*>(record_ptr(gm, row, a.dst_group0 + blk)) : nullptr;
      if (h == 0 && tt == 0) {   // each kind's group keeps its own copy
        s_rec[kind][par][tbm] = reinterpret_cast<uint32_t*>(dst);
        if (kind == 0 && valid && dst == nullptr) flags |= KVQ_DEV_BAD_PAGE;   // page outside the pool: nothing is written
      }
      asm volatile("cp.async.wait_group 0;\n" ::: "memory");
      const uint4* src = reinterpret_cast<const uint4*>(xs);
      double s0 = 0.0, s1 = 0.0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 rv = valid ? src[i] : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const double x0 = in16f<BF>(w[k] & 0xFFFFu), x1 = in16f<BF>(w[k] >> 16);
          s0 = fma(x0, x0, s0);
          s1 = fma(x1, x1, s1);
        }
      }
      // the raw 16-bit pairs are the A operand as they stand (coordinate pair j = column j)
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        uint32_t xv[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 rv = valid ? src[4 * g + i] : make_uint4(0, 0, 0, 0);
          xv[4 * i] = rv.x;
          xv[4 * i + 1] = rv.y;
          xv[4 * i + 2] = rv.z;
          xv[4 * i + 3] = rv.w;
        }
        tmem_st16(t_hi + 32 * h + 16 * g, xv);
      }
      stage_rows(t + gridDim.x);   // this thread's staged rows are consumed
      sNP[(2 * kind + h) * 128 + m] = s0 + s1;
      bar_pair(pair_bar);
      ss = sNP[(2 * kind) * 128 + m] + sNP[(2 * kind + 1) * 128 + m];
      if (h == 0 && !isfinite(ss)) flags |= KVQ_DEV_NONFINITE_INPUT;
      const double n = sqrt(ss);
      // D = 16 n y: thresholds 16 n t_k (the table holds 256 t_k), and 64 y = D * 4 / n
      const float tn = (float)(n * (1.0 / 16.0));
      T4 = tn * t4;
      T5 = tn * t5;
      T6 = tn * t6;
      c4 = n > 0.0 ? (float)(4.0 / n) : 0.f;
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_a[kind]);
    };
    stage_rows(blockIdx.x);
    if (blockIdx.x < n_tiles) stage_a(blockIdx.x, 0);
    int64_t it = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      // ---------------------------------------------------------- y: codes (keys also e)
      // (ok is made warp-uniform: tcgen05.ld / st and the shuffle below are warp-collective)
      bool ok = __all_sync(0xffffffffu, mbar_wait_nap(&bar_d[kind], kind ? (uint32_t)(it & 1) : 0u, &s_abort, a.wait_cycles));
      if (!ok) s_abort = 1;
      if (kind == 0) {
        float es = 0.f;
        if (ok) {
          tc_fence_after();
          uint32_t kx[4][2];   // pair indices of slots 8 h .. 8 h + 7 of quad lane tc, one byte each
#pragma unroll
          for (int c = 0; c < 4; ++c) {   // 16 coordinates (8 pairs) at a time
            uint32_t rr[16];
            tmem_ld16(t_d + 64 * h + 16 * c, rr);
            tc_wait_ld();
            uint32_t eh[8], el[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
              const float y0 = __uint_as_float(rr[2 * p]), y1 = __uint_as_float(rr[2 * p + 1]);   // 16 n y
              const uint32_t c0 = cell_sym(y0, T4, T5, T6), c1 = cell_sym(y1, T4, T5, T6);
              // pair 32 h + 8 c + p: quad lane p & 3, slot 8 h + 2 c + p / 4
              const uint32_t idx = (c0 + 8u * c1) << (8 * (2 * (c & 1) + (p >> 2)));
              if ((c & 1) == 0 && (p >> 2) == 0) kx[p & 3][c >> 1] = idx;
              else kx[p & 3][c >> 1] |= idx;
              const float e0 = fmaf(y0, c4, -s_lv64[c0]), e1 = fmaf(y1, c4, -s_lv64[c1]);   // 64 e
              es = fmaf(e0, e0, es);
              es = fmaf(e1, e1, es);
              split_pair<BF>(e0, e1, eh[p], el[p]);
            }
            tmem_st8(t_hi + 32 * h + 8 * c, eh);
            tmem_st8(t_lo + 32 * h + 8 * c, el);
          }
          // key pair indices: lane 4 gr + tc of the block, slots 16 nt + 8 h .. + 7
          uint8_t* ik = sIK + tbm * 32 * kIKRow + 16 * (tt >> 3) + 8 * h;
#pragma unroll
          for (int tc = 0; tc < 4; ++tc)
            *reinterpret_cast<uint2*>(ik + (4 * (tt & 7) + tc) * kIKRow) = make_uint2(kx[tc][0], kx[tc][1]);
          if (h == 0) sEP[m] = es;
          // S e: the residual into the A operand, then the signs
          tc_wait_st();
          tc_fence_before();
          mbar_arrive(&bar_a[0]);
          ok = __all_sync(0xffffffffu, mbar_wait_nap(&bar_d[0], 1u, &s_abort, a.wait_cycles));
          if (!ok) s_abort = 1;
        }
        uint32_t sw[4] = {0u, 0u, 0u, 0u};
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t rr[16];
            tmem_ld16(t_d + 64 * h + 16 * c, rr);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int i = 64 * h + 16 * c + j;   // sketch row: quad lane (i >> 1) & 3, bit 2 kt + rho (+ 16)
              const uint32_t bit = 1u << (2 * (i >> 4) + ((i >> 3) & 1) + 16 * (i & 1));
              if (__uint_as_float(rr[j]) >= 0.f) sw[(i >> 1) & 3] |= bit;
            }
          }
        }
        if (h == 0) *reinterpret_cast<uint4*>(sSW + 4 * m) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
        bar_pair(pair_bar);   // both halves reach it, whatever their waits returned
        // a half whose wait gave up set s_abort before the barrier: its words are then incomplete
        const bool both = ok && !s_abort;
        if (both && h == 1) {
          const uint4 o = *reinterpret_cast<const uint4*>(sSW + 4 * m);
          const double n = sqrt(ss);
          const __half hn = __double2half(n);
          const __half hg = __double2half(n * sqrt((double)(sEP[m] + es) * (1.0 / 4096.0)));
          if (isinf(__half2float(hn)) || isinf(__half2float(hg))) flags |= KVQ_DEV_PARAM_OVERFLOW;
          if (dst != nullptr) {
            uint32_t* sg = reinterpret_cast<uint32_t*>(dst + kTqSigns) + 4 * (4 * (tt & 7)) + (tt >> 3);
            sg[0] = sw[0] | o.x;
            sg[4] = sw[1] | o.y;
            sg[8] = sw[2] | o.z;
            sg[12] = sw[3] | o.w;
            reinterpret_cast<uint32_t*>(dst + kTqKMeta)[entry] =
                (uint32_t)__half_as_ushort(hn) | ((uint32_t)__half_as_ushort(hg) << 16);
          }
        }
      } else if (ok) {
        tc_fence_after();
        uint32_t cw[16];   // codes of coordinates 64 h + 4 k .. + 3, one byte each
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t rr[16];
          tmem_ld16(t_d + 64 * h + 16 * c, rr);
          tc_wait_ld();
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const uint32_t pr = cell_sym(__uint_as_float(rr[2 * p]), T4, T5, T6) |
                                (cell_sym(__uint_as_float(rr[2 * p + 1]), T4, T5, T6) << 8);
            if (p & 1) cw[4 * c + (p >> 1)] |= pr << 16;
            else cw[4 * c + (p >> 1)] = pr;
          }
        }
        // value pair indices: this token's codes plus 8 x the next token's (the next lane)
#pragma unroll
        for (int k = 0; k < 16; ++k) cw[k] += __shfl_down_sync(0xffffffffu, cw[k], 1) << 3;
        if ((lane & 1) == 0) {
          uint4* iv = reinterpret_cast<uint4*>(sIV + (m >> 1) * kIVRow + 64 * h);
#pragma unroll
          for (int k = 0; k < 4; ++k) iv[k] = make_uint4(cw[4 * k], cw[4 * k + 1], cw[4 * k + 2], cw[4 * k + 3]);
        }
        if (h == 0) {
          const __half hv = __double2half(sqrt(ss));
          if (isinf(__half2float(hv))) flags |= KVQ_DEV_PARAM_OVERFLOW;
          if (dst != nullptr) reinterpret_cast<uint16_t*>(dst + kTqVMeta)[entry] = __half_as_ushort(hv);
        }
      }
      // The key and value warps (256 each) run as two groups from here: each
      // agrees on stopping, packs the code words of its own kind from its own
      // index tile, and frees that tile with its own barrier.  Keys start the
      // next tile's A stage before packing (the next y then runs meanwhile);
      // values pack first, while the key warps wait for S e and take signs.
      const int grp_bar = 9 + kind;
      if (bar_red_or(grp_bar, kTokThreads / 2, !ok)) {
        flags |= KVQ_DEV_WAIT_TIMEOUT;
        break;
      }
      const bool more = tile + gridDim.x < n_tiles;
      if (kind == 0 && more) stage_a(tile + gridDim.x, (int)((it + 1) & 1));

      // ---------------------------------------------------------- pack this kind's code words of the tile
      // word i of a block's key (value) codes: i < 384 is word 4 (i / 128) + i % 4
      // of lane (i / 4) % 32, i >= 384 word 12 of lane i - 384
      const int gtid = tid - kind * (kTokThreads / 2);
#pragma unroll 1
      for (int item = gtid; item < 4 * 416; item += kTokThreads / 2) {
        const int tb = item / 416, i = item - 416 * tb;
        uint32_t* out = s_rec[kind][it & 1][tb];
        if (out == nullptr) continue;
        const int ln = i < 384 ? (i >> 2) & 31 : i - 384;
        const int w = i < 384 ? 4 * (i >> 7) + (i & 3) : 12;
        uint32_t word = 0;
        if (kind == 0) {
          // slots 5 w .. 5 w + 4 of the lane's 64 index bytes
          const uint8_t* ib = sIK + tb * 32 * kIKRow + ln * kIKRow;
          const int b0 = 5 * w;
          const uint32_t lo = *reinterpret_cast<const uint32_t*>(ib + (b0 & ~3));
          const uint32_t hi = (b0 & ~3) + 4 < 64 ? *reinterpret_cast<const uint32_t*>(ib + (b0 & ~3) + 4) : 0u;
          const uint64_t v = ((uint64_t)hi << 32 | lo) >> (8 * (b0 & 3));
#pragma unroll
          for (int f = 0; f < 5; ++f) word |= (uint32_t)((v >> (8 * f)) & 0x3Fu) << (6 * f);
          if (w == 12) word &= 0x00FFFFFFu;   // slots 60..63 only
        } else {
          // value pair (kt, nt, rho) of slot s: coordinate 8 nt + gr, token pair 8 kt + 4 rho + tc
          const int gr = ln >> 2, tc = ln & 3;
#pragma unroll
          for (int f = 0; f < 5; ++f) {
            const int sl = 5 * w + f;
            if (sl < 64) {
              const int kt = sl >> 5, nt = (sl >> 1) & 15, rho = sl & 1;
              word |= (uint32_t)sIV[(16 * tb + 8 * kt + 4 * rho + tc) * kIVRow + 8 * nt + gr] << (6 * f);
            }
          }
        }
        out[(kind ? kTqVCodes : kTqKCodes) / 4 + i] = word;
      }
      if (kind == 1 && more) stage_a(tile + gridDim.x, (int)((it + 1) & 1));
      asm volatile("bar.sync %0, %1;\n" ::"r"(grp_bar), "r"(kTokThreads / 2) : "memory");   // index tile free
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");   // no staging copy outlives the loop
  }

  if (flags) atomicOr(&s_flags, flags);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, kTcCols);
  if (tid == 0 && s_flags) atomicOr(gm.status, s_flags);
}

}  // namespace

void launch_tq_quantize_tc(const QuantArgs& a, cudaStream_t st) {
  const int64_t tasks = (int64_t)a.geom.B * a.geom.Hkv * a.n_groups;
  if (tasks <= 0) return;
  auto kern = a.geom.dtype == KVQ_BF16 ? tq_quantize_tc_kernel<true> : tq_quantize_tc_kernel<false>;
  static bool attr_set[2] = {false, false};
  const int di = a.geom.dtype == KVQ_BF16;
  if (!attr_set[di]) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSmem::BYTES);
    attr_set[di] = true;
  }
  const int64_t tiles = (tasks + 3) / 4;
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  kern<<<grid, kTcThreads, TcSmem::BYTES, st>>>(a);
  count_launch(1);
}

}  // namespace kvq

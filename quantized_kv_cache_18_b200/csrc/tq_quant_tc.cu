// TurboQuant-style quantization on the 5th-generation tensor cores (dense QR
// rotation, 16-bit sources).  The arithmetic and the readings are those of
// tq_quantize_kernel in tq_quant.cu ("Quantification du KV-Cache : TurboQuant
// et l'etat de l'art en 2026", "TurboQuant : les cinq innovations", items 1-3):
// n = ||x|| (fp64 sum), u = x / n, y = Pi u to about fp32 precision, the 3-bit
// Lloyd-Max cell of each coordinate of y (a coordinate equal to a threshold
// goes to the lower cell), the residual e = y - c_hat in rotated coordinates,
// the signs of S e (exactly 0 gives bit 1) and gamma = n ||e||.
//
// A tile is 128 tokens: four 32-token blocks (tasks) in task order.  Each
// product is one chain of tcgen05.mma over the whole tile (M = 128 tokens,
// N = 128 outputs, K = 128 summed coordinates in 8 steps of 16), as three fp16
// terms hi*hi + hi*lo + lo*hi accumulated in fp32 (the dropped lo*lo term is
// below 2^-22 of each product):
//   A  (16 u) or (64 e) split into fp16 hi + lo, in tensor memory, one lane
//      per token, written by the thread that owns the token;
//   B  16 Pi and S split the same way, images from the parameter block kept
//      in shared memory for the whole launch;
//   D  fp32 in tensor memory: 256 y, then 64 S e.
// The scalings keep the lo parts clear of fp16 subnormals.
//
// Warp roles (288 threads, one persistent CTA per SM):
//   warps 0-3  keys; thread (w, l) owns token 32 w + l of the tile: norm and
//              split u; after y its codes, e, ||e||^2 and split e; after S e
//              its sign bits and (n, gamma)
//   warps 4-7  values, the same rows: norm, split u, codes, n
//   warp 8     lane 0 issues the mma chains and commits them to mbarriers
// Tensor memory (512 columns): keys D 0-127, A hi 128-191, A lo 192-255 (e
// reuses A, S e reuses D); values D 256-383, A hi 384-447, A lo 448-511.  The
// value chain runs while the key warps code y, the S e chain while the value
// warps code theirs.  The eight token warps then pack the tile's code words.
// Every wait is bounded; a wait that gives up sets KVQ_DEV_WAIT_TIMEOUT and
// the CTA stops at the next tile boundary, after its issued chains complete.
#include <cuda_runtime.h>

#include "kvq_internal.cuh"
#include "tc_common.cuh"

namespace kvq {

namespace {

constexpr int kTcTok = 128;
constexpr int kTcThreads = 288;
constexpr int kTcCols = 512;
constexpr int kCodeRow = 144;   // code tile row stride (bytes): 16-byte aligned rows, 4 banks apart

struct TcSmem {
  static constexpr int B = 0;                               // 16 Pi hi, 16 Pi lo, S hi, S lo
  static constexpr int CK = B + 4 * kTqBImgBytes;           // uint8 [128][kCodeRow] key codes
  static constexpr int CV = CK + kTcTok * kCodeRow;         // uint8 [128][kCodeRow] value codes
  static constexpr int BYTES = CV + kTcTok * kCodeRow;
};
static_assert(TcSmem::BYTES <= 227 * 1024, "TurboQuant tensor-core quantizer exceeds shared memory");

// fp16 hi + lo split of two fp32 values, packed as fp16x2 pairs
__device__ __forceinline__ void split_pair(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(v0, v1);
  const float2 hf = __half22float2(h);
  hi = h2_as_u32(h);
  lo = h2_as_u32(__floats2half2_rn(v0 - hf.x, v1 - hf.y));
}

// The chain D = A_hi B_hi + A_hi B_lo + A_lo B_hi over K = 128.
__device__ __forceinline__ void issue_product(uint32_t d, uint32_t a_hi, uint32_t a_lo, const unsigned char* b_hi,
                                              const unsigned char* b_lo) {
  constexpr uint32_t idesc = umma_idesc_f16(kTcTok, kTqD);
#pragma unroll
  for (int kk = 0; kk < kTqD / 16; ++kk) {
    const uint64_t bh = umma_sdesc(b_hi + kk * 4096, 2048, 128);
    const uint64_t bl = umma_sdesc(b_lo + kk * 4096, 2048, 128);
    umma_ts(d, a_hi + 8 * kk, bh, idesc, kk > 0);
    umma_ts(d, a_hi + 8 * kk, bl, idesc, true);
    umma_ts(d, a_lo + 8 * kk, bh, idesc, true);
  }
}

// Loads the thread's token (128 16-bit coordinates; zeros when src is null),
// returns n = ||x|| and writes (16 u) split hi | lo into its tensor-memory lane.
__device__ __forceinline__ double load_split_unit(const uint16_t* src, int dtype, uint32_t t_hi, uint32_t t_lo,
                                                  uint32_t& flags) {
  uint4 raw[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) raw[i] = src != nullptr ? ldg_nc_v4(src + 8 * i) : make_uint4(0, 0, 0, 0);
  double s0 = 0.0, s1 = 0.0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const double x0 = in16_to_float((uint16_t)(w[q] & 0xFFFFu), dtype);
      const double x1 = in16_to_float((uint16_t)(w[q] >> 16), dtype);
      s0 = fma(x0, x0, s0);
      s1 = fma(x1, x1, s1);
    }
  }
  const double s = s0 + s1;
  if (!isfinite(s)) flags |= KVQ_DEV_NONFINITE_INPUT;
  const double n = sqrt(s);
  const float f = n > 0.0 ? (float)(1.0 / n) * 16.f : 0.f;
#pragma unroll
  for (int h = 0; h < 4; ++h) {   // 32 coordinates = 16 columns at a time
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 r = raw[4 * h + i];
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        split_pair(in16_to_float((uint16_t)(w[q] & 0xFFFFu), dtype) * f, in16_to_float((uint16_t)(w[q] >> 16), dtype) * f,
                   hi[4 * i + q], lo[4 * i + q]);
    }
    tmem_st16(t_hi + 16 * h, hi);
    tmem_st16(t_lo + 16 * h, lo);
  }
  return n;
}

// code of 256 y against the thresholds scaled by 256 (ascending; the cell
// count of thresholds strictly below)
__device__ __forceinline__ uint32_t cell_of(float acc, const float* t) {
  uint32_t c = 0;
#pragma unroll
  for (int k = 0; k < 7; ++k) c += acc > t[k] ? 1u : 0u;
  return c;
}

__global__ void __launch_bounds__(kTcThreads, 1) tq_quantize_tc_kernel(QuantArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar_b, bar_fin, bar_a[2], bar_d[2];
  __shared__ uint32_t s_tmem, s_flags;
  __shared__ int s_abort;
  __shared__ float s_t256[8], s_lv64[8];

  const Geom& gm = a.geom;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned char* sB = smem + TcSmem::B;
  uint8_t* sCK = smem + TcSmem::CK;
  uint8_t* sCV = smem + TcSmem::CV;

  if (tid == 0) {
    mbar_init(&bar_b, 1);
    mbar_init(&bar_fin, 1);
    mbar_init(&bar_a[0], 128);
    mbar_init(&bar_a[1], 128);
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

  if (warp == 8) {
    // ------------------------------------------------------------ mma issue
    if (lane == 0) {
      mbar_expect_tx(&bar_b, 4 * kTqBImgBytes);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        bulk_g2s(sB + i * kTqBImgBytes, gm.params + kTqBImg + i * kTqBImgBytes, kTqBImgBytes, &bar_b);
      bool ok = mbar_wait(&bar_b, 0, &s_abort);
      if (!ok) mbar_drain(&bar_b, 0);
      const unsigned char *pi_hi = sB, *pi_lo = sB + kTqBImgBytes;
      const unsigned char *s_hi = sB + 2 * kTqBImgBytes, *s_lo = sB + 3 * kTqBImgBytes;
      int64_t it = 0;
      for (int64_t tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++it) {
        if (!(ok = mbar_wait(&bar_a[0], 0, &s_abort))) break;
        tc_fence_after();
        issue_product(tbase, tbase + 128, tbase + 192, pi_hi, pi_lo);
        umma_commit(&bar_d[0]);
        if (!(ok = mbar_wait(&bar_a[1], (uint32_t)(it & 1), &s_abort))) break;
        tc_fence_after();
        issue_product(tbase + 256, tbase + 384, tbase + 448, pi_hi, pi_lo);
        umma_commit(&bar_d[1]);
        if (!(ok = mbar_wait(&bar_a[0], 1, &s_abort))) break;
        tc_fence_after();
        issue_product(tbase, tbase + 128, tbase + 192, s_hi, s_lo);
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
    const int wg = warp >> 2;                       // 0 keys, 1 values
    const int m = 32 * (warp & 3) + lane;           // token row of the tile
    const uint32_t t_d = tbase + ((uint32_t)(32 * (warp & 3)) << 16) + (wg ? 256u : 0u);
    const uint32_t t_hi = t_d + 128, t_lo = t_d + 192;
    float thr[7];
#pragma unroll
    for (int k = 0; k < 7; ++k) thr[k] = s_t256[k];
    const int tt = m & 31;                          // token of its block
    const int entry = 8 * ((tt >> 1) & 3) + 4 * (tt >> 4) + 2 * ((tt >> 3) & 1) + (tt & 1);
    int64_t it = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int64_t task = tile * 4 + (m >> 5);
      const bool valid = task < n_tasks;
      int row = 0;
      int64_t blk = 0;
      if (valid) {
        row = (int)(task / a.n_groups);
        blk = task - (int64_t)row * a.n_groups;
      }
      const uint16_t* src =
          valid ? (wg ? a.src_v : a.src_k) + (int64_t)row * a.src_row_stride + (blk * kTB + tt) * kTqD
                : nullptr;
      unsigned char* dst = valid ? reinterpret_cast<unsigned char*>(record_ptr(gm, row, a.dst_group0 + blk)) : nullptr;

      // y: the unit vector into the A operand
      const double n = load_split_unit(src, gm.dtype, t_hi, t_lo, flags);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_a[wg]);

      bool ok = mbar_wait(&bar_d[wg], wg ? (uint32_t)(it & 1) : 0u, &s_abort);
      if (ok) {
        tc_fence_after();
        uint8_t* crow = (wg ? sCV : sCK) + m * kCodeRow;
        float es0 = 0.f, es1 = 0.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(t_d + 32 * c, r);
          tc_wait_ld();
          uint32_t cw[8], eh[16], el[16];
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const float y0 = __uint_as_float(r[2 * p]), y1 = __uint_as_float(r[2 * p + 1]);
            const uint32_t c0 = cell_of(y0, thr), c1 = cell_of(y1, thr);
            const uint32_t pr = c0 | (c1 << 8);
            if (p & 1) cw[p >> 1] |= pr << 16;
            else cw[p >> 1] = pr;
            if (wg == 0) {
              const float e0 = fmaf(y0, 0.25f, -s_lv64[c0]), e1 = fmaf(y1, 0.25f, -s_lv64[c1]);   // 64 e
              es0 = fmaf(e0, e0, es0);
              es1 = fmaf(e1, e1, es1);
              split_pair(e0, e1, eh[p], el[p]);
            }
          }
          *reinterpret_cast<uint4*>(crow + 32 * c) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
          *reinterpret_cast<uint4*>(crow + 32 * c + 16) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
          if (wg == 0) {
            tmem_st16(t_hi + 16 * c, eh);
            tmem_st16(t_lo + 16 * c, el);
          }
        }
        if (wg == 0) {
          // S e: the residual into the A operand, then the signs
          tc_wait_st();
          tc_fence_before();
          mbar_arrive(&bar_a[0]);
          ok = mbar_wait(&bar_d[0], 1u, &s_abort);
          if (ok) {
            tc_fence_after();
            uint32_t sw[4] = {0u, 0u, 0u, 0u};
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32];
              tmem_ld32(t_d + 32 * c, r);
              tc_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int i = 32 * c + j;   // sketch row: lane tc = (i >> 1) & 3 of the quad, bit 2 kt + rho (+ 16)
                const uint32_t bit = 1u << (2 * (i >> 4) + ((i >> 3) & 1) + 16 * (i & 1));
                if (__uint_as_float(r[j]) >= 0.f) sw[(i >> 1) & 3] |= bit;
              }
            }
            const __half hn = __double2half(n);
            const __half hg = __double2half(n * sqrt((double)(es0 + es1) * (1.0 / 4096.0)));
            if (isinf(__half2float(hn)) || isinf(__half2float(hg))) flags |= KVQ_DEV_PARAM_OVERFLOW;
            if (dst != nullptr) {
              const int nt = tt >> 3, gr = tt & 7;
              uint32_t* sg = reinterpret_cast<uint32_t*>(dst + kTqSigns);
#pragma unroll
              for (int q = 0; q < 4; ++q) sg[4 * (4 * gr + q) + nt] = sw[q];
              reinterpret_cast<uint32_t*>(dst + kTqKMeta)[entry] =
                  (uint32_t)__half_as_ushort(hn) | ((uint32_t)__half_as_ushort(hg) << 16);
            }
          }
        } else {
          const __half hv = __double2half(n);
          if (isinf(__half2float(hv))) flags |= KVQ_DEV_PARAM_OVERFLOW;
          if (dst != nullptr) reinterpret_cast<uint16_t*>(dst + kTqVMeta)[entry] = __half_as_ushort(hv);
        }
      }
      if (!ok) s_abort = 1;
      // all 256 token threads agree on stopping before the code tiles are packed
      if (bar_red_or(1, 256, !ok)) {
        flags |= KVQ_DEV_WAIT_TIMEOUT;
        break;
      }

      // ---------------------------------------------------------- pack the tile's code words
      for (int item = tid; item < 4 * 2 * 416; item += 256) {
        const int tb = item / (2 * 416);
        const int qw = item - tb * (2 * 416);
        const int64_t tb_task = tile * 4 + tb;
        if (tb_task >= n_tasks) continue;
        const int trow = (int)(tb_task / a.n_groups);
        const int64_t tblk = tb_task - (int64_t)trow * a.n_groups;
        uint32_t* out = reinterpret_cast<uint32_t*>(record_ptr(gm, trow, a.dst_group0 + tblk));
        if (out == nullptr) {
          flags |= KVQ_DEV_BAD_PAGE;   // page outside the pool: nothing is written
          continue;
        }
        const int vblk = qw >= 416;
        const int q = qw - 416 * vblk;
        const int ln = q < 384 ? (q >> 2) & 31 : q - 384;
        const int w = q < 384 ? 4 * (q >> 7) + (q & 3) : 12;
        const int gr = ln >> 2, tc = ln & 3;
        const uint8_t* ct = (vblk ? sCV : sCK) + 32 * tb * kCodeRow;
        uint32_t word = 0;
#pragma unroll
        for (int f = 0; f < 5; ++f) {
          const int slot = 5 * w + f;
          if (slot < 64) {
            uint32_t idx;
            if (!vblk) {   // key pair (nt, kt, rho): token 8 nt + gr, coordinates 16 kt + 8 rho + 2 tc (+1)
              const int nt = slot >> 4, kt = (slot >> 1) & 7, rho = slot & 1;
              const uint8_t* cp = ct + (8 * nt + gr) * kCodeRow + 16 * kt + 8 * rho + 2 * tc;
              idx = cp[0] + 8u * cp[1];
            } else {       // value pair (kt, nt, rho): coordinate 8 nt + gr, tokens 16 kt + 8 rho + 2 tc (+1)
              const int kt = slot >> 5, nt = (slot >> 1) & 15, rho = slot & 1;
              const uint8_t* cp = ct + (16 * kt + 8 * rho + 2 * tc) * kCodeRow + 8 * nt + gr;
              idx = cp[0] + 8u * cp[kCodeRow];
            }
            word |= idx << (6 * f);
          }
        }
        out[(vblk ? kTqVCodes : kTqKCodes) / 4 + q] = word;
      }
      asm volatile("bar.sync 1, 256;\n" ::: "memory");   // the code tiles are free for the next tile
    }
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
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(tq_quantize_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSmem::BYTES);
    attr_set = true;
  }
  const int64_t tiles = (tasks + 3) / 4;
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  tq_quantize_tc_kernel<<<grid, kTcThreads, TcSmem::BYTES, st>>>(a);
  count_launch(1);
}

}  // namespace kvq

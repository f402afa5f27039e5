// FP8 E4M3 token rows of the mixed-format cache: recent and protected
// ("Anchor") pages stay in FP8 while older ones move to TQ3 ("KV-cache
// compresse et modeles 4-bit ...", section "Minima-KV : la compression sans
// eviction").  Per token vector (key or value of one kv head, d = 128):
// s = RNE_fp16(max |x| / 448), code_c = RNE_e4m3(x_c / s) with saturation to
// +-448 (which this scale never reaches) and a code rounding to zero stored as
// +0; the row is the 128 codes, s in fp16 and 14 zero bytes.  Both quotients
// are taken in fp32: for 16-bit x and fp16 s they never fall within fp32
// rounding of an fp16 or E4M3 midpoint without being on it, so rounding the
// fp32 quotient once decides exactly as the exact quotient would.
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kRowsPerBlock = 4;   // token rows per CTA (8 warps: one per row and K / V)

__global__ void __launch_bounds__(256) fp8_rows_kernel(Geom g, const uint16_t* k, const uint16_t* v, int64_t seq,
                                                       int64_t t0, int n, unsigned char* dst, int64_t row_stride,
                                                       int64_t kv_stride, int slot0) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kRowsPerBlock + (warp >> 1), kv = warp & 1;
  const int row = blockIdx.y;
  if (j >= n) return;
  const uint16_t* src = (kv ? v : k) + ((int64_t)row * seq + t0 + j) * kTqD;
  const uint2 raw = *reinterpret_cast<const uint2*>(src + 4 * lane);   // channels 4 lane .. 4 lane + 3
  const uint16_t h[4] = {(uint16_t)(raw.x & 0xFFFFu), (uint16_t)(raw.x >> 16), (uint16_t)(raw.y & 0xFFFFu),
                         (uint16_t)(raw.y >> 16)};
  float x[4], mx = 0.f;
  bool fin = true;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[e] = in16_to_float(h[e], g.dtype);
    fin &= isfinite(x[e]);
    mx = fmaxf(mx, fabsf(x[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  fin = __all_sync(0xffffffffu, fin);
  const __half hs = __float2half_rn(mx / 448.f);
  const float s = __half2float(hs);
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t c = 0;
    if (s > 0.f) c = (uint32_t)__nv_cvt_float_to_fp8(x[e] / s, __NV_SATFINITE, __NV_E4M3);
    if ((c & 0x7Fu) == 0) c = 0;   // zero is stored as +0
    word |= c << (8 * e);
  }
  unsigned char* out = dst + (int64_t)row * row_stride + kv * kv_stride + (int64_t)(slot0 + j) * kFp8RowBytes;
  reinterpret_cast<uint32_t*>(out)[lane] = word;
  if (lane == 0) {
    *reinterpret_cast<uint4*>(out + 128) = make_uint4((uint32_t)__half_as_ushort(hs), 0u, 0u, 0u);
    if (!fin) atomicOr(g.status, KVQ_DEV_NONFINITE_INPUT);
    if (isinf(s)) atomicOr(g.status, KVQ_DEV_PARAM_OVERFLOW);
  }
}

}  // namespace

void launch_fp8_rows(const Geom& g, const uint16_t* k, const uint16_t* v, int64_t seq, int64_t t0, int n,
                     unsigned char* dst, int64_t row_stride, int64_t kv_stride, int slot0, cudaStream_t st) {
  if (n <= 0) return;
  const dim3 grid((n + kRowsPerBlock - 1) / kRowsPerBlock, g.B * g.Hkv);
  fp8_rows_kernel<<<grid, 256, 0, st>>>(g, k, v, seq, t0, n, dst, row_stride, kv_stride, slot0);
  count_launch(1);
}

}  // namespace kvq

// Internal declarations shared by the libkvq CUDA sources (sm_100a only).
//
// Packed KIVI format v1 (one "group record" per G tokens of a (batch, kv head)
// row).  A token block (TB) is 32 tokens; lane L of a warp has gr = L >> 2 and
// tc = L & 3, the coordinates of the m16n8k16 mma.sync fragments.
//
//  key codes of a TB    pair (nt, kt, rho) of lane (gr, tc) = token 8nt+gr,
//                       channels 16kt+8rho+2tc (+0 low half, +1 high half);
//                       u = 2kt + rho
//                       2-bit: j'=u&3, slot=nt*(d/32)+(u>>2), word=slot>>1, j=4(slot&1)+j'
//                       4-bit: j'=u&1, slot=nt*(d/16)+(u>>1), word=slot>>1, j=2(slot&1)+j'
//  value codes of a TB  pair (kt, nt, rho) of lane (gr, tc) = channel 8nt+gr,
//                       tokens 16kt+8rho+2tc (+0 low, +1 high); u = 2kt + rho
//                       2-bit: j'=u,   slot=nt,          word=slot>>1, j=4(slot&1)+j'
//                       4-bit: j'=u&1, slot=2nt+(u>>1),  word=slot>>1, j=2(slot&1)+j'
//  low code of pair j at bit b*j, high code at bit 16+b*j; word w of lane L at
//  byte 16*(32*(w>>2)+L) + 4*(w&3) of the TB's code block.
//  key meta   d fp16 scales, then d fp16 zeros; channel 16kt+8rho+2tc+e at
//             position 8(4(kt>>1)+tc) + 4(kt&1) + 2rho + e (one 16-byte chunk
//             per (k-tile pair, tc), adjacent across tc).
//  value meta per TB, 32 x {fp16 scale, fp16 zero}; token 16kt+8rho+2tc+e at
//             entry 8tc+4kt+2rho+e.
//  record     [key TBs][value TBs][key scales][key zeros][value meta TBs]
//
// The format puts every pair a lane needs for one mma.sync B operand inside one
// 32-bit word at the bit positions (b*j, 16+b*j), so a single LOP3 turns two
// codes into the mantissas of an fp16x2 and one HFMA2 makes them exact small
// integers.  A warp reads a TB's codes as 16-byte pieces, one per lane.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kTB = 32;         // tokens per token block
constexpr int kFp8RowBytes = 144;   // FP8 token row: 128 E4M3 codes, fp16 scale, 14 zero bytes (d = 128)
constexpr int kMaxDecodeCtas = 160;   // decode launches use at most this many CTAs (one per SM)
constexpr int kDecodeWinTok = 32;     // window tokens per decode work item
constexpr int kKiviConsumersTM = 12;  // KIVI decode consumer warps, token-major formulation (GQA groups <= 4)
constexpr int kKiviConsumersHM = 12;  // KIVI decode consumer warps, hybrid formulation (GQA groups of 8)
constexpr int kTqDecodeConsumers = 11; // TurboQuant decode consumer warps
constexpr long long kWaitCyclesDefault = 2000000000ll;   // decode wait bound: about 1 s of SM cycles

struct Geom {
  int scheme, d, bits, G, R, cap, B, Hkv, Hq, g, dtype;
  int rot_wht;              // TURBO: Pi is the Walsh-Hadamard rotation H / sqrt(d)
  const int32_t* page_table;   // paged: [rows][pages_per_row] pool pages, else null
  int page_recs;               // paged: records per page (a power of two)
  int page_shift;              // paged: log2(page_recs)
  int num_pages;               // paged: pages in the pool
  int64_t pages_per_row;
  int fp8;                     // TURBO mixed cache: window (and anchors) in FP8 token rows
  int anchor;                  // fp8: anchor tokens A per row
  unsigned char* anchors;      // fp8: [rows][2][A][kFp8RowBytes]
  int64_t groups_per_row;   // record capacity of a row
  int64_t rec_bytes;        // bytes of one group record
  int64_t tb_code_bytes;    // bytes of one TB's key (or value) codes
  char* records;            // [B][Hkv][groups_per_row][rec_bytes]
  uint16_t* window;         // [B][Hkv][2][cap][d]
  uint32_t* status;         // device status word
  unsigned char* params;    // TURBO: deployment constants (kTq* offsets)
};

// ------------------------------------------------------------------ TurboQuant-style format (head_dim = m = 128)
// Token block (32 tokens of one row), kTqTbBytes bytes:
//   [key codes 1664][value codes 1664][key sign bits 512][key meta 128][value meta 64]
// Codes: the two 3-bit codes of a fragment pair form the 6-bit index lo + 8 hi;
// five indices fill a 32-bit word (bits 6f..6f+5).  Lane L owns 64 pairs per
// code block, slot s in word s / 5, field s % 5; words 0..11 of lane L sit at
// byte 16 (32 (w >> 2) + L) + 4 (w & 3) and word 12 at 1536 + 4 L, so word q of
// the block (in that order) is at byte 4 q.
//   key pair   (nt, kt, rho), slot 16 nt + 2 kt + rho: token 8 nt + gr,
//              coordinates 16 kt + 8 rho + 2 tc (lo) and + 1 (hi)
//   value pair (kt, nt, rho), slot 32 kt + 2 nt + rho: coordinate 8 nt + gr,
//              tokens 16 kt + 8 rho + 2 tc (lo) and + 1 (hi)
// Sign bits of the key sketch: pair (nt, kt, rho) of lane L (token 8 nt + gr,
// sketch rows 16 kt + 8 rho + 2 tc and + 1) in word nt of the lane's 16-byte
// piece at byte 16 L, bits 2 kt + rho (lo) and 16 + 2 kt + rho (hi).
// Meta: token 16 kt + 8 rho + 2 tc + e at entry 8 tc + 4 kt + 2 rho + e; keys
// as (fp16 norm, fp16 gamma) words, values as fp16 norms.
constexpr int kTqD = 128;
constexpr int kTqM = 128;
constexpr int kTqTbBytes = 4032;
constexpr int kTqKCodes = 0;
constexpr int kTqVCodes = 1664;
constexpr int kTqSigns = 3328;
constexpr int kTqKMeta = 3840;
constexpr int kTqVMeta = 3968;
// Parameter block (inside the cache buffer, written by kvq_turbo_setup):
constexpr int kTqPi = 0;                      // float [d][d], Pi[i][j] (y = Pi u)
constexpr int kTqPiT = kTqPi + kTqD * kTqD * 4;    // float [d][d], transpose of Pi
constexpr int kTqST = kTqPiT + kTqD * kTqD * 4;    // float [d][m], transpose of S
constexpr int kTqLevels = kTqST + kTqD * kTqM * 4; // float [8] codebook levels
constexpr int kTqThr = kTqLevels + 32;             // float [8] thresholds (7 used, [7] = +inf)
constexpr int kTqLevels16 = kTqThr + 32;           // fp16 [8] levels
constexpr int kTqLut = kTqLevels + 128;            // uint32 [64]: fp16x2 (level[lo], level[hi]) of index lo + 8 hi
constexpr int kTqSPiT = kTqLut + 256;              // float [d][m], transpose of S Pi (the sketch of a rotated query)
// Tensor-core operand images of the quantizer's products 16 Pi x and S e: two
// sets of four [128][128] matrices B[n][k] (16 Pi hi, 16 Pi lo, S hi, S lo; hi
// + lo approximates the fp32 value), the first in fp16 (for fp16 inputs), the
// second in bf16 (for bf16 inputs: an mma takes A and B of one type), each in
// the no-swizzle K-major layout of tcgen05.mma: the 8 x 8 core matrix
// (n / 8, k / 8) at byte 2048 (k / 8) + 128 (n / 8), row n % 8 at 16-byte steps.
constexpr int kTqBImg = kTqSPiT + kTqD * kTqM * 4;
constexpr int kTqBImgBytes = 32768;                // one image
constexpr int kTqBImgSet = 4 * kTqBImgBytes;       // one set; the bf16 set follows the fp16 one
constexpr int kTqParamBytes = kTqBImg + 2 * kTqBImgSet;
constexpr int kTqQPrepBytes = 2 * (kTqD / 16) * 32 * 16;   // rotated query fragments of one row

__host__ __device__ inline int64_t rec_kscale_off(const Geom& g) { return (int64_t)g.G * g.d * g.bits / 4; }
__host__ __device__ inline int64_t rec_kzero_off(const Geom& g) { return rec_kscale_off(g) + 2 * g.d; }
__host__ __device__ inline int64_t rec_vmeta_off(const Geom& g) { return rec_kscale_off(g) + 4 * g.d; }

// Address of record `group` of `row`.  Paged caches look the page up in the
// block table; a page outside the pool gives null (the caller skips the access
// and reports KVQ_DEV_BAD_PAGE).
__device__ inline char* record_ptr(const Geom& g, int row, int64_t group) {
  if (g.page_table == nullptr) return g.records + ((int64_t)row * g.groups_per_row + group) * g.rec_bytes;
  const int64_t p = group >> g.page_shift;
  const int32_t page = __ldg(g.page_table + (int64_t)row * g.pages_per_row + p);
  if (page < 0 || page >= g.num_pages) return nullptr;
  return g.records + (((int64_t)page << g.page_shift) + (group & (g.page_recs - 1))) * g.rec_bytes;
}
__host__ __device__ inline uint16_t* ring_ptr(const Geom& g, int row, int kv) {
  return g.window + ((int64_t)row * 2 + kv) * g.cap * g.d;
}

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ void mma_f16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// 16-bit input pattern -> float (exact).
__device__ __forceinline__ float in16_to_float(uint16_t bits, int dtype) {
  if (dtype == KVQ_BF16) return __uint_as_float((uint32_t)bits << 16);
  return __half2float(__ushort_as_half(bits));
}

// Exact code decision: q = clamp(round_half_even((x - z) / s), 0, levels), by
// comparing t = 2(x - z), carried as an error-free double sum hi + lo, with the
// exact thresholds (2k + 1) s.  A double-precision estimate is corrected by
// exact comparisons (at most a couple of steps each way).
__device__ __forceinline__ bool t_above(double hi, double lo, double T) {
  return hi > T || (hi == T && lo > 0.0);
}
__device__ __forceinline__ int exact_code(double x, double z, double s, double inv_s, int levels) {
  if (!(s > 0.0)) return 0;
  double hi = x - z;
  double bb = hi - x;
  double lo = (x - (hi - bb)) + (-z - bb);
  hi *= 2.0;
  lo *= 2.0;
  double est = ceil((hi * inv_s - 1.0) * 0.5);
  int k = est < 0.0 ? 0 : (est > (double)levels ? levels : (int)est);
  // k must count the thresholds strictly below t
  for (int it = 0; it < 4 && k > 0 && !t_above(hi, lo, (2.0 * k - 1.0) * s); ++it) --k;
  for (int it = 0; it < 4 && k < levels && t_above(hi, lo, (2.0 * k + 1.0) * s); ++it) ++k;
  if (k < levels && hi == (2.0 * k + 1.0) * s && lo == 0.0 && (k & 1)) ++k;
  return k;
}

// Unpack one 32-bit code word into exact fp16x2 values.
// 2-bit: 8 pairs, pair j at bits (2j, 16+2j); 4-bit: 4 pairs at (4j, 16+4j);
// the upper four (two) pairs are read after shifting the word down by 8, so a
// pair sits at position j' (0..3 for 2-bit, 0..1 for 4-bit) of its half word.
// (w & field) | 0x6400 is the fp16 1024 + code * 2^(b*j'); subtracting 1024
// leaves code * 2^(b*j'), an exact normal fp16 (at most 3*64 or 15*16).  The
// factor 2^(b*j') is undone on the other mma operand, where it is an exact
// power-of-two rescale (pos_comp).
constexpr uint32_t kMagic = 0x64006400u;   // fp16x2 (1024, 1024)

template <int BITS, int JP>
__device__ __forceinline__ uint32_t unpack_pair(uint32_t x, uint32_t magic) {
  constexpr uint32_t M = (BITS == 2 ? 0x00030003u : 0x000F000Fu) << (BITS * JP);
  uint32_t f, d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(f) : "r"(x), "n"(M), "r"(magic));   // (x & M) | magic
  asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(f), "r"(magic));
  return d;
}
// One half word (already shifted down for the upper half): J pairs.
template <int BITS>
__device__ __forceinline__ void unpack_half(uint32_t x, uint32_t* out, uint32_t magic) {
  out[0] = unpack_pair<BITS, 0>(x, magic);
  out[1] = unpack_pair<BITS, 1>(x, magic);
  if (BITS == 2) {
    out[2] = unpack_pair<BITS, 2>(x, magic);
    out[3] = unpack_pair<BITS, 3>(x, magic);
  }
}
template <int BITS>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t* out, uint32_t magic) {
  constexpr int J = BITS == 2 ? 4 : 2;
  unpack_half<BITS>(w, out, magic);
  unpack_half<BITS>(w >> 8, out + J, magic);
}
// 2^(-b*j'): the compensation of pair position j', as fp16x2 and as float
__host__ __device__ constexpr uint32_t pos_comp(int bits, int jp) {
  return bits == 2 ? (jp == 0 ? 0x3C003C00u : jp == 1 ? 0x34003400u : jp == 2 ? 0x2C002C00u : 0x24002400u)
                   : (jp == 0 ? 0x3C003C00u : 0x2C002C00u);
}
__host__ __device__ constexpr float pos_comp_f(int bits, int jp) {
  return bits == 2 ? (jp == 0 ? 1.f : jp == 1 ? 0.25f : jp == 2 ? 0.0625f : 0.015625f) : (jp == 0 ? 1.f : 0.0625f);
}

// 2^x with the MUFU instruction (inputs are <= 0 here; ftz is harmless)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ kernels (launchers in kvq_api.cu)
struct QuantArgs {
  Geom geom;
  const uint16_t* src_k;   // token 0 of group `src_group0` of row 0
  const uint16_t* src_v;
  int64_t src_row_stride;  // elements between rows
  const unsigned char* src_fp8;   // TURBO mixed flush: FP8 window rows of the first token (ring layout), or null
  int64_t dst_group0;      // first record index written
  int n_groups;            // groups per row handled by this launch
  long long wait_cycles;   // bound of the tensor-core quantizer's waits (SM cycles)
  int withhold_first_stage;   // test hook: CTA 0 of the tensor-core quantizer skips its operand-image copy
};

struct AttnArgs {
  Geom geom;
  const unsigned char* qprep;   // TURBO: [rows][kTqQPrepBytes] query fragments
  float qjl_c;                  // TURBO: sqrt(pi / 2) / m
  const uint16_t* q;       // [B][Hq][d]
  float* out;              // [B][Hq][d]
  float* ws;               // partials [n_cta + rows][g][d + 2] (o[d], m, l)
  unsigned* counters;      // [rows] arrival counters, zero between launches
  float scale_log2;        // softmax scale * log2(e)
  int64_t n_groups;        // quantized groups per row (T_q / G)
  int n_cta;               // CTAs of the launch (one per SM at most)
  int r;                   // window tokens
  int head;                // ring slot of the oldest window token
  // Fused append (or null): window token r - 1 is the new token of each row,
  // read from k_new / v_new ([B][Hkv][d]) instead of the ring, and the CTA
  // that attends it also stores it into ring slot (head + r - 1) % cap.
  const uint16_t* k_new;
  const uint16_t* v_new;
  // Work partition, computed on the host: CTA c owns the global items
  // item0[c] .. item0[c + 1] - 1 (strictly increasing), where a row's items
  // are its n_groups quantized items, then its window-type chunks.
  int32_t n_items;                        // items per row
  // Bound of the kernel's waits in SM cycles (kWaitCycles unless a test set a
  // shorter one) and, for tests of the timeout path, whether CTA 0 withholds
  // the copy of its first stage (a wait that nothing completes).
  long long wait_cycles;
  int withhold_first_stage;
  int32_t item0[kMaxDecodeCtas + 1];
};

void launch_kivi_quantize(const QuantArgs& a, cudaStream_t st);
void launch_window_copy(const Geom& g, const uint16_t* k, const uint16_t* v, int64_t seq_len, int64_t t0,
                        int n, cudaStream_t st);
// FP8 token rows of tokens t0 .. t0 + n - 1 of every row of a [rows][seq][d]
// 16-bit input: row r's token j goes to dst + r * row_stride + kv * kv_stride +
// (slot0 + j) * kFp8RowBytes.
void launch_fp8_rows(const Geom& g, const uint16_t* k, const uint16_t* v, int64_t seq, int64_t t0, int n,
                     unsigned char* dst, int64_t row_stride, int64_t kv_stride, int slot0, cudaStream_t st);
void launch_append(const Geom& g, const uint16_t* k, const uint16_t* v, int slot, cudaStream_t st);
void launch_kivi_attention(const AttnArgs& a, cudaStream_t st);
void launch_clear_words(uint32_t* words, int n, cudaStream_t st);
void launch_turbo_setup(const Geom& g, const float* rot_gauss, const float* qjl_gauss, bool wht, cudaStream_t st);
void launch_tq_quantize(const QuantArgs& a, cudaStream_t st);
// the tensor-core quantizer (16-bit sources, either rotation); launch_tq_quantize routes to it
void launch_tq_quantize_tc(const QuantArgs& a, cudaStream_t st);
void launch_tq_query_prep(const Geom& g, const uint16_t* q, unsigned char* qprep, cudaStream_t st);
void launch_tq_attention(const AttnArgs& a, cudaStream_t st);
size_t cache_workspace_bytes(const kvq_cache* cache);   // kvq_workspace_bytes of the cache's config

int num_sms();
void count_launch(int n = 1);

}  // namespace kvq

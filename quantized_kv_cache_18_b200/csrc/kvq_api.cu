// Host side of the C ABI declared in include/kvq.h: argument validation, the
// cache-buffer layout, host-side length counters, split planning and launches.
// No call here allocates device memory; every computation runs in the kernels.
#include <cuda_runtime.h>

#include <atomic>
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>

#include "kvq_internal.cuh"

struct kvq_cache {
  kvq_config cfg;
  kvq_layout lay;
  char* base;
  int32_t seq_len;
  int32_t tq;
  int32_t r;
  int32_t head;
  bool tq_ready;   // TURBO: the parameter block holds the deployment constants
  bool tq_wht;     // TURBO: the rotation is the Walsh-Hadamard one
  const int32_t* page_table;   // paged: [rows][pages_per_row] pool pages (device, caller-owned)
};

namespace kvq {

static std::atomic<uint64_t> g_launches{0};
static thread_local const char* g_cuda_error = "no error";
// Test hook of the decode kernels' bounded waits (kvq_debug_set_wait_test).
static std::atomic<long long> g_wait_cycles{0};   // 0: the default bound
static std::atomic<int> g_withhold{0};
// the hook's values for a quantizer launch
static void quant_wait_args(QuantArgs& a) {
  const long long wc = g_wait_cycles.load(std::memory_order_relaxed);
  a.wait_cycles = wc > 0 ? wc : kWaitCyclesDefault;
  a.withhold_first_stage = g_withhold.load(std::memory_order_relaxed);
}

// Records the failing CUDA call's message for kvq_cuda_error_string.
static kvq_status cuda_failed(cudaError_t e) {
  g_cuda_error = cudaGetErrorString(e);
  return KVQ_ERR_CUDA;
}
// Checks the launches just enqueued (launch-configuration errors surface here).
static kvq_status check_launch() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVQ_OK : cuda_failed(e);
}
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

static uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

static bool config_ok(const kvq_config* c) {
  if (!c) return false;
  if (c->scheme == KVQ_KIVI) {
    if (!(c->bits == 2 || c->bits == 4)) return false;
    if (!(c->group == 32 || c->group == 64)) return false;
    if (!(c->head_dim == 64 || c->head_dim == 128)) return false;
  } else if (c->scheme == KVQ_TURBO) {
    if (c->bits != 3 || c->group != kTB || c->head_dim != kTqD || c->qjl_dim != kTqM) return false;
  } else {
    return false;
  }
  if (c->residual < 0 || c->residual % c->group != 0) return false;
  if (c->num_kv_heads <= 0 || c->num_q_heads <= 0 || c->num_q_heads % c->num_kv_heads != 0) return false;
  const int g = c->num_q_heads / c->num_kv_heads;
  if (!(g == 1 || g == 2 || g == 4 || g == 8)) return false;
  if (c->batch <= 0 || c->max_seq <= 0) return false;
  if ((int64_t)c->batch * c->num_kv_heads > 65535) return false;
  if (!(c->dtype == KVQ_BF16 || c->dtype == KVQ_FP16)) return false;
  if (c->page_records < 0 || c->num_pages < 0) return false;
  if ((c->page_records == 0) != (c->num_pages == 0)) return false;   // both set or both zero
  if (c->page_records & (c->page_records - 1)) return false;          // a power of two
  if (!(c->fp8_recent == 0 || c->fp8_recent == 1)) return false;
  if (c->fp8_recent && c->scheme != KVQ_TURBO) return false;          // the mixed cache is TQ3 + FP8
  if (c->anchor_tokens < 0 || c->anchor_tokens % 32 != 0) return false;
  if (c->anchor_tokens > 0 && !c->fp8_recent) return false;
  return true;
}

static kvq_layout make_layout(const kvq_config* c) {
  kvq_layout L;
  std::memset(&L, 0, sizeof(L));
  const uint64_t rows = (uint64_t)c->batch * c->num_kv_heads;
  const uint64_t d = c->head_dim, G = c->group;
  L.record_bytes = c->scheme == KVQ_TURBO ? (uint64_t)kTqTbBytes : G * d * c->bits / 4 + 4 * d + 4 * G;
  const int64_t q_room = (int64_t)c->max_seq - c->residual - c->anchor_tokens;   // tokens that can be quantized
  L.groups_per_row = q_room > 0 ? (uint64_t)q_room / G : 0;
  L.ring_tokens = (uint64_t)c->residual + G;
  L.token_row_bytes = c->fp8_recent ? (uint64_t)kFp8RowBytes : 2 * d;
  L.records_offset = 0;
  const uint64_t n_records = c->page_records > 0 ? (uint64_t)c->num_pages * c->page_records : rows * L.groups_per_row;
  L.pages_per_row = c->page_records > 0 ? (L.groups_per_row + c->page_records - 1) / c->page_records : 0;
  uint64_t off = align_up(n_records * L.record_bytes, 256);
  L.window_offset = off;
  off = align_up(off + rows * 2 * L.ring_tokens * L.token_row_bytes, 256);
  L.anchor_offset = off;
  off = align_up(off + rows * 2 * (uint64_t)c->anchor_tokens * L.token_row_bytes, 256);
  L.params_offset = off;
  L.params_bytes = c->scheme == KVQ_TURBO ? (uint64_t)kTqParamBytes : 0;
  off = align_up(off + L.params_bytes, 256);
  L.status_offset = off;               // status word, then one counter per row
  L.total_bytes = align_up(off + 4 + 4 * rows, 256);
  return L;
}

static Geom make_geom(const kvq_cache* h) {
  Geom g;
  const kvq_config& c = h->cfg;
  g.scheme = c.scheme;
  g.rot_wht = h->tq_wht ? 1 : 0;
  g.page_table = c.page_records > 0 ? h->page_table : nullptr;
  g.page_recs = c.page_records;
  g.page_shift = 0;
  while (c.page_records > 0 && (1 << g.page_shift) < c.page_records) ++g.page_shift;
  g.pages_per_row = (int64_t)h->lay.pages_per_row;
  g.num_pages = c.num_pages;
  g.fp8 = c.fp8_recent;
  g.anchor = c.anchor_tokens;
  g.anchors = reinterpret_cast<unsigned char*>(h->base + h->lay.anchor_offset);
  g.d = c.head_dim;
  g.bits = c.bits;
  g.G = c.group;
  g.R = c.residual;
  g.cap = c.residual + c.group;
  g.B = c.batch;
  g.Hkv = c.num_kv_heads;
  g.Hq = c.num_q_heads;
  g.g = c.num_q_heads / c.num_kv_heads;
  g.dtype = c.dtype;
  g.groups_per_row = (int64_t)h->lay.groups_per_row;
  g.rec_bytes = (int64_t)h->lay.record_bytes;
  g.tb_code_bytes = c.scheme == KVQ_TURBO ? (int64_t)(kTqVCodes - kTqKCodes) : (int64_t)kTB * c.head_dim * c.bits / 8;
  g.records = h->base + h->lay.records_offset;
  g.window = reinterpret_cast<uint16_t*>(h->base + h->lay.window_offset);
  g.status = reinterpret_cast<uint32_t*>(h->base + h->lay.status_offset);
  g.params = reinterpret_cast<unsigned char*>(h->base + h->lay.params_offset);
  return g;
}

// The decode work partition.  A row's items are n_q quantized items (KIVI
// groups, TurboQuant token blocks) and then n_w window-type chunks of 32
// tokens.  The kernels take a CTA's quantized items `sg` at a time from the
// start of its range, one stage per `sg` items, and one stage per window
// chunk; a stage takes about the same time whatever its bytes, since the
// consumer warps' instruction stream, not HBM, sets the pace.  So the
// partition balances stages, not bytes: a row is a sequence of ceil(n_q / sg)
// stage chunks of weight ws (each starting at a multiple of sg) and n_w window
// chunks of weight ww, and CTA c takes the chunks whose start weight lies in
// [c U / n, (c + 1) U / n), U the total weight.  Fills item0[0 .. n] (the
// first item of each CTA, then the end); false when a CTA would own no chunk.
static bool partition_items(int64_t rows, int64_t n_q, int sg, int64_t n_w, int64_t ws, int64_t ww, int n,
                            int32_t* item0) {
  const int64_t n_items = n_q + n_w, S = (n_q + sg - 1) / sg;
  const int64_t U_row = S * ws + n_w * ww, U = rows * U_row;
  for (int c = 0; c <= n; ++c) {
    const int64_t x = (int64_t)c * U / n;
    const int64_t row = x / U_row;
    int64_t it;
    if (row >= rows) {
      it = rows * n_items;
    } else {
      const int64_t off = x - row * U_row;
      const int64_t k = off <= S * ws ? (off + ws - 1) / ws : S + (off - S * ws + ww - 1) / ww;   // first chunk
      it = row * n_items + (k < S ? k * sg : n_q + (k - S));   // k == S + n_w is the next row's item 0
    }
    item0[c] = (int32_t)it;
    if (c > 0 && item0[c] <= item0[c - 1]) return false;
  }
  return true;
}

// Quantized items one decode stage carries (the kernels' consumer warps take
// one 32-token block each).
static int decode_stage_items(const kvq_config& c) {
  if (c.scheme == KVQ_TURBO) return kTqDecodeConsumers;
  const int g = c.num_q_heads / c.num_kv_heads;
  return (g <= 4 ? kKiviConsumersTM : kKiviConsumersHM) / (c.group / kTB);
}

// Decode launch size and partition: one CTA per SM at most (kMaxDecodeCtas),
// and few enough that every CTA owns at least one chunk, so each CTA between a
// row's first and last contributor has work in that row.  Returns the CTA
// count (0 when the item indices would not fit in 32 bits).
static int plan_decode(const kvq_config& c, int64_t n_groups, int r, int sms_avail, int32_t* n_items,
                       int32_t* item0) {
  // weights of a stage of quantized items and of a window chunk: a window
  // chunk's stage takes about 1.5 times a full stage of groups (measured)
  constexpr int64_t kWs = 2, kWw = 3;
  const int64_t rows = (int64_t)c.batch * c.num_kv_heads;
  const int A = c.scheme == KVQ_TURBO ? c.anchor_tokens : 0;
  const int64_t n_w = (r + kDecodeWinTok - 1) / kDecodeWinTok + A / kDecodeWinTok;
  const int sg = decode_stage_items(c);
  // nothing to attend (an empty cache): no launch, and no partition to divide by
  if (rows * (n_groups + n_w) == 0) return 0;
  if (rows * (n_groups + n_w) >= ((int64_t)1 << 31)) return 0;
  *n_items = (int32_t)(n_groups + n_w);
  const int64_t U = rows * (((n_groups + sg - 1) / sg) * kWs + n_w * kWw);
  const int64_t sms = sms_avail < kMaxDecodeCtas ? sms_avail : kMaxDecodeCtas;
  int n = (int)std::max<int64_t>(1, std::min<int64_t>(sms, U / kWw));
  while (n > 1 && !partition_items(rows, n_groups, sg, n_w, kWs, kWw, n, item0)) --n;
  if (n == 1) partition_items(rows, n_groups, sg, n_w, kWs, kWw, 1, item0);
  return n;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace kvq

size_t kvq::cache_workspace_bytes(const kvq_cache* h) { return h ? kvq_workspace_bytes(&h->cfg) : 0; }

using namespace kvq;

extern "C" {

size_t kvq_cache_bytes(const kvq_config* cfg) {
  if (!config_ok(cfg)) return 0;
  return (size_t)make_layout(cfg).total_bytes;
}

// KIVI: partial states, (rows + SMs) slots of g x (d + 2) floats.  TURBO: the
// rotated query fragments of every row, then (2 rows + SMs) partial slots (a
// row's token blocks and window chunks give separate partials).
static size_t tq_qprep_bytes(const kvq_config* cfg) {
  return (size_t)cfg->batch * cfg->num_kv_heads * kTqQPrepBytes;
}
size_t kvq_workspace_bytes(const kvq_config* cfg) {
  if (!config_ok(cfg)) return 0;
  const int64_t rows = (int64_t)cfg->batch * cfg->num_kv_heads;
  const int g = cfg->num_q_heads / cfg->num_kv_heads;
  if (cfg->scheme == KVQ_TURBO)
    return tq_qprep_bytes(cfg) + (size_t)((2 * rows + num_sms()) * g * (cfg->head_dim + 2) * sizeof(float));
  // KIVI partial rows are (o[d], m, l) padded to d + 4 floats for 16-byte loads
  return (size_t)((rows + num_sms()) * g * (cfg->head_dim + 4) * sizeof(float));
}

kvq_status kvq_get_layout(const kvq_config* cfg, kvq_layout* out) {
  if (!out) return KVQ_ERR_INVALID_ARG;
  if (!config_ok(cfg)) return KVQ_ERR_UNSUPPORTED;
  *out = make_layout(cfg);
  return KVQ_OK;
}

kvq_status kvq_cache_init(const kvq_config* cfg, void* dev_buf, size_t bytes, void* stream, kvq_cache** out) {
  if (!cfg || !dev_buf || !out) return KVQ_ERR_INVALID_ARG;
  if (!config_ok(cfg)) return KVQ_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(dev_buf) & 255u) != 0) return KVQ_ERR_INVALID_ARG;
  const kvq_layout L = make_layout(cfg);
  if (bytes < L.total_bytes) return KVQ_ERR_INVALID_ARG;
  kvq_cache* h = new (std::nothrow) kvq_cache;
  if (!h) return KVQ_ERR_INVALID_ARG;
  h->cfg = *cfg;
  h->lay = L;
  h->base = static_cast<char*>(dev_buf);
  h->seq_len = h->tq = h->r = h->head = 0;
  h->tq_ready = false;
  h->tq_wht = false;
  h->page_table = nullptr;
  launch_clear_words(reinterpret_cast<uint32_t*>(h->base + L.status_offset),
                     1 + cfg->batch * cfg->num_kv_heads, (cudaStream_t)stream);
  if (check_launch() != KVQ_OK) {
    delete h;
    return KVQ_ERR_CUDA;
  }
  *out = h;
  return KVQ_OK;
}

kvq_status kvq_cache_set_page_table(kvq_cache* h, const int32_t* table) {
  if (!h) return KVQ_ERR_INVALID_ARG;
  if (h->cfg.page_records == 0) return KVQ_ERR_UNSUPPORTED;
  if (!table || !aligned16(table)) return KVQ_ERR_INVALID_ARG;
  h->page_table = table;
  return KVQ_OK;
}

// A paged cache needs its block table before any call that touches records.
static bool records_ready(const kvq_cache* h) { return h->cfg.page_records == 0 || h->page_table != nullptr; }

kvq_status kvq_turbo_setup(kvq_cache* h, const float* rot_gauss, const float* qjl_gauss, void* stream) {
  if (!h || !rot_gauss || !qjl_gauss) return KVQ_ERR_INVALID_ARG;
  if (h->cfg.scheme != KVQ_TURBO) return KVQ_ERR_UNSUPPORTED;
  if (!aligned16(rot_gauss) || !aligned16(qjl_gauss)) return KVQ_ERR_INVALID_ARG;
  if (h->seq_len != 0) return KVQ_ERR_INVALID_ARG;
  h->tq_wht = false;
  launch_turbo_setup(make_geom(h), rot_gauss, qjl_gauss, false, (cudaStream_t)stream);
  if (check_launch() != KVQ_OK) return KVQ_ERR_CUDA;
  h->tq_ready = true;
  return KVQ_OK;
}

kvq_status kvq_turbo_setup_wht(kvq_cache* h, const float* qjl_gauss, void* stream) {
  if (!h || !qjl_gauss) return KVQ_ERR_INVALID_ARG;
  if (h->cfg.scheme != KVQ_TURBO) return KVQ_ERR_UNSUPPORTED;
  if (!aligned16(qjl_gauss)) return KVQ_ERR_INVALID_ARG;
  if (h->seq_len != 0) return KVQ_ERR_INVALID_ARG;
  h->tq_wht = true;
  launch_turbo_setup(make_geom(h), nullptr, qjl_gauss, true, (cudaStream_t)stream);
  if (check_launch() != KVQ_OK) return KVQ_ERR_CUDA;
  h->tq_ready = true;
  return KVQ_OK;
}

kvq_status kvq_quantize_prefill(kvq_cache* h, const void* k, const void* v, int32_t seq_len, void* stream) {
  if (!h || !k || !v || seq_len < 0) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return KVQ_ERR_INVALID_ARG;
  if (h->seq_len != 0) return KVQ_ERR_INVALID_ARG;
  if (h->cfg.scheme == KVQ_TURBO && !h->tq_ready) return KVQ_ERR_INVALID_ARG;
  if (!records_ready(h)) return KVQ_ERR_INVALID_ARG;
  if (seq_len > h->cfg.max_seq) return KVQ_ERR_CAPACITY;
  const kvq_config& c = h->cfg;
  const int32_t G = c.group, R = c.residual, A = c.anchor_tokens;
  if (seq_len < A) return KVQ_ERR_INVALID_ARG;   // the anchors come with the prefill
  const int32_t rest = seq_len - A;               // tokens after the anchors
  const int32_t tq = rest > R ? G * ((rest - R) / G) : 0;
  const Geom g = make_geom(h);
  cudaStream_t st = (cudaStream_t)stream;
  QuantArgs a;
  a.geom = g;
  a.src_k = static_cast<const uint16_t*>(k) + (int64_t)A * c.head_dim;
  a.src_v = static_cast<const uint16_t*>(v) + (int64_t)A * c.head_dim;
  a.src_row_stride = (int64_t)seq_len * c.head_dim;
  a.src_fp8 = nullptr;
  a.dst_group0 = 0;
  a.n_groups = tq / G;
  quant_wait_args(a);
  if (c.scheme == KVQ_TURBO) launch_tq_quantize(a, st);
  else launch_kivi_quantize(a, st);
  if (c.fp8_recent) {
    const uint16_t* k16 = static_cast<const uint16_t*>(k);
    const uint16_t* v16 = static_cast<const uint16_t*>(v);
    const int64_t ring_row = (int64_t)2 * g.cap * kFp8RowBytes, anc_row = (int64_t)2 * A * kFp8RowBytes;
    launch_fp8_rows(g, k16, v16, seq_len, 0, A, g.anchors, anc_row, (int64_t)A * kFp8RowBytes, 0, st);
    launch_fp8_rows(g, k16, v16, seq_len, A + tq, rest - tq, reinterpret_cast<unsigned char*>(g.window), ring_row,
                    (int64_t)g.cap * kFp8RowBytes, 0, st);
  } else {
    launch_window_copy(g, a.src_k, a.src_v, seq_len, tq, seq_len - tq, st);
  }
  if (check_launch() != KVQ_OK) return KVQ_ERR_CUDA;
  h->seq_len = seq_len;
  h->tq = tq;
  h->r = rest - tq;
  h->head = 0;
  return KVQ_OK;
}

kvq_status kvq_append_token(kvq_cache* h, const void* k_new, const void* v_new, void* stream) {
  if (!h || !k_new || !v_new) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return KVQ_ERR_INVALID_ARG;
  if (h->seq_len + 1 > h->cfg.max_seq) return KVQ_ERR_CAPACITY;
  if (h->cfg.scheme == KVQ_TURBO && !h->tq_ready) return KVQ_ERR_INVALID_ARG;
  if (!records_ready(h)) return KVQ_ERR_INVALID_ARG;
  const kvq_config& c = h->cfg;
  const int32_t G = c.group, R = c.residual, cap = R + G;
  const Geom g = make_geom(h);
  cudaStream_t st = (cudaStream_t)stream;
  const int slot = (h->head + h->r) % cap;
  int32_t r = h->r + 1, head = h->head, tq = h->tq;
  if (r == R + G && (uint64_t)(tq / G) >= h->lay.groups_per_row) return KVQ_ERR_CAPACITY;
  if (c.fp8_recent)
    launch_fp8_rows(g, static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new), 1, 0, 1,
                    reinterpret_cast<unsigned char*>(g.window), (int64_t)2 * cap * kFp8RowBytes,
                    (int64_t)cap * kFp8RowBytes, slot, st);
  else
    launch_append(g, static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new), slot, st);
  if (r == R + G) {
    QuantArgs a;
    a.geom = g;
    a.src_k = g.window + (int64_t)head * c.head_dim;
    a.src_v = g.window + ((int64_t)cap + head) * c.head_dim;
    a.src_row_stride = (int64_t)2 * cap * c.head_dim;
    // mixed cache: the flushed tokens are the window's FP8 rows
    a.src_fp8 = c.fp8_recent ? reinterpret_cast<const unsigned char*>(g.window) + (int64_t)head * kFp8RowBytes
                             : nullptr;
    a.dst_group0 = tq / G;
    a.n_groups = 1;
    quant_wait_args(a);
    if (c.scheme == KVQ_TURBO) launch_tq_quantize(a, st);
    else launch_kivi_quantize(a, st);
    head = (head + G) % cap;
    r -= G;
    tq += G;
  }
  if (check_launch() != KVQ_OK) return KVQ_ERR_CUDA;
  h->r = r;
  h->head = head;
  h->tq = tq;
  h->seq_len += 1;
  return KVQ_OK;
}

// Argument checks of a decode attention call (also those of the fused call).
static kvq_status check_attention_args(const kvq_cache* h, const void* q, const float* out, float softmax_scale,
                                       const void* workspace, size_t workspace_bytes) {
  if (!h || !q || !out || !workspace) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return KVQ_ERR_INVALID_ARG;
  if (!(std::isfinite(softmax_scale))) return KVQ_ERR_INVALID_ARG;
  if (workspace_bytes < kvq_workspace_bytes(&h->cfg)) return KVQ_ERR_INVALID_ARG;
  if (h->cfg.scheme == KVQ_TURBO && !h->tq_ready) return KVQ_ERR_INVALID_ARG;
  if (!records_ready(h)) return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

// Launches the attention over the cache state (T_q = h->tq, window of r tokens
// from h->head); with k_new / v_new the window's last token is the new one.
static kvq_status launch_attention(const kvq_cache* h, int r, const void* q, float* out, float softmax_scale,
                                   void* workspace, cudaStream_t st, const void* k_new, const void* v_new) {
  const kvq_config& c = h->cfg;
  AttnArgs a;
  a.geom = make_geom(h);
  a.q = static_cast<const uint16_t*>(q);
  a.out = out;
  a.ws = static_cast<float*>(workspace);
  a.qprep = nullptr;
  a.qjl_c = 0.f;
  if (c.scheme == KVQ_TURBO) {
    unsigned char* qp = static_cast<unsigned char*>(workspace);
    a.qprep = qp;
    a.ws = reinterpret_cast<float*>(qp + tq_qprep_bytes(&c));
    a.qjl_c = (float)(std::sqrt(3.14159265358979323846 / 2.0) / c.qjl_dim);
  }
  a.counters = reinterpret_cast<unsigned*>(h->base + h->lay.status_offset) + 1;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.n_groups = h->tq / c.group;
  a.n_cta = plan_decode(c, a.n_groups, r, num_sms(), &a.n_items, a.item0);
  if (a.n_cta <= 0) return KVQ_ERR_UNSUPPORTED;
  a.r = r;
  a.head = h->head;
  const long long wc = g_wait_cycles.load(std::memory_order_relaxed);
  a.wait_cycles = wc > 0 ? wc : kWaitCyclesDefault;
  a.withhold_first_stage = g_withhold.load(std::memory_order_relaxed);
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  if (c.scheme == KVQ_TURBO) {
    launch_tq_query_prep(a.geom, a.q, const_cast<unsigned char*>(a.qprep), st);
    launch_tq_attention(a, st);
  } else {
    launch_kivi_attention(a, st);
  }
  if (check_launch() != KVQ_OK) return KVQ_ERR_CUDA;
  return KVQ_OK;
}

kvq_status kvq_decode_attention(const kvq_cache* h, const void* q, float* out, float softmax_scale, void* workspace,
                                size_t workspace_bytes, void* stream) {
  const kvq_status e = check_attention_args(h, q, out, softmax_scale, workspace, workspace_bytes);
  if (e != KVQ_OK) return e;
  if (h->seq_len <= 0) return KVQ_ERR_INVALID_ARG;
  return launch_attention(h, h->r, q, out, softmax_scale, workspace, (cudaStream_t)stream, nullptr, nullptr);
}

kvq_status kvq_append_decode(kvq_cache* h, const void* k_new, const void* v_new, const void* q, float* out,
                             float softmax_scale, void* workspace, size_t workspace_bytes, void* stream) {
  const kvq_status e = check_attention_args(h, q, out, softmax_scale, workspace, workspace_bytes);
  if (e != KVQ_OK) return e;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return KVQ_ERR_INVALID_ARG;
  if (h->seq_len + 1 > h->cfg.max_seq) return KVQ_ERR_CAPACITY;
  const int32_t r_new = h->r + 1;
  if (r_new == h->cfg.residual + h->cfg.group || h->cfg.fp8_recent) {
    // a flush is due, or the window holds FP8 rows (the new token is converted
    // by kvq_append_token): append, then attend
    const kvq_status ea = kvq_append_token(h, k_new, v_new, stream);
    if (ea != KVQ_OK) return ea;
    return launch_attention(h, h->r, q, out, softmax_scale, workspace, (cudaStream_t)stream, nullptr, nullptr);
  }
  const kvq_status el = launch_attention(h, r_new, q, out, softmax_scale, workspace, (cudaStream_t)stream, k_new, v_new);
  if (el != KVQ_OK) return el;
  h->r = r_new;
  h->seq_len += 1;
  return KVQ_OK;
}

kvq_status kvq_get_status(kvq_cache* h, uint32_t* bits, int32_t clear, void* stream) {
  if (!h) return KVQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t v = 0;
  uint32_t* dev = reinterpret_cast<uint32_t*>(h->base + h->lay.status_offset);
  cudaError_t e = cudaMemcpyAsync(&v, dev, sizeof(v), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_failed(e);
  // the clear also zeroes the rows' arrival counters, which a launch whose
  // waits ran out may have left behind
  if (clear) launch_clear_words(dev, 1 + h->cfg.batch * h->cfg.num_kv_heads, st);
  if (bits) *bits = v;
  return v ? KVQ_ERR_DEVICE_STATUS : KVQ_OK;
}

int32_t kvq_seq_len(const kvq_cache* h) { return h ? h->seq_len : -1; }
int32_t kvq_quantized_len(const kvq_cache* h) { return h ? h->tq : -1; }
int32_t kvq_window_len(const kvq_cache* h) { return h ? h->r : -1; }
int32_t kvq_window_head(const kvq_cache* h) { return h ? h->head : -1; }

kvq_status kvq_cache_set_state(kvq_cache* h, int32_t seq_len, int32_t quantized_len, int32_t window_head) {
  if (!h) return KVQ_ERR_INVALID_ARG;
  const kvq_config& c = h->cfg;
  const int32_t G = c.group, cap = c.residual + c.group;
  if (seq_len < 0 || quantized_len < 0 || quantized_len % G != 0 || window_head < 0 || window_head >= cap ||
      window_head % G != 0)
    return KVQ_ERR_INVALID_ARG;
  const int32_t r = seq_len - c.anchor_tokens - quantized_len;
  if (r < 0 || r >= cap) return KVQ_ERR_INVALID_ARG;
  if (seq_len > c.max_seq || (uint64_t)(quantized_len / G) > h->lay.groups_per_row) return KVQ_ERR_CAPACITY;
  h->seq_len = seq_len;
  h->tq = quantized_len;
  h->r = r;
  h->head = window_head;
  h->tq_ready = true;   // TURBO: the restored buffer carries its parameter block
  return KVQ_OK;
}

void kvq_cache_destroy(kvq_cache* h) { delete h; }

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "capacity exceeded";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    case KVQ_ERR_DEVICE_STATUS: return "device status word set";
  }
  return "unknown status";
}

uint64_t kvq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

kvq_status kvq_debug_set_wait_test(uint64_t wait_cycles, int32_t withhold_first_stage) {
  if (wait_cycles > (uint64_t)kWaitCyclesDefault) return KVQ_ERR_INVALID_ARG;
  g_wait_cycles.store((long long)wait_cycles, std::memory_order_relaxed);
  g_withhold.store(withhold_first_stage ? 1 : 0, std::memory_order_relaxed);
  return KVQ_OK;
}

const char* kvq_cuda_error_string(void) { return g_cuda_error; }

int32_t kvq_decode_splits(const kvq_cache* h) {
  if (!h) return -1;
  if (h->seq_len <= 0) return 0;   // an empty cache launches nothing
  int32_t n_items, item0[kMaxDecodeCtas + 1];
  return plan_decode(h->cfg, h->tq / h->cfg.group, h->r, num_sms(), &n_items, item0);
}

int32_t kvq_decode_partition(const kvq_config* cfg, int64_t n_groups, int32_t r, int32_t sms, int32_t* item0,
                             int32_t cap, int32_t* n_items) {
  if (!cfg || !item0 || !n_items || !config_ok(cfg) || n_groups < 0 || r < 0 || sms < 1) return 0;
  int32_t tmp[kMaxDecodeCtas + 1];
  int32_t ni = 0;
  const int n = plan_decode(*cfg, n_groups, r, sms, &ni, tmp);
  if (n <= 0 || cap < n + 1) return 0;
  std::memcpy(item0, tmp, sizeof(int32_t) * (size_t)(n + 1));
  *n_items = ni;
  return n;
}

}  // extern "C"

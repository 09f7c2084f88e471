// runtime.cu -- the bt_* C-ABI: model creation, prefill and decode schedules.
//
// Schedules follow the inference stages of "Block Transformer: Global-to-Local
// Language Modeling for Fast Inference" (§3.4 "Prefill vs. decode" and the
// per-component cost analyses):
//   prefill  embed all prompt blocks, run the block decoder over them (KV
//            cache filled), then only the last block's context enters the
//            token decoder (prefix rows) -> logits for the next token;
//   decode   every call feeds one token; a token that completes its block
//            triggers one block-decoder step (one new cache entry) and a new
//            token-decoder block from the fresh context; other tokens append
//            one row to the token decoder's local cache.
// Each decode call is one CUDA-graph launch (graphs captured lazily per step
// kind); the step position lives in device memory so graphs are reusable.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <string>
#include <vector>

#include "../../include/bt.h"
#include "common.cuh"
#include "kernels.h"

using namespace bt;

static thread_local std::string g_last_cuda;

void bt::note_cuda_error(const char* what, cudaError_t e) {
  g_last_cuda = std::string(what) + ": " + cudaGetErrorString(e);
}

#define BT_CUDA(call)                                      \
  do {                                                     \
    cudaError_t e__ = (call);                              \
    if (e__ != cudaSuccess) {                              \
      g_last_cuda = std::string(#call) + ": " + cudaGetErrorString(e__); \
      return BT_ECUDA;                                     \
    }                                                      \
  } while (0)

namespace {

struct LayerW {
  void* w_qkv1 = nullptr;  // [Nq + 4D, D] rows q | k | v | fc1
  void* w_o2 = nullptr;    // [D, 5D]   cols W_o | W_2
  float* b_qkv1 = nullptr; // [Nq + 4D]
  int Hk = 0;              // key/value heads (block decoder: H_kv; token decoder: H)
  int Nq = 0;              // q | k | v width: D + 2 Hk d_head (3D without GQA)
  float* b_o2 = nullptr;   // [D]       b_o + b_2
  float *ln1_g = nullptr, *ln1_b = nullptr, *ln2_g = nullptr, *ln2_b = nullptr;
};

// Bump allocator over the caller's workspace (dry run when base == nullptr).
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  void* take(size_t bytes) {
    off = (off + 255) & ~(size_t)255;
    void* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  }
};

struct Dims {
  int V, D, H, d, L, Nb, Nt, P, rot, Bmax, max_seq, dt, tokdec;
  // context injection: inj 0 = prefix, 1 = summation; w = window of context
  // embeddings; Pp = rows per projected context embedding (prefix_len);
  // prows = output rows of the context projection (Pp, or L_B in
  // summation). P above = the token decoder's context rows (w * Pp, or 1).
  int inj, w, Pp, prows;
  int Hkb;     // block decoder's key/value heads (grouped-query attention when < H)
  size_t eb;
  int n_cap;   // block-cache entries per sequence
  int l_cap;   // local-cache rows per sequence
  int R;       // activation rows
  int tab_pos; // rotary table positions
};

int dims_of(const bt_config* c, Dims* o) {
  if (!c) return BT_EINVAL;
  Dims d{};
  d.V = c->vocab; d.D = c->d_model; d.H = c->n_heads; d.L = c->block_len;
  d.Nb = c->n_block_layers; d.tokdec = c->use_token_decoder ? 1 : 0;
  d.Nt = d.tokdec ? c->n_token_layers : 0;
  d.P = d.tokdec ? c->prefix_len : 0;
  d.rot = c->rotary_dims; d.Bmax = c->max_batch; d.max_seq = c->max_seq; d.dt = c->dtype;
  if (d.V <= 0 || d.D <= 0 || d.H <= 0 || d.L <= 0 || d.Nb < 0 || d.Nt < 0 || d.Bmax <= 0 ||
      d.max_seq <= 0)
    return BT_EINVAL;
  if (d.dt != BT_FP32 && d.dt != BT_BF16) return BT_EINVAL;
  if (d.D % d.H || d.D % d.L || d.D % 8) return BT_EINVAL;
  d.d = d.D / d.H;
  if (d.d != 32 && d.d != 64 && d.d != 128) return BT_ENOTSUP;
  if (d.rot < 0 || d.rot > d.d || (d.rot & 1)) return BT_EINVAL;
  if ((d.D / d.L) * (int)dt_size(d.dt) % 4) return BT_ENOTSUP;
  if (d.tokdec) {
    if (d.P < 1) return BT_EINVAL;
  } else if (d.L != 1) {
    return BT_EINVAL;  // vanilla mode is the L_B = 1 special case
  }
  d.inj = d.tokdec ? c->context_injection : 0;
  d.w = (d.tokdec && c->context_window > 0) ? c->context_window : 1;
  if (d.inj != 0 && d.inj != 1) return BT_EINVAL;
  if (d.inj == 1 && (d.P != 1 || d.w != 1)) return BT_EINVAL;
  d.Pp = d.P;
  d.prows = d.inj ? d.L : d.Pp;
  d.Hkb = c->n_kv_heads > 0 ? c->n_kv_heads : d.H;
  if (d.H % d.Hkb) return BT_EINVAL;
  if (d.tokdec && !d.inj) d.P = d.w * d.Pp;
  if (!(c->ln_eps > 0.f) || !(c->rope_base > 0.f)) return BT_EINVAL;
  d.eb = dt_size(d.dt);
  d.n_cap = (d.max_seq + d.L - 1) / d.L;
  d.l_cap = d.tokdec ? d.P + d.L - 1 : 1;
  {
    // every buffer's element count must stay below 2^31: kernels index
    // within one buffer (one layer of a cache) with 32-bit arithmetic. The
    // widest per-row activation buffer is [rows, 5D] (attention output |
    // GELU(fc1), the out|fc2 GEMM's input)
    const long long lim = 1LL << 31;
    const long long B = d.Bmax, D = d.D;
    const long long rows = B * (d.n_cap > d.l_cap ? d.n_cap : d.l_cap);
    const long long vt_ld = (d.n_cap + 63) / 64 * 64;
    if (rows * 5 * D >= lim || B * d.V >= lim || B * D * vt_ld >= lim || B * D * d.n_cap >= lim)
      return BT_ENOTSUP;
  }
  const int rows_blk = d.Bmax * d.n_cap;
  // token-decoder rows of one call: P prefix rows plus up to L_B - 1
  // trailing prompt tokens at prefill
  const int rows_tok = d.Bmax * (d.tokdec ? d.P + d.L - 1 : 1);
  d.R = rows_blk > rows_tok ? rows_blk : rows_tok;
  d.tab_pos = d.n_cap > d.l_cap ? d.n_cap : d.l_cap;
  *o = d;
  return BT_OK;
}

}  // namespace

struct bt_model {
  bt_config cfg;
  Dims d;
  cudaStream_t stream = nullptr;      // caller's
  cudaStream_t cap_stream = nullptr;  // private, for graph capture
  std::vector<LayerW> blk, tok;
  void *blk_emb = nullptr, *tok_emb = nullptr, *w_prefix = nullptr, *w_lm = nullptr;
  float *b_prefix = nullptr, *lnf_b_g = nullptr, *lnf_b_b = nullptr, *lnf_t_g = nullptr,
        *lnf_t_b = nullptr;
  void *kb = nullptr, *vb = nullptr, *kt = nullptr, *vt = nullptr;
  size_t kb_layer = 0, kt_layer = 0;  // elements per layer
  float *h_b = nullptr, *h_t = nullptr, *logits = nullptr;
  void *x1 = nullptr, *qkv = nullptr, *qrot = nullptr, *a2 = nullptr, *xf = nullptr;
  int32_t *next = nullptr, *fed = nullptr, *block_tok = nullptr;
  // per-sequence prefill layout of a ragged batch (zeros for a uniform one):
  // row_lag [B_max] blocks behind the longest sequence, row_pad [B_max] left
  // pad ids, row_len [B_max] prompt tokens, row_col0 [B_max] first trailing token
  int *row_lag = nullptr, *row_pad = nullptr, *row_len = nullptr, *row_col0 = nullptr;
  bool ragged = false;
  // bound of the waits inside persistent kernels (SM clock cycles): ~1 s at
  // B200 clocks; BT_WAIT_CYCLES (read at bt_create) overrides it
  long long wait_cycles = 2000000000LL;
  int *dstate = nullptr, *status = nullptr;
  float2* rope_tab = nullptr;
  void* attn_scratch = nullptr;
  void* vtr = nullptr;         // V transposed [B_max*H*d][vt_ld] for the prefill attention
  int vt_ld = 0;
  float2* arg_part = nullptr;  // LM-head per-tile argmax partials
  int* ln_cnt = nullptr;       // per-row counters of the LayerNorm fused into GEMM epilogues
  float *ts_p1 = nullptr, *ts_p2 = nullptr;  // fused token step: split-K partials
  long long* ts_fx = nullptr;                // fused token step: fixed-point split-K sums [Bmax][D]
  unsigned long long* ts_key = nullptr;      // fused token step: argmax keys [Bmax]
  unsigned* ts_bar = nullptr;                // fused token step: grid-barrier words
  float* ts_att = nullptr;                   // fused block step: decode-attention partials
  int* ts_cnt = nullptr;                     // fused block step: merge counters [B_max * H]
  unsigned* ts2_ctr = nullptr;               // token_step2: counters
  size_t ts2_ctr_bytes = 0;
  float2* ts_hstat = nullptr;                // token_step2: per-(row, tile) statistics of h
  float* ctx_proj = nullptr;                 // context projection output [B, prows, D]
  float* ctx_ring = nullptr;                 // window of projected context rows [B, w*Pp, D]
  float* sum_add = nullptr;                  // summation vectors s_1.. [B, L_B - 1, D]
  bf16* ts_hb = nullptr;                     // token_step2: bf16 copy of h
  void* l2_base = nullptr;                   // L2 persisting window of the fused token step
  size_t l2_window = 0;                      //   bytes (0: none)
  float l2_hit = 0.f;                        //   hit ratio
  GemmScratch gs{};
  int B = 0, t = 0;
  bool prefilled = false;
  bool use_graphs = true;
  cudaGraphExec_t graphs[2][2][2] = {};  // [block_step][greedy][logits wanted]
  long long graph_kernels[2][2][2] = {};
  int graph_B = 0;
  long long kernels = 0;  // kernels enqueued for execution
  // profiler
  bool prof = false;
  bool capturing = false;
  std::vector<cudaEvent_t> ev;
  std::vector<bt_profile_record> rec;
  std::vector<int> rec_direct;  // per record: event-pair index (direct launch) or -1
  int n_direct = 0;
  int cap_records = 0;
  // profiled decode graphs: event-record nodes around every kernel
  struct Pair { bt_profile_record r; cudaEvent_t a, b; };
  cudaGraphExec_t pgraphs[2][2][2] = {};
  long long pgraph_kernels[2][2][2] = {};
  std::vector<Pair> pairs[2][2][2];
  std::vector<Pair>* cap_pairs = nullptr;  // list being captured into
};

// Event pair around one kernel launch while the profiler is on.
struct ProfScope {
  bt_model* m;
  cudaStream_t s;
  int idx = -1;
  cudaEvent_t end = nullptr;
  ProfScope(bt_model* m_, cudaStream_t s_, int kind, int M, int N, int K) : m(m_), s(s_) {
    if (!m->prof) return;
    if (m->capturing) {
      // inside a profiled graph: the pair becomes two event-record nodes
      if (!m->cap_pairs) return;
      bt_model::Pair p{bt_profile_record{kind, M, N, K, 0.f}, nullptr, nullptr};
      if (cudaEventCreate(&p.a) != cudaSuccess || cudaEventCreate(&p.b) != cudaSuccess) return;
      // external record nodes: real timestamps on every replay
      cudaEventRecordWithFlags(p.a, s, cudaEventRecordExternal);
      end = p.b;
      m->cap_pairs->push_back(p);
      return;
    }
    if ((int)m->rec.size() >= m->cap_records || 2 * (m->n_direct + 1) > (int)m->ev.size()) return;
    idx = m->n_direct++;
    m->rec.push_back(bt_profile_record{kind, M, N, K, 0.f});
    m->rec_direct.push_back(idx);
    cudaEventRecord(m->ev[2 * idx], s);
  }
  ~ProfScope() {
    if (end) cudaEventRecordWithFlags(end, s, cudaEventRecordExternal);
    else if (idx >= 0) cudaEventRecord(m->ev[2 * idx + 1], s);
  }
};

static size_t carve(bt_model* m, const Dims& d, void* ws) {
  Carver c(ws);
  const size_t eb = d.eb;
  const size_t D = d.D;
  auto layer = [&](LayerW& w, int Hk) {
    w.Hk = Hk;
    w.Nq = (int)(D + 2 * (size_t)Hk * d.d);
    w.w_qkv1 = c.take((w.Nq + 4 * D) * D * eb);
    w.w_o2 = c.take(5 * D * D * eb);
    w.b_qkv1 = (float*)c.take((w.Nq + 4 * D) * 4);
    w.b_o2 = (float*)c.take(D * 4);
    w.ln1_g = (float*)c.take(D * 4); w.ln1_b = (float*)c.take(D * 4);
    w.ln2_g = (float*)c.take(D * 4); w.ln2_b = (float*)c.take(D * 4);
  };
  m->blk.assign(d.Nb, LayerW());
  m->tok.assign(d.Nt, LayerW());
  for (auto& w : m->blk) layer(w, d.Hkb);
  for (auto& w : m->tok) layer(w, d.H);
  m->blk_emb = c.take((size_t)d.V * (D / d.L) * eb);
  m->lnf_b_g = (float*)c.take(D * 4); m->lnf_b_b = (float*)c.take(D * 4);
  if (d.tokdec) {
    m->tok_emb = c.take((size_t)d.V * D * eb);
    m->w_prefix = c.take((size_t)d.prows * D * D * eb);
    m->b_prefix = (float*)c.take((size_t)d.prows * D * 4);
    m->lnf_t_g = (float*)c.take(D * 4); m->lnf_t_b = (float*)c.take(D * 4);
  }
  // the LM head and the token decoder's local caches are adjacent: one L2
  // persisting window can cover them (see bt_create)
  m->w_lm = c.take((size_t)d.V * D * eb);
  // caches: [layer][B][H][cap][d]
  m->kt_layer = (size_t)d.Bmax * D * d.l_cap;
  m->kt = c.take(m->kt_layer * (d.Nt > 0 ? d.Nt : 0) * eb);
  m->vt = c.take(m->kt_layer * (d.Nt > 0 ? d.Nt : 0) * eb);
  m->kb_layer = (size_t)d.Bmax * d.Hkb * d.d * d.n_cap;
  m->kb = c.take(m->kb_layer * d.Nb * eb);
  m->vb = c.take(m->kb_layer * d.Nb * eb);
  // activations
  const size_t R = d.R;
  m->h_b = (float*)c.take(R * D * 4);
  m->h_t = (float*)c.take((size_t)d.Bmax * (d.tokdec ? d.P + d.L - 1 : 1) * D * 4);
  m->x1 = c.take(R * 2 * D * eb);
  m->qkv = c.take(R * 3 * D * eb);
  m->qrot = c.take(R * D * eb);
  m->a2 = c.take(R * 5 * D * eb);
  m->xf = c.take((size_t)d.Bmax * D * eb);
  m->logits = (float*)c.take((size_t)d.Bmax * d.V * 4);
  m->next = (int32_t*)c.take((size_t)d.Bmax * 4);
  m->fed = (int32_t*)c.take((size_t)d.Bmax * 4);
  m->block_tok = (int32_t*)c.take((size_t)d.Bmax * d.L * 4);
  m->row_lag = (int*)c.take((size_t)d.Bmax * 4 * sizeof(int));
  if (d.tokdec && (d.inj || d.w > 1)) {
    // context-injection variants: projection output, window ring, the
    // summation vectors of the token rows
    m->ctx_proj = (float*)c.take((size_t)d.Bmax * d.prows * D * 4);
    if (d.w > 1) m->ctx_ring = (float*)c.take((size_t)d.Bmax * d.w * d.Pp * D * 4);
    if (d.inj) m->sum_add = (float*)c.take((size_t)d.Bmax * (d.L > 1 ? d.L - 1 : 1) * D * 4);
  }
  m->row_pad = m->row_lag ? m->row_lag + d.Bmax : nullptr;
  m->row_len = m->row_lag ? m->row_lag + 2 * d.Bmax : nullptr;
  m->row_col0 = m->row_lag ? m->row_lag + 3 * d.Bmax : nullptr;
  m->dstate = (int*)c.take(64);
  m->status = (int*)c.take(64);
  m->rope_tab = (float2*)c.take((size_t)d.tab_pos * (d.rot / 2 > 0 ? d.rot / 2 : 1) * 8);
  m->attn_scratch = c.take(attn_decode_scratch_bytes(d.Bmax, d.H, d.d, d.n_cap, d.dt));
  m->arg_part = (float2*)c.take((size_t)((d.V + 127) / 128) * d.Bmax * sizeof(float2));
  m->ln_cnt = (int*)c.take((size_t)d.Bmax * (d.P > 1 ? d.P : 1) * sizeof(int));
  if (d.tokdec && d.Bmax > 0) {
    m->ts_p1 = (float*)c.take(std::max(token_step_scratch_floats(d.Bmax, d.D, 1),
                                       token_step2_scratch_floats(d.Bmax, d.D, 1)) * 4);
    m->ts_p2 = (float*)c.take(std::max(token_step_scratch_floats(d.Bmax, d.D, 2),
                                       token_step2_scratch_floats(d.Bmax, d.D, 2)) * 4);
    m->ts_bar = (unsigned*)c.take(64);
    m->ts_fx = (long long*)c.take((size_t)d.Bmax * d.D * sizeof(long long));
    m->ts_key = (unsigned long long*)c.take((size_t)d.Bmax * sizeof(unsigned long long));
    m->ts_att = (float*)c.take(token_step_scratch_floats(d.Bmax, d.D, 3, d.H, d.n_cap) * 4);
    m->ts_cnt = (int*)c.take((size_t)d.Bmax * d.H * sizeof(int));
    m->ts2_ctr_bytes = token_step2_counter_bytes(d.D);
    m->ts2_ctr = (unsigned*)c.take(m->ts2_ctr_bytes);
    m->ts_hstat = (float2*)c.take(token_step2_scratch_floats(d.Bmax, d.D, 3) * 4);
    m->ts_hb = (bf16*)c.take(token_step2_scratch_floats(d.Bmax, d.D, 4) * 4);
  }
  m->vt_ld = (d.n_cap + 63) / 64 * 64;
  m->vtr = c.take((size_t)d.Bmax * D * m->vt_ld * eb);
  const int maxN = 7 * d.D > d.V ? 7 * d.D : d.V;
  m->gs.part_bytes = gemm_scratch_bytes(d.Bmax, maxN);
  m->gs.part = (float*)c.take(m->gs.part_bytes);
  m->gs.n_counters = gemm_counter_count(maxN);
  m->gs.counters = (int*)c.take((size_t)m->gs.n_counters * 4);
  return c.off + 256;
}

extern "C" {

const char* bt_strerror(int s) {
  switch (s) {
    case BT_OK: return "ok";
    case BT_EINVAL: return "invalid argument or configuration";
    case BT_EWORKSPACE: return "workspace missing, misaligned or too small";
    case BT_ECAPACITY: return "batch or sequence capacity exceeded";
    case BT_ESTATE: return "decode before prefill";
    case BT_ECUDA: return "CUDA runtime error";
    case BT_EDEVICE: return "device-side failure reported through the status word";
    case BT_ENOTSUP: return "unsupported shape";
    default: return "unknown status";
  }
}

const char* bt_last_cuda_error(void) { return g_last_cuda.c_str(); }

size_t bt_workspace_bytes(const bt_config* cfg) {
  Dims d;
  if (dims_of(cfg, &d) != BT_OK) return 0;
  bt_model tmp;
  return carve(&tmp, d, nullptr);
}

static int copy_layer(bt_model* m, const LayerW& w, const bt_layer_weights& s) {
  const Dims& d = m->d;
  const size_t D = d.D, eb = d.eb;
  cudaStream_t st = m->stream;
  if (!s.w_qkv_dev || !s.w_o_dev || !s.w_1_dev || !s.w_2_dev || !s.b_qkv_dev || !s.b_o_dev ||
      !s.b_1_dev || !s.b_2_dev || !s.ln1_g_dev || !s.ln1_b_dev || !s.ln2_g_dev || !s.ln2_b_dev)
    return BT_EINVAL;
  uint8_t* q1 = (uint8_t*)w.w_qkv1;
  const size_t Nq = w.Nq;
  BT_CUDA(cudaMemcpyAsync(q1, s.w_qkv_dev, Nq * D * eb, cudaMemcpyDeviceToDevice, st));
  BT_CUDA(cudaMemcpyAsync(q1 + Nq * D * eb, s.w_1_dev, 4 * D * D * eb,
                          cudaMemcpyDeviceToDevice, st));
  uint8_t* o2 = (uint8_t*)w.w_o2;
  BT_CUDA(cudaMemcpy2DAsync(o2, 5 * D * eb, s.w_o_dev, D * eb, D * eb, D,
                            cudaMemcpyDeviceToDevice, st));
  BT_CUDA(cudaMemcpy2DAsync(o2 + D * eb, 5 * D * eb, s.w_2_dev, 4 * D * eb, 4 * D * eb, D,
                            cudaMemcpyDeviceToDevice, st));
  BT_CUDA(launch_convert_to_f32(d.dt, s.b_qkv_dev, w.b_qkv1, Nq, st));
  BT_CUDA(launch_convert_to_f32(d.dt, s.b_1_dev, w.b_qkv1 + Nq, 4 * D, st));
  BT_CUDA(launch_add_to_f32(d.dt, s.b_o_dev, s.b_2_dev, w.b_o2, D, st));
  BT_CUDA(launch_convert_to_f32(d.dt, s.ln1_g_dev, w.ln1_g, D, st));
  BT_CUDA(launch_convert_to_f32(d.dt, s.ln1_b_dev, w.ln1_b, D, st));
  BT_CUDA(launch_convert_to_f32(d.dt, s.ln2_g_dev, w.ln2_g, D, st));
  BT_CUDA(launch_convert_to_f32(d.dt, s.ln2_b_dev, w.ln2_b, D, st));
  return BT_OK;
}

int bt_create(const bt_config* cfg, const bt_weights* w, void* ws, size_t ws_bytes, void* stream,
              bt_model** out) {
  if (!out || !w) return BT_EINVAL;
  *out = nullptr;
  Dims d;
  int rc = dims_of(cfg, &d);
  if (rc != BT_OK) return rc;
  if (!ws || ((uintptr_t)ws & 255)) return BT_EWORKSPACE;
  bt_model* m = new bt_model();
  m->cfg = *cfg;
  m->d = d;
  m->stream = (cudaStream_t)stream;
  const size_t need = carve(m, d, ws);
  if (ws_bytes < need) { delete m; return BT_EWORKSPACE; }
  const char* ng = getenv("BT_NO_GRAPH");
  m->use_graphs = !(ng && ng[0] == '1');
  if (const char* wc = getenv("BT_WAIT_CYCLES")) {
    const long long v = atoll(wc);
    if (v > 0) m->wait_cycles = v;
  }
  if (!w->blk_emb_dev || !w->lnf_b_g_dev || !w->lnf_b_b_dev || !w->w_lm_dev ||
      (d.Nb > 0 && !w->block_layers) || (d.Nt > 0 && !w->token_layers) ||
      (d.tokdec && (!w->w_prefix_dev || !w->b_prefix_dev || !w->tok_emb_dev ||
                    !w->lnf_t_g_dev || !w->lnf_t_b_dev))) {
    delete m;
    return BT_EINVAL;
  }
  cudaStream_t st = m->stream;
  auto fail = [&](int code) { delete m; return code; };
#define BT_TRY(x) do { int r__ = (x); if (r__ != BT_OK) return fail(r__); } while (0)
#define BT_TRYC(x) do { cudaError_t e__ = (x); if (e__ != cudaSuccess) { g_last_cuda = std::string(#x) + ": " + cudaGetErrorString(e__); return fail(BT_ECUDA); } } while (0)
  for (int l = 0; l < d.Nb; ++l) BT_TRY(copy_layer(m, m->blk[l], w->block_layers[l]));
  for (int l = 0; l < d.Nt; ++l) BT_TRY(copy_layer(m, m->tok[l], w->token_layers[l]));
  const size_t D = d.D, eb = d.eb;
  BT_TRYC(cudaMemcpyAsync(m->blk_emb, w->blk_emb_dev, (size_t)d.V * (D / d.L) * eb,
                          cudaMemcpyDeviceToDevice, st));
  BT_TRYC(launch_convert_to_f32(d.dt, w->lnf_b_g_dev, m->lnf_b_g, D, st));
  BT_TRYC(launch_convert_to_f32(d.dt, w->lnf_b_b_dev, m->lnf_b_b, D, st));
  if (d.tokdec) {
    BT_TRYC(cudaMemcpyAsync(m->tok_emb, w->tok_emb_dev, (size_t)d.V * D * eb,
                            cudaMemcpyDeviceToDevice, st));
    BT_TRYC(cudaMemcpyAsync(m->w_prefix, w->w_prefix_dev, (size_t)d.prows * D * D * eb,
                            cudaMemcpyDeviceToDevice, st));
    BT_TRYC(launch_convert_to_f32(d.dt, w->b_prefix_dev, m->b_prefix, (size_t)d.prows * D, st));
    BT_TRYC(launch_convert_to_f32(d.dt, w->lnf_t_g_dev, m->lnf_t_g, D, st));
    BT_TRYC(launch_convert_to_f32(d.dt, w->lnf_t_b_dev, m->lnf_t_b, D, st));
  }
  BT_TRYC(cudaMemcpyAsync(m->w_lm, w->w_lm_dev, (size_t)d.V * D * eb, cudaMemcpyDeviceToDevice, st));
  BT_TRYC(launch_rope_table(m->rope_tab, d.tab_pos, d.rot, cfg->rope_base, st));
  BT_TRYC(cudaMemsetAsync(m->status, 0, 64, st));
  BT_TRYC(cudaMemsetAsync(m->dstate, 0, 64, st));
  BT_TRYC(cudaMemsetAsync(m->attn_scratch, 0, attn_decode_scratch_bytes(d.Bmax, d.H, d.d, d.n_cap, d.dt), st));
  BT_TRYC(cudaMemsetAsync(m->gs.counters, 0, (size_t)m->gs.n_counters * 4, st));
  BT_TRYC(cudaMemsetAsync(m->block_tok, 0, (size_t)d.Bmax * d.L * 4, st));
  BT_TRYC(cudaMemsetAsync(m->row_lag, 0, (size_t)d.Bmax * 4 * sizeof(int), st));
  BT_TRYC(cudaMemsetAsync(m->ln_cnt, 0, (size_t)d.Bmax * (d.P > 1 ? d.P : 1) * sizeof(int), st));
  if (m->ts_bar) BT_TRYC(cudaMemsetAsync(m->ts_bar, 0, 64, st));
  if (m->ts_fx) BT_TRYC(cudaMemsetAsync(m->ts_fx, 0, (size_t)d.Bmax * d.D * sizeof(long long), st));
  if (m->ts_key) BT_TRYC(cudaMemsetAsync(m->ts_key, 0, (size_t)d.Bmax * sizeof(unsigned long long), st));
  if (m->ts_cnt) BT_TRYC(cudaMemsetAsync(m->ts_cnt, 0, (size_t)d.Bmax * d.H * sizeof(int), st));
  if (m->ts2_ctr) BT_TRYC(cudaMemsetAsync(m->ts2_ctr, 0, m->ts2_ctr_bytes, st));
  {
    // The token decoder's local caches (K and V of every layer, at most
    // P + L_B - 1 rows per sequence and head) are written and re-read by
    // every token step of a block: the fused token-step launches carry a
    // persisting L2 access-policy window over them, and this context's
    // persisting set-aside is sized to it as far as the device allows (hit
    // ratio = the fraction that fits). The weights, LM head included, stream
    // through with an evict-first hint. BT_L2_WINDOW=0 turns the window off.
    const char* env = getenv("BT_L2_WINDOW");
    const size_t kv = d.Nt > 0 ? (size_t)((uint8_t*)m->vt + m->kt_layer * d.Nt * d.eb - (uint8_t*)m->kt) : 0;
    int dev = 0, max_persist = 0, max_window = 0;
    if (kv > 0 && !(env && env[0] == '0') && cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&max_persist, cudaDevAttrMaxPersistingL2CacheSize, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&max_window, cudaDevAttrMaxAccessPolicyWindowSize, dev) == cudaSuccess &&
        max_persist > 0 && max_window > 0 && kv <= (size_t)max_window) {
      const size_t want = std::min(kv, (size_t)max_persist);
      size_t cur = 0;
      if (cudaDeviceGetLimit(&cur, cudaLimitPersistingL2CacheSize) == cudaSuccess &&
          (cur >= want || cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, want) == cudaSuccess)) {
        m->l2_base = m->kt;
        m->l2_window = kv;
        m->l2_hit = (float)std::min(1.0, (double)std::max(cur, want) / (double)kv);
      }
      cudaGetLastError();
    }
  }
  BT_TRYC(cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking));
  if (d.dt == BT_BF16) BT_TRYC(gemm_tc_prepare());
  BT_TRYC(attn_prepare());
#undef BT_TRY
#undef BT_TRYC
  *out = m;
  return BT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// schedule pieces
// ---------------------------------------------------------------------------
enum AttnKind { ATT_PREFILL, ATT_DECODE, ATT_LOCAL };

// LayerNorm to fuse into the epilogue of a GEMM that completes residual rows
// (decode): dual (g2 != null) -> x1; single -> rows m % step == off of xf.
struct NextLN {
  const float *g1 = nullptr, *b1 = nullptr, *g2 = nullptr, *b2 = nullptr;
  void* out = nullptr;
  int step = 1, off = 0;
};

static void attach_ln(bt_model* m, Epi& e, const NextLN* nl) {
  if (!nl || !nl->g1) return;
  e.ln_g1 = nl->g1; e.ln_b1 = nl->b1; e.ln_g2 = nl->g2; e.ln_b2 = nl->b2;
  e.ln_out = nl->out; e.ln_cnt = m->ln_cnt; e.ln_step = nl->step; e.ln_off = nl->off;
  e.ln_eps = m->cfg.ln_eps;
}

static NextLN dual_ln(bt_model* m, const LayerW& w) {
  NextLN n;
  n.g1 = w.ln1_g; n.b1 = w.ln1_b; n.g2 = w.ln2_g; n.b2 = w.ln2_b; n.out = m->x1;
  return n;
}

static NextLN single_ln(bt_model* m, const float* g, const float* b, int step, int off) {
  NextLN n;
  n.g1 = g; n.b1 = b; n.out = m->xf; n.step = step; n.off = off;
  return n;
}

// The decode schedule with every LayerNorm fused (ingest and GEMM epilogues)
// needs the tensor-core decode GEMMs and P = 1.
// The decode step runs one LayerNorm kernel per layer by default. With
// BT_DECODE_LN=fused (read when a step kind is first recorded) the GEMM
// epilogues normalise instead: the last tile to finish a row normalises it.
// That schedule has fewer launches but measured slower at batch 64 on B200:
// one CTA then normalises a whole 64-row chunk at the end of the GEMM, where
// the separate kernel spreads the rows over 64 CTAs.
static bool fused_decode(const bt_model* m, int B) {
  const Dims& d = m->d;
  const char* env = getenv("BT_DECODE_LN");
  if (!env || strcmp(env, "fused") != 0) return false;
  return d.dt == BT_BF16 && B <= 256 && d.D <= 2048 && (d.D % 128) == 0 &&
         gemm_tc_supported(d.dt, B, d.D, 5 * d.D, 1 << 30, 0) && (!d.tokdec || (d.P == 1 && !d.inj));
}

static int run_layer(bt_model* m, const LayerW& w, float* h, int M, PosSpec pos, void* kc,
                     void* vc, int cap, AttnKind ak, int n_prefill, cudaStream_t s,
                     bool ln_done = false, const NextLN* next = nullptr) {
  const Dims& d = m->d;
  const int D = d.D;
  if (!ln_done) {
    ProfScope p(m, s, BT_K_LAYERNORM, M, D, 0);
    BT_CUDA(launch_ln_dual(d.dt, h, M, D, w.ln1_g, w.ln1_b, w.ln2_g, w.ln2_b, m->cfg.ln_eps, m->x1, s));
  }
  // the fused rotary epilogue does not write V^T, which the tensor-core
  // prefill attention reads: prefill takes the separate rotary kernel then
  const bool pf_tc = ak == ATT_PREFILL && attn_prefill_tc_supported(d.dt, d.d, D, m->vt_ld);
  const int Nq = w.Nq, N1 = w.Nq + 4 * D;  // q|k|v width (w.Hk key/value heads), + fc1
  if (!pf_tc && gemm_rope_fusable(d.dt, M, N1, D, Nq, D, d.d, d.rot)) {
    // q|k|v|fc1 GEMM with rotary and the KV-cache append in its epilogue
    ProfScope p(m, s, BT_K_GEMM, M, N1, D);
    Epi e1{EPI_QKV1_ROPE, m->qrot, D, m->a2, 5 * D, w.b_qkv1, Nq, D,
           m->rope_tab, d.rot, d.H, kc, vc, cap, pos};
    e1.Hk = w.Hk;
    BT_CUDA(launch_gemm(d.dt, m->x1, 2 * D, w.w_qkv1, D, M, N1, D, Nq, D, e1, m->gs, m->status, s));
  } else {
    {
      ProfScope p(m, s, BT_K_GEMM, M, N1, D);
      Epi e1{EPI_QKV1, m->qkv, Nq, m->a2, 5 * D, w.b_qkv1, Nq, D};
      BT_CUDA(launch_gemm(d.dt, m->x1, 2 * D, w.w_qkv1, D, M, N1, D, Nq, D, e1, m->gs, m->status, s));
    }
    ProfScope p(m, s, BT_K_ROPE_APPEND, M, Nq, 0);
    // the tensor-core prefill attention reads V through its transpose
    BT_CUDA(launch_rope_append(d.dt, m->qkv, M, D, d.H, d.rot, m->rope_tab, pos, m->qrot, kc, vc,
                               cap, s, pf_tc ? m->vtr : nullptr, m->vt_ld, w.Hk));
  }
  const int Bseq = M / pos.rows_per_seq;
  if (ak == ATT_PREFILL) {
    ProfScope p(m, s, BT_K_ATTN_PREFILL, Bseq * d.H, n_prefill, d.d);
    if (attn_prefill_tc_supported(d.dt, d.d, D, m->vt_ld))
      BT_CUDA(launch_attn_prefill_tc(m->qrot, D, kc, m->vtr, m->vt_ld, Bseq, d.H, d.d, cap, n_prefill,
                                     m->a2, 5 * D, m->status, s, w.Hk));
    else
      BT_CUDA(launch_attn_prefill(d.dt, m->qrot, D, kc, vc, Bseq, d.H, d.d, cap, n_prefill, m->a2, 5 * D, s,
                                  w.Hk));
  } else if (ak == ATT_DECODE) {
    // entries read: the block index of the fed token + 1 (known on the host)
    ProfScope p(m, s, BT_K_ATTN_DECODE, Bseq * d.H, m->t / d.L + 1, d.d);
    BT_CUDA(launch_attn_decode(d.dt, m->qrot, D, kc, vc, Bseq, d.H, d.d, cap, pos, m->a2, 5 * D,
                               m->attn_scratch, m->status, s, w.Hk));
  } else {
    ProfScope p(m, s, BT_K_ATTN_LOCAL, M * d.H, cap, d.d);
    BT_CUDA(launch_attn_small(d.dt, m->qrot, D, kc, vc, Bseq, d.H, d.d, cap, pos, m->a2, 5 * D, s, w.Hk));
  }
  {
    ProfScope p(m, s, BT_K_GEMM, M, D, 5 * D);
    Epi e2{EPI_RESID, h, D, nullptr, 0, w.b_o2, 0, D};
    attach_ln(m, e2, next);
    BT_CUDA(launch_gemm(d.dt, m->a2, 5 * D, w.w_o2, 5 * D, M, D, 5 * D, 1 << 30, 0, e2, m->gs, m->status, s));
  }
  return BT_OK;
}

static void* layer_ptr(void* base, size_t layer_elems, int l, size_t eb) {
  return (uint8_t*)base + (size_t)l * layer_elems * eb;
}

// token decoder over rows_per_seq rows per sequence, then LN_t of the last
// of them into xf
static int run_token_decoder(bt_model* m, int B, PosSpec pos, cudaStream_t s) {
  const Dims& d = m->d;
  const int M = B * pos.rows_per_seq;
  for (int l = 0; l < d.Nt; ++l) {
    int rc = run_layer(m, m->tok[l], m->h_t, M, pos, layer_ptr(m->kt, m->kt_layer, l, d.eb),
                       layer_ptr(m->vt, m->kt_layer, l, d.eb), d.l_cap, ATT_LOCAL, 0, s);
    if (rc != BT_OK) return rc;
  }
  ProfScope p(m, s, BT_K_LAYERNORM, B, d.D, 0);
  BT_CUDA(launch_ln_rows(d.dt, m->h_t, B, pos.rows_per_seq, pos.rows_per_seq - 1, d.D, m->lnf_t_g,
                         m->lnf_t_b, m->cfg.ln_eps, m->xf, s));
  return BT_OK;
}

// Trailing prompt tokens entering the token decoder after the prefix rows.
struct Tail {
  const int32_t* tokens = nullptr;  // [B, T_len]
  int T_len = 0, col0 = 0, r = 0;   // tokens col0 .. col0 + r - 1 of each row
  const int* row_col0 = nullptr;    // per-sequence col0 (ragged batches)
};

// context rows (B rows of h_b, row r*row_step + row_off) -> LN_b -> either the
// prefix projection and the token decoder over P rows (plus the trailing
// prompt tokens of `tail`), or (vanilla) xf.
static int run_context_to_head_input(bt_model* m, int B, int row_step, int row_off, cudaStream_t s,
                                     const Tail& tail = Tail(), const int* row_lag = nullptr,
                                     bool block_call = false) {
  const Dims& d = m->d;
  {
    ProfScope p(m, s, BT_K_LAYERNORM, B, d.D, 0);
    BT_CUDA(launch_ln_rows(d.dt, m->h_b, B, row_step, row_off, d.D, m->lnf_b_g, m->lnf_b_b,
                           m->cfg.ln_eps, m->xf, s, row_lag));
  }
  if (!d.tokdec) return BT_OK;
  const int rows = d.P + tail.r;  // token-decoder rows per sequence
  if (!d.inj && d.w == 1) {
    // prefix rows: h_t[b*rows + p, :] = (W_p c_b + b_p)[p*D:(p+1)*D]
    ProfScope p(m, s, BT_K_GEMM, B, d.P * d.D, d.D);
    Epi ep{EPI_F32, m->h_t, rows * d.D, nullptr, 0, m->b_prefix, 0, d.D};
    BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_prefix, d.D, B, d.P * d.D, d.D, 1 << 30, 0, ep, m->gs,
                        m->status, s));
  } else if (d.inj) {
    // summation: s = W_p c + b_p -> [B, L_B, D]; s_0 is the context row,
    // s_1.. wait for the block's token rows
    {
      ProfScope p(m, s, BT_K_GEMM, B, d.prows * d.D, d.D);
      Epi ep{EPI_F32, m->ctx_proj, d.prows * d.D, nullptr, 0, m->b_prefix, 0, d.D};
      BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_prefix, d.D, B, d.prows * d.D, d.D, 1 << 30, 0, ep, m->gs,
                          m->status, s));
    }
    ProfScope p(m, s, BT_K_OTHER, B, d.L, d.D);
    BT_CUDA(launch_ctx_rows(CTX_SUM_SPLIT, m->ctx_proj, nullptr, m->h_t, m->sum_add, B, 1, 1, d.L, d.D, rows, s));
  } else if (block_call) {
    // window, block step: project the new context embedding, move the
    // window on by one (oldest first) and keep it for the next block
    {
      ProfScope p(m, s, BT_K_GEMM, B, d.Pp * d.D, d.D);
      Epi ep{EPI_F32, m->ctx_proj, d.Pp * d.D, nullptr, 0, m->b_prefix, 0, d.D};
      BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_prefix, d.D, B, d.Pp * d.D, d.D, 1 << 30, 0, ep, m->gs,
                          m->status, s));
    }
    ProfScope p(m, s, BT_K_OTHER, B, d.P, d.D);
    BT_CUDA(launch_ctx_rows(CTX_WINDOW_SHIFT, m->ctx_proj, m->ctx_ring, m->h_t, nullptr, B, d.w, d.Pp, d.L, d.D,
                            rows, s));
    BT_CUDA(launch_ctx_rows(CTX_WINDOW_SAVE, nullptr, m->ctx_ring, m->h_t, nullptr, B, d.w, d.Pp, d.L, d.D, rows,
                            s));
  } else {
    // window, prefill: the last w context embeddings of every sequence,
    // oldest first, each projected into its Pp rows; zero vectors before the
    // first block (their rows are b_p)
    for (int q = 0; q < d.w; ++q) {
      const int o = row_off - (d.w - 1 - q);
      if (o >= 0) {
        ProfScope p(m, s, BT_K_LAYERNORM, B, d.D, 0);
        BT_CUDA(launch_ln_rows(d.dt, m->h_b, B, row_step, o, d.D, m->lnf_b_g, m->lnf_b_b, m->cfg.ln_eps, m->xf, s,
                               row_lag));
      } else {
        BT_CUDA(cudaMemsetAsync(m->xf, 0, (size_t)B * d.D * d.eb, s));
      }
      ProfScope p(m, s, BT_K_GEMM, B, d.Pp * d.D, d.D);
      Epi ep{EPI_F32, m->h_t + (size_t)q * d.Pp * d.D, rows * d.D, nullptr, 0, m->b_prefix, 0, d.D};
      BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_prefix, d.D, B, d.Pp * d.D, d.D, 1 << 30, 0, ep, m->gs,
                          m->status, s));
    }
    ProfScope p(m, s, BT_K_OTHER, B, d.P, d.D);
    BT_CUDA(launch_ctx_rows(CTX_WINDOW_SAVE, nullptr, m->ctx_ring, m->h_t, nullptr, B, d.w, d.Pp, d.L, d.D, rows,
                            s));
  }
  if (tail.r > 0) {
    ProfScope p(m, s, BT_K_EMBED, B * tail.r, d.D, 0);
    BT_CUDA(launch_embed_tail(d.dt, tail.tokens, B, tail.T_len, tail.col0, tail.r, rows, d.P, m->tok_emb, d.V,
                              d.D, m->h_t, m->block_tok, d.L, m->status, s, tail.row_col0,
                              d.inj ? m->sum_add : nullptr));
  }
  PosSpec pos{nullptr, POS_ZERO, 0, rows};
  return run_token_decoder(m, B, pos, s);
}

static int run_head(bt_model* m, int B, bool want_logits, cudaStream_t s) {
  const Dims& d = m->d;
  if (gemm_argmax_fusable(d.dt, B, d.V, d.D)) {
    // LM head with the greedy argmax in its epilogue; logits stored only
    // when the caller asked for them
    {
      ProfScope p(m, s, BT_K_GEMM, B, d.V, d.D);
      Epi el{EPI_LOGITS_ARGMAX, want_logits ? m->logits : nullptr, d.V, nullptr, 0, nullptr, 0, d.D};
      el.aux = m->arg_part;
      BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_lm, d.D, B, d.V, d.D, 1 << 30, 0, el, m->gs, m->status, s));
    }
    ProfScope p(m, s, BT_K_ARGMAX, B, d.V, 0);
    BT_CUDA(launch_argmax_reduce(m->arg_part, (d.V + 127) / 128, B, m->next, s));
    return BT_OK;
  }
  {
    ProfScope p(m, s, BT_K_GEMM, B, d.V, d.D);
    Epi el{EPI_F32, m->logits, d.V, nullptr, 0, nullptr, 0, d.D};
    BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_lm, d.D, B, d.V, d.D, 1 << 30, 0, el, m->gs, m->status, s));
  }
  {
    ProfScope p(m, s, BT_K_ARGMAX, B, d.V, 0);
    BT_CUDA(launch_argmax(m->logits, B, d.V, d.V, m->next, s));
  }
  return BT_OK;
}

static int copy_outputs(bt_model* m, float* logits, int32_t* next) {
  const Dims& d = m->d;
  if (logits)
    BT_CUDA(cudaMemcpyAsync(logits, m->logits, (size_t)m->B * d.V * 4, cudaMemcpyDeviceToDevice, m->stream));
  if (next)
    BT_CUDA(cudaMemcpyAsync(next, m->next, (size_t)m->B * 4, cudaMemcpyDeviceToDevice, m->stream));
  return BT_OK;
}

// Decode call with every LayerNorm fused: the ingest kernel normalises the
// gathered row for the first layer, each layer's residual GEMM normalises the
// completed rows for the next layer (or the final norm), and the argmax
// reduction advances the position.
static int enqueue_decode_fused(bt_model* m, bool block_step, bool greedy, bool want_logits,
                                cudaStream_t s) {
  const Dims& d = m->d;
  const int B = m->B;
  const int32_t* src = greedy ? m->next : m->fed;
  const NextLN lnb = single_ln(m, m->lnf_b_g, m->lnf_b_b, 1, 0);
  const NextLN lnt = d.tokdec ? single_ln(m, m->lnf_t_g, m->lnf_t_b, 1, 0) : NextLN();
  // first LayerNorm of this call
  NextLN first;
  if (block_step) first = d.Nb > 0 ? dual_ln(m, m->blk[0]) : lnb;
  else first = d.Nt > 0 ? dual_ln(m, m->tok[0]) : lnt;
  {
    ProfScope p(m, s, BT_K_EMBED, B, d.D, 0);
    BT_CUDA(launch_ingest_ln(src, m->block_tok, m->dstate, B, d.L, d.V, d.D, block_step ? 1 : 0,
                             m->blk_emb, m->tok_emb, block_step ? m->h_b : m->h_t, first.g1,
                             first.b1, first.g2, first.b2, m->cfg.ln_eps, first.out, m->status, s));
  }
  int rc;
  auto token_layers = [&](PosSpec pos) -> int {
    for (int l = 0; l < d.Nt; ++l) {
      const NextLN nx = (l + 1 < d.Nt) ? dual_ln(m, m->tok[l + 1]) : lnt;
      int r = run_layer(m, m->tok[l], m->h_t, B, pos, layer_ptr(m->kt, m->kt_layer, l, d.eb),
                        layer_ptr(m->vt, m->kt_layer, l, d.eb), d.l_cap, ATT_LOCAL, 0, s, true, &nx);
      if (r != BT_OK) return r;
    }
    return BT_OK;
  };
  if (block_step) {
    PosSpec pos{m->dstate, POS_BLOCK, 0, 1, m->row_lag};
    for (int l = 0; l < d.Nb; ++l) {
      const NextLN nx = (l + 1 < d.Nb) ? dual_ln(m, m->blk[l + 1]) : lnb;
      rc = run_layer(m, m->blk[l], m->h_b, B, pos, layer_ptr(m->kb, m->kb_layer, l, d.eb),
                     layer_ptr(m->vb, m->kb_layer, l, d.eb), d.n_cap, ATT_DECODE, 0, s, true, &nx);
      if (rc != BT_OK) return rc;
    }
    if (d.tokdec) {
      // prefix rows (P = 1) with the token decoder's first LayerNorm fused
      const NextLN nx = d.Nt > 0 ? dual_ln(m, m->tok[0]) : lnt;
      ProfScope p(m, s, BT_K_GEMM, B, d.D, d.D);
      Epi ep{EPI_F32, m->h_t, d.D, nullptr, 0, m->b_prefix, 0, d.D};
      attach_ln(m, ep, &nx);
      BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_prefix, d.D, B, d.D, d.D, 1 << 30, 0, ep, m->gs,
                          m->status, s));
    }
    if (d.tokdec) {
      rc = token_layers(PosSpec{nullptr, POS_ZERO, 0, 1});
      if (rc != BT_OK) return rc;
    }
  } else {
    rc = token_layers(PosSpec{m->dstate, POS_LOCAL, d.P, 1});
    if (rc != BT_OK) return rc;
  }
  // LM head on xf (already normalised) + argmax; the reduction advances the step
  if (gemm_argmax_fusable(d.dt, B, d.V, d.D)) {
    {
      ProfScope p(m, s, BT_K_GEMM, B, d.V, d.D);
      Epi el{EPI_LOGITS_ARGMAX, want_logits ? m->logits : nullptr, d.V, nullptr, 0, nullptr, 0, d.D};
      el.aux = m->arg_part;
      BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_lm, d.D, B, d.V, d.D, 1 << 30, 0, el, m->gs, m->status, s));
    }
    ProfScope p(m, s, BT_K_ARGMAX, B, d.V, 0);
    BT_CUDA(launch_argmax_reduce(m->arg_part, (d.V + 127) / 128, B, m->next, s, m->dstate, d.L));
    return BT_OK;
  }
  rc = run_head(m, B, want_logits, s);
  if (rc != BT_OK) return rc;
  ProfScope p(m, s, BT_K_OTHER, 1, 0, 0);
  BT_CUDA(launch_advance(m->dstate, d.L, s));
  return BT_OK;
}

// The token-decoder half of a decode call (every token-decoder layer, the
// final LayerNorm, the LM head, the argmax and the position advance) runs as
// one persistent kernel where the shape allows; BT_DECODE_TOKEN_STEP=chain
// keeps the kernel-per-operation schedule instead (read when a step kind is
// first recorded).
// Layer l's parameters at a fixed stride from layer 0's (the fused kernels
// address layers by that stride).
static bool uniform_layers(const std::vector<LayerW>& v, long long ls) {
  for (size_t l = 0; l < v.size(); ++l) {
    const LayerW& w = v[l];
    const LayerW& w0 = v[0];
    auto at = [&](const void* p, const void* p0) {
      return (const uint8_t*)p == (const uint8_t*)p0 + (long long)l * ls;
    };
    if (!at(w.w_qkv1, w0.w_qkv1) || !at(w.w_o2, w0.w_o2) || !at(w.b_qkv1, w0.b_qkv1) ||
        !at(w.b_o2, w0.b_o2) || !at(w.ln1_g, w0.ln1_g) || !at(w.ln1_b, w0.ln1_b) ||
        !at(w.ln2_g, w0.ln2_g) || !at(w.ln2_b, w0.ln2_b))
      return false;
  }
  return true;
}

// Which fused kernel runs the token-decoder half of a decode call: 1 = the
// grid-barrier kernel (decode_step.cu, prefix length 1), 2 = the
// counter-synchronised kernel (token_step.cu, any prefix length), 0 = none
// (kernel per operation). BT_DECODE_TOKEN_STEP=chain | v1 | v2 (read when a
// step kind is first recorded) forces one of them.
static int token_step_kind(const bt_model* m, int B) {
  const Dims& d = m->d;
  const char* env = getenv("BT_DECODE_TOKEN_STEP");
  if (env && strcmp(env, "chain") == 0) return 0;
  if (!d.tokdec || d.Nt < 1 || !m->ts_bar) return 0;
  if (d.inj || d.w > 1) return 0;  // context-injection variants: kernel chain
  const long long ls = d.Nt > 1 ? (long long)((uint8_t*)m->tok[1].w_qkv1 - (uint8_t*)m->tok[0].w_qkv1) : 0;
  if (!uniform_layers(m->tok, ls)) return 0;
  const bool only1 = env && strcmp(env, "v1") == 0, only2 = env && strcmp(env, "v2") == 0;
  const bool ok1 = token_step_supported(d.dt, B, d.D, d.H, d.rot, d.V, d.Nt, d.P, d.l_cap);
  const bool ok2 = token_step2_supported(d.dt, B, d.D, d.H, d.rot, d.V, d.Nt, d.l_cap);
  if (only1) return ok1 ? 1 : 0;
  if (only2) return ok2 ? 2 : 0;
  return ok1 ? 1 : (ok2 ? 2 : 0);
}

static bool token_step_fused(const bt_model* m, int B) { return token_step_kind(m, B) != 0; }

// The block-step form of the same kernel (block embedding, block-decoder
// layers with the decode attention as one of its phases, LN_b and the
// prefix projection) is opt-in: BT_DECODE_BLOCK_STEP=fused. On B200 at batch
// 64 it beats the kernel chain while the block cache is short (392 against
// 435 us per block step at ~35 entries) but loses as the cache grows: the
// attention phase has four worker warps per SM where the separate decode-
// attention kernel keeps sixteen consumer warps per SM busy.
static bool block_step_fused(const bt_model* m, int B) {
  const Dims& d = m->d;
  const char* env = getenv("BT_DECODE_BLOCK_STEP");
  if (!env || strcmp(env, "fused") != 0) return false;
  // its attention phase assumes one cache length for the whole batch
  if (!m->ts_att || d.Nb < 1 || d.P != 1 || d.inj || d.Hkb != d.H || m->ragged) return false;
  if (!token_step_block_supported(d.dt, B, d.D, d.H, d.rot, d.V, d.Nt, d.Nb, d.P, d.l_cap, d.n_cap, d.L))
    return false;
  const long long ls = d.Nt > 1 ? (long long)((uint8_t*)m->tok[1].w_qkv1 - (uint8_t*)m->tok[0].w_qkv1) : 0;
  const long long lsb = d.Nb > 1 ? (long long)((uint8_t*)m->blk[1].w_qkv1 - (uint8_t*)m->blk[0].w_qkv1) : ls;
  if (d.Nt > 1 && d.Nb > 1 && ls != lsb) return false;
  const long long stride = d.Nt > 1 ? ls : lsb;
  for (int l = 0; l < d.Nb; ++l) {
    const LayerW& w = m->blk[l];
    const LayerW& w0 = m->blk[0];
    auto at = [&](const void* p, const void* p0) {
      return (const uint8_t*)p == (const uint8_t*)p0 + (long long)l * stride;
    };
    if (!at(w.w_qkv1, w0.w_qkv1) || !at(w.w_o2, w0.w_o2) || !at(w.b_qkv1, w0.b_qkv1) ||
        !at(w.b_o2, w0.b_o2) || !at(w.ln1_g, w0.ln1_g) || !at(w.ln1_b, w0.ln1_b) ||
        !at(w.ln2_g, w0.ln2_g) || !at(w.ln2_b, w0.ln2_b))
      return false;
  }
  return true;
}

static int run_token_step(bt_model* m, int B, bool ingest, PosSpec pos, const int32_t* src,
                          bool want_logits, cudaStream_t s, bool block = false) {
  const Dims& d = m->d;
  const LayerW& w0 = m->tok[0];
  TokenStepArgs a{};
  a.B = B; a.D = d.D; a.H = d.H; a.dh = d.d; a.rot = d.rot; a.V = d.V; a.Nt = d.Nt; a.L_B = d.L;
  a.l_cap = d.l_cap; a.eps = m->cfg.ln_eps; a.ingest = ingest ? 1 : 0; a.pos = pos;
  a.src = src; a.block_tok = m->block_tok; a.tok_emb = (const bf16*)m->tok_emb; a.dstate = m->dstate;
  a.b_qkv1 = w0.b_qkv1; a.b_o2 = w0.b_o2; a.ln1_g = w0.ln1_g; a.ln1_b = w0.ln1_b;
  a.ln2_g = w0.ln2_g; a.ln2_b = w0.ln2_b;
  a.layer_stride = d.Nt > 1 ? (long long)((uint8_t*)m->tok[1].w_qkv1 - (uint8_t*)w0.w_qkv1) : 0;
  a.kt = (bf16*)m->kt; a.vt = (bf16*)m->vt; a.kt_layer = (long long)m->kt_layer;
  a.rope_tab = m->rope_tab; a.lnf_g = m->lnf_t_g; a.lnf_b = m->lnf_t_b;
  a.h = m->h_t; a.x1 = (bf16*)m->x1; a.a2 = (bf16*)m->a2; a.xf = (bf16*)m->xf;
  a.logits = want_logits ? m->logits : nullptr; a.next = m->next; a.arg_part = m->arg_part;
  a.p1 = m->ts_p1; a.p2 = m->ts_p2; a.fx = m->ts_fx; a.arg_key = m->ts_key; a.bar = m->ts_bar;
  a.status = m->status;
  a.wait_cycles = m->wait_cycles;
  a.l2_window_base = m->l2_base;
  a.l2_window_bytes = m->l2_window;
  a.l2_hit_ratio = m->l2_hit;
  const void *wqb = nullptr, *wob = nullptr;
  if (block) {
    const LayerW& b0 = m->blk[0];
    a.block = 1; a.Nb = d.Nb; a.n_cap = d.n_cap;
    if (d.Nt <= 1 && d.Nb > 1)
      a.layer_stride = (long long)((uint8_t*)m->blk[1].w_qkv1 - (uint8_t*)b0.w_qkv1);
    a.blk_emb = (const bf16*)m->blk_emb; a.h_b = m->h_b;
    a.bb_qkv1 = b0.b_qkv1; a.bb_o2 = b0.b_o2; a.bln1_g = b0.ln1_g; a.bln1_b = b0.ln1_b;
    a.bln2_g = b0.ln2_g; a.bln2_b = b0.ln2_b;
    a.kb = (bf16*)m->kb; a.vb = (bf16*)m->vb; a.kb_layer = (long long)m->kb_layer;
    a.lnb_g = m->lnf_b_g; a.lnb_b = m->lnf_b_b; a.b_prefix = m->b_prefix;
    a.att_part = m->ts_att; a.att_cnt = m->ts_cnt;
    wqb = b0.w_qkv1; wob = b0.w_o2;
  }
  ProfScope p(m, s, block ? BT_K_BLOCK_STEP : BT_K_TOKEN_STEP, B, d.V, d.D);
  if (!block && token_step_kind(m, B) == 2) {
    a.bar = m->ts2_ctr;
    a.hstat = m->ts_hstat;
    a.hb = m->ts_hb;
    BT_CUDA(launch_token_step2(a, w0.w_qkv1, w0.w_o2, m->w_lm, s));
    return BT_OK;
  }
  BT_CUDA(launch_token_step(a, w0.w_qkv1, w0.w_o2, m->w_lm, wqb, wob, block ? m->w_prefix : nullptr, s));
  return BT_OK;
}

// Decode call with the token-decoder half fused into one kernel.
static int enqueue_decode_token_step(bt_model* m, bool block_step, bool greedy, bool want_logits,
                                     cudaStream_t s) {
  const Dims& d = m->d;
  const int B = m->B;
  const int32_t* src = greedy ? m->next : m->fed;
  if (!block_step) return run_token_step(m, B, true, PosSpec{m->dstate, POS_LOCAL, d.P, 1}, src, want_logits, s);
  if (block_step_fused(m, B))
    return run_token_step(m, B, false, PosSpec{nullptr, POS_ZERO, 0, 1}, src, want_logits, s, true);
  {
    ProfScope p(m, s, BT_K_EMBED, B, d.D, 0);
    BT_CUDA(launch_ingest(d.dt, src, m->block_tok, m->dstate, B, d.L, d.V, d.D, 1, m->blk_emb,
                          m->tok_emb, m->h_b, m->status, s));
  }
  PosSpec pos{m->dstate, POS_BLOCK, 0, 1, m->row_lag};
  for (int l = 0; l < d.Nb; ++l) {
    int rc = run_layer(m, m->blk[l], m->h_b, B, pos, layer_ptr(m->kb, m->kb_layer, l, d.eb),
                       layer_ptr(m->vb, m->kb_layer, l, d.eb), d.n_cap, ATT_DECODE, 0, s);
    if (rc != BT_OK) return rc;
  }
  {
    ProfScope p(m, s, BT_K_LAYERNORM, B, d.D, 0);
    BT_CUDA(launch_ln_rows(d.dt, m->h_b, B, 1, 0, d.D, m->lnf_b_g, m->lnf_b_b, m->cfg.ln_eps, m->xf, s));
  }
  {
    // the prefix rows h_t[b * P + p] = (W_p c_b + b_p)[p D, (p + 1) D)
    ProfScope p(m, s, BT_K_GEMM, B, d.P * d.D, d.D);
    Epi ep{EPI_F32, m->h_t, d.P * d.D, nullptr, 0, m->b_prefix, 0, d.D};
    BT_CUDA(launch_gemm(d.dt, m->xf, d.D, m->w_prefix, d.D, B, d.P * d.D, d.D, 1 << 30, 0, ep, m->gs,
                        m->status, s));
  }
  if (d.P == 1) return run_token_step(m, B, false, PosSpec{nullptr, POS_ZERO, 0, 1}, src, want_logits, s);
  // several prefix rows: the token decoder over them as separate kernels
  int rc = run_token_decoder(m, B, PosSpec{nullptr, POS_ZERO, 0, d.P}, s);
  if (rc != BT_OK) return rc;
  rc = run_head(m, B, want_logits, s);
  if (rc != BT_OK) return rc;
  ProfScope p(m, s, BT_K_OTHER, 1, 0, 0);
  BT_CUDA(launch_advance(m->dstate, d.L, s));
  return BT_OK;
}

// the body of one decode call (captured into a graph or run directly)
static int enqueue_decode(bt_model* m, bool block_step, bool greedy, bool want_logits,
                          cudaStream_t s) {
  const Dims& d = m->d;
  const int B = m->B;
  if (token_step_fused(m, B)) return enqueue_decode_token_step(m, block_step, greedy, want_logits, s);
  if (fused_decode(m, B)) return enqueue_decode_fused(m, block_step, greedy, want_logits, s);
  const int32_t* src = greedy ? m->next : m->fed;
  {
    ProfScope p(m, s, BT_K_EMBED, B, d.D, 0);
    BT_CUDA(launch_ingest(d.dt, src, m->block_tok, m->dstate, B, d.L, d.V, d.D, block_step ? 1 : 0,
                          m->blk_emb, m->tok_emb, block_step ? m->h_b : m->h_t, m->status, s,
                          d.inj ? m->sum_add : nullptr));
  }
  int rc;
  if (block_step) {
    PosSpec pos{m->dstate, POS_BLOCK, 0, 1, m->row_lag};
    for (int l = 0; l < d.Nb; ++l) {
      rc = run_layer(m, m->blk[l], m->h_b, B, pos, layer_ptr(m->kb, m->kb_layer, l, d.eb),
                     layer_ptr(m->vb, m->kb_layer, l, d.eb), d.n_cap, ATT_DECODE, 0, s);
      if (rc != BT_OK) return rc;
    }
    rc = run_context_to_head_input(m, B, 1, 0, s, Tail(), nullptr, true);
    if (rc != BT_OK) return rc;
  } else {
    PosSpec pos{m->dstate, POS_LOCAL, d.P, 1};
    rc = run_token_decoder(m, B, pos, s);
    if (rc != BT_OK) return rc;
  }
  rc = run_head(m, B, want_logits, s);
  if (rc != BT_OK) return rc;
  {
    ProfScope p(m, s, BT_K_OTHER, 1, 0, 0);
    BT_CUDA(launch_advance(m->dstate, d.L, s));
  }
  return BT_OK;
}

static void drop_graphs(bt_model* m) {
  for (auto& a : m->graphs)
    for (auto& b : a)
      for (auto& g : b)
        if (g) { cudaGraphExecDestroy(g); g = nullptr; }
}

extern "C" {

}  // extern "C"

// Prefill of B sequences whose prompts sit at the start of the rows of
// tokens [B, T_stride]. lengths == nullptr: every prompt has T_stride tokens.
// Otherwise lengths[b] (host) tokens each; pad_id >= 0 left-pads every prompt
// to a block boundary with that id, pad_id < 0 requires the same remainder
// mod L_B for every length.
static int prefill_impl(bt_model* m, const int32_t* tokens, int T_stride, int B, const int32_t* lengths,
                        int pad_id, float* logits, int32_t* next) {
  if (!m || !tokens) return BT_EINVAL;
  const Dims& d = m->d;
  if (B < 1 || B > d.Bmax) return BT_ECAPACITY;
  // per-sequence layout: padded length, complete blocks, lag behind the longest
  std::vector<int> host(4 * (size_t)d.Bmax, 0);
  int T = T_stride;  // the longest (padded) prompt
  bool ragged = false;
  if (lengths) {
    if (pad_id >= d.V) return BT_EINVAL;
    int rem = -1;
    T = 0;
    for (int b = 0; b < B; ++b) {
      const int len = lengths[b];
      if (len < 1 || len > T_stride) return BT_EINVAL;
      const int pad = pad_id >= 0 ? (d.L - len % d.L) % d.L : 0;
      const int Tb = len + pad;
      if (Tb < d.L) return BT_EINVAL;
      if (rem < 0) rem = Tb % d.L;
      else if (Tb % d.L != rem) return BT_EINVAL;  // the token decoders must stay in step
      host[d.Bmax + b] = pad;
      host[2 * d.Bmax + b] = len;
      if (Tb > T) T = Tb;
      if (Tb != T_stride || pad) ragged = true;
    }
    for (int b = 0; b < B; ++b) {
      const int Tb = host[2 * d.Bmax + b] + host[d.Bmax + b];
      host[b] = (T - Tb) / d.L;                                    // lag in blocks
      host[3 * d.Bmax + b] = (Tb / d.L) * d.L - host[d.Bmax + b];  // first trailing token
    }
  }
  if (T < d.L) return BT_EINVAL;
  if (T >= d.max_seq) return BT_ECAPACITY;
  cudaStream_t s = m->stream;
  m->B = B;
  m->t = T;
  if (m->ragged != ragged) drop_graphs(m);  // the block-step schedule depends on it
  m->ragged = ragged;
  const int n = T / d.L;       // complete blocks of the longest sequence: block-decoder rows
  const int r = T - n * d.L;   // trailing tokens: the current block so far
  const int M = B * n;
  BT_CUDA(cudaMemcpyAsync(m->row_lag, host.data(), host.size() * sizeof(int), cudaMemcpyHostToDevice, s));
  // a new session: merge counters of the decode attention start from zero
  BT_CUDA(cudaMemsetAsync(m->attn_scratch, 0,
                          attn_decode_scratch_bytes(d.Bmax, d.H, d.d, d.n_cap, d.dt), s));
  // and the fused token step's barrier words (an aborted step leaves them set)
  if (m->ts_bar) BT_CUDA(cudaMemsetAsync(m->ts_bar, 0, 64, s));
  // and its fixed-point accumulators (an aborted step can leave sums in them)
  if (m->ts_fx) BT_CUDA(cudaMemsetAsync(m->ts_fx, 0, (size_t)d.Bmax * d.D * sizeof(long long), s));
  if (m->ts_key) BT_CUDA(cudaMemsetAsync(m->ts_key, 0, (size_t)d.Bmax * sizeof(unsigned long long), s));
  if (m->ts_cnt) BT_CUDA(cudaMemsetAsync(m->ts_cnt, 0, (size_t)d.Bmax * d.H * sizeof(int), s));
  if (m->ts2_ctr) BT_CUDA(cudaMemsetAsync(m->ts2_ctr, 0, m->ts2_ctr_bytes, s));
  const long long k0 = launch_count();
  BT_CUDA(launch_set_state(m->dstate, T, d.L, s));
  {
    ProfScope p(m, s, BT_K_EMBED, M, d.D, 0);
    BT_CUDA(launch_embed_prompt(d.dt, tokens, B, T_stride, d.L, m->blk_emb, d.V, d.D, m->h_b, m->status, s, n,
                                ragged ? m->row_pad : nullptr, ragged ? m->row_len : nullptr,
                                pad_id >= 0 ? pad_id : 0));
  }
  // a shorter sequence's blocks sit at positions 0 .. n_b - 1 of its rows; the
  // rows after them are computed but never read (causal attention)
  PosSpec pos{nullptr, POS_ZERO, 0, n};
  for (int l = 0; l < d.Nb; ++l) {
    int rc = run_layer(m, m->blk[l], m->h_b, M, pos, layer_ptr(m->kb, m->kb_layer, l, d.eb),
                       layer_ptr(m->vb, m->kb_layer, l, d.eb), d.n_cap, ATT_PREFILL, n, s);
    if (rc != BT_OK) return rc;
  }
  Tail tail;
  tail.tokens = tokens; tail.T_len = T_stride; tail.col0 = n * d.L; tail.r = r;
  tail.row_col0 = ragged ? m->row_col0 : nullptr;
  int rc = run_context_to_head_input(m, B, n, n - 1, s, tail, ragged ? m->row_lag : nullptr);
  if (rc != BT_OK) return rc;
  rc = run_head(m, B, logits != nullptr, s);
  if (rc != BT_OK) return rc;
  m->kernels += launch_count() - k0;
  m->prefilled = true;
  if (m->graph_B != B) { drop_graphs(m); m->graph_B = B; }
  return copy_outputs(m, logits, next);
}

extern "C" {

int bt_prefill(bt_model* m, const int32_t* tokens, int32_t B, int32_t T, float* logits,
               int32_t* next) {
  if (!m || !tokens) return BT_EINVAL;
  if (T < m->d.L) return BT_EINVAL;
  return prefill_impl(m, tokens, T, B, nullptr, -1, logits, next);
}

int bt_prefill_ragged(bt_model* m, const int32_t* tokens, int32_t row_stride, const int32_t* lengths,
                      int32_t B, int32_t pad_id, float* logits, int32_t* next) {
  if (!m || !tokens || !lengths || row_stride < 1) return BT_EINVAL;
  if (m->d.w > 1) return BT_ENOTSUP;  // the window's missing slots would differ per sequence
  return prefill_impl(m, tokens, row_stride, B, lengths, pad_id, logits, next);
}

int bt_decode_step(bt_model* m, const int32_t* tokens, float* logits, int32_t* next) {
  if (!m) return BT_EINVAL;
  if (!m->prefilled) return BT_ESTATE;
  const Dims& d = m->d;
  if (m->t + 1 > d.max_seq) return BT_ECAPACITY;
  const bool block_step = (m->t % d.L) == d.L - 1;
  const bool greedy = tokens == nullptr;
  if (!greedy)
    BT_CUDA(cudaMemcpyAsync(m->fed, tokens, (size_t)m->B * 4, cudaMemcpyDeviceToDevice, m->stream));
  if (m->use_graphs) {
    const int bi = block_step ? 1 : 0, gi = greedy ? 1 : 0, li = logits ? 1 : 0;
    cudaGraphExec_t& g = m->prof ? m->pgraphs[bi][gi][li] : m->graphs[bi][gi][li];
    long long& gk = m->prof ? m->pgraph_kernels[bi][gi][li] : m->graph_kernels[bi][gi][li];
    if (!g) {
      // capture on the private stream, ordered after the caller's stream
      cudaEvent_t ev;
      BT_CUDA(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
      BT_CUDA(cudaEventRecord(ev, m->stream));
      BT_CUDA(cudaStreamWaitEvent(m->cap_stream, ev, 0));
      BT_CUDA(cudaStreamSynchronize(m->cap_stream));
      cudaEventDestroy(ev);
      cudaGraph_t graph;
      BT_CUDA(cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal));
      const long long c0 = launch_count();
      m->capturing = true;
      m->cap_pairs = m->prof ? &m->pairs[bi][gi][li] : nullptr;
      int rc = enqueue_decode(m, block_step, greedy, logits != nullptr, m->cap_stream);
      m->capturing = false;
      m->cap_pairs = nullptr;
      gk = launch_count() - c0;
      cudaError_t ce = cudaStreamEndCapture(m->cap_stream, &graph);
      if (rc != BT_OK) return rc;
      BT_CUDA(ce);
      BT_CUDA(cudaGraphInstantiate(&g, graph, 0));
      cudaGraphDestroy(graph);
    }
    BT_CUDA(cudaGraphLaunch(g, m->stream));
    m->kernels += gk;
    if (m->prof) {
      // read this replay's event pairs
      BT_CUDA(cudaStreamSynchronize(m->stream));
      for (auto& p : m->pairs[bi][gi][li]) {
        if ((int)m->rec.size() >= m->cap_records) break;
        bt_profile_record r = p.r;
        if (r.kind == BT_K_ATTN_DECODE) r.n = m->t / d.L + 1;
        BT_CUDA(cudaEventElapsedTime(&r.ms, p.a, p.b));
        m->rec.push_back(r);
        m->rec_direct.push_back(-1);
      }
    }
  } else {
    const long long c0 = launch_count();
    int rc = enqueue_decode(m, block_step, greedy, logits != nullptr, m->stream);
    if (rc != BT_OK) return rc;
    m->kernels += launch_count() - c0;
  }
  m->t += 1;
  return copy_outputs(m, logits, next);
}

int bt_sync(bt_model* m) {
  if (!m) return BT_EINVAL;
  BT_CUDA(cudaStreamSynchronize(m->stream));
  int st = 0;
  BT_CUDA(cudaMemcpy(&st, m->status, sizeof(int), cudaMemcpyDeviceToHost));
  if (st) {
    BT_CUDA(cudaMemsetAsync(m->status, 0, sizeof(int), m->stream));
    BT_CUDA(cudaStreamSynchronize(m->stream));
    return BT_EDEVICE;
  }
  return BT_OK;
}

int bt_position(const bt_model* m) {
  if (!m) return BT_EINVAL;
  if (!m->prefilled) return BT_ESTATE;
  return m->t;
}

int64_t bt_kernel_launches(const bt_model* m) { return m ? (int64_t)m->kernels : -1; }

static void free_events(bt_model* m) {
  for (auto e : m->ev) cudaEventDestroy(e);
  m->ev.clear();
}

static void drop_pgraphs(bt_model* m) {
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 2; ++j)
      for (int k = 0; k < 2; ++k) {
        if (m->pgraphs[i][j][k]) { cudaGraphExecDestroy(m->pgraphs[i][j][k]); m->pgraphs[i][j][k] = nullptr; }
        for (auto& p : m->pairs[i][j][k]) { cudaEventDestroy(p.a); cudaEventDestroy(p.b); }
        m->pairs[i][j][k].clear();
      }
}

int bt_profile_begin(bt_model* m, int32_t capacity) {
  if (!m || capacity <= 0) return BT_EINVAL;
  free_events(m);
  drop_pgraphs(m);
  m->rec.clear();
  m->rec_direct.clear();
  m->n_direct = 0;
  m->rec.reserve(capacity);
  // event pairs for direct launches (prefill); decode graphs carry their own
  m->ev.resize(2 * (size_t)(capacity < 8192 ? capacity : 8192));
  for (auto& e : m->ev) BT_CUDA(cudaEventCreate(&e));
  m->cap_records = capacity;
  m->prof = true;
  return BT_OK;
}

int bt_profile_end(bt_model* m, bt_profile_record* out, int32_t capacity, int32_t* n_out) {
  if (!m || !m->prof) return BT_EINVAL;
  m->prof = false;
  BT_CUDA(cudaStreamSynchronize(m->stream));
  const int n = (int)m->rec.size() < capacity ? (int)m->rec.size() : capacity;
  for (int i = 0; i < n; ++i) {
    if (m->rec_direct[i] >= 0) {
      float ms = 0.f;
      BT_CUDA(cudaEventElapsedTime(&ms, m->ev[2 * m->rec_direct[i]], m->ev[2 * m->rec_direct[i] + 1]));
      m->rec[i].ms = ms;
    }
    if (out) out[i] = m->rec[i];
  }
  if (n_out) *n_out = n;
  free_events(m);
  drop_pgraphs(m);
  return BT_OK;
}

int bt_destroy(bt_model* m) {
  if (!m) return BT_EINVAL;
  cudaStreamSynchronize(m->stream);
  free_events(m);
  drop_pgraphs(m);
  drop_graphs(m);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  delete m;
  return BT_OK;
}

}  // extern "C"

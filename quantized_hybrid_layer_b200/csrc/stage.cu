// Stage runtime and the C ABI (include/qhl_stage.h).
//
// A stage owns, on one GPU: the packed weights of its layer range, a rollback
// ring of DeltaNet state snapshots per DeltaNet layer, an f16 KV cache per
// attention layer, activation buffers for up to 16 tokens, and one CUDA graph
// per token count.  stage_forward launches that graph, a single submission per
// pass as on the pages (SwarmLLM README, paragraph after the peer diagram).
// Inside the graph every kernel after the first is launched with programmatic
// dependent launch, so a projection's weights start streaming while the
// previous kernel drains.
//
// The position of the pass and each DeltaNet layer's current ring slot live in
// a small device control block (ctrl[0] = committed length, ctrl[1 + i] = ring
// slot of DeltaNet layer i), so the graphs never change; commit advances them
// with one tiny kernel and rollback touches nothing on the device.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/qhl_stage.h"
#include "launch.h"

using namespace qhl;

namespace qhl {
void set_last_error(const std::string& s);   // kernel_abi.cu: message for qhl_last_error()
}

namespace {

constexpr int kMaxTok = 16;
constexpr int kRing = kMaxTok + 1;
// Programmatic dependent launch between the pass's kernels: as the CTAs of a
// projection finish, the next kernel's CTAs take their place and start
// streaming weights while the last tiles are still being finished.  Measured
// on the 64-layer decode pass: 4.19 ms with it, 4.73 ms in plain stream order.
constexpr bool kUsePdl = true;

struct Layer {
  int index = 0;
  bool attn = false;
  uint8_t* w_in = nullptr;
  int in_rows = 0, in_tiles = 0;
  uint8_t* w_out = nullptr;
  int out_cols = 0;
  uint8_t* w_gu = nullptr;
  uint8_t* w_down = nullptr;
  size_t in_bytes = 0, out_bytes = 0, gu_bytes = 0, down_bytes = 0;   // packed sizes, for the launch checks
  float* norm1 = nullptr;
  float* norm2 = nullptr;
  float* qn = nullptr;
  float* kn = nullptr;
  float* ring = nullptr;   // DeltaNet: [kRing][Hv][128][128]
  int dn_slot = -1;
  uint16_t* K = nullptr;   // attention: [Hkv][max_ctx][256] f16 bits
  uint16_t* V = nullptr;
};

std::string cuda_msg(const char* what, cudaError_t e) {
  return std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
}

}  // namespace

struct stage {
  stage_config cfg{};
  int begin = 0, end = 0;
  cudaStream_t stream = nullptr;   // caller's stream: orders every call
  cudaStream_t cap = nullptr;      // private stream used only to capture graphs
  int device = 0, sms = 0;
  std::vector<Layer> layers;
  std::vector<void*> allocs;
  float *h = nullptr, *ss = nullptr, *y = nullptr;
  // GEMV inputs in block fixed point (qact.cuh): normed hidden, mixer output, SwiGLU product
  uint8_t *qz = nullptr, *qo = nullptr, *qu = nullptr;
  int qz_stride = 0, qo_stride = 0, qu_stride = 0;
  float *pm = nullptr, *pl = nullptr, *po = nullptr;
  int nchunk = 0;
  float2* rope = nullptr;
  float* partials = nullptr;
  int* counters = nullptr;
  unsigned* err = nullptr;
  int* ctrl = nullptr;
  int n_dn = 0;
  int ss_stride = 0, y_stride = 0;
  long long state_elems = 0;
  int committed = 0, pending_n = 0, pending_pos = 0;
  std::vector<int> cur;
  // one graph per (kind of pass, token count): kind 0 = forward (per-token
  // snapshots), 1 = exact prefill, 2 = chunked prefill (DnMode)
  cudaGraphExec_t exec[3][kMaxTok + 1] = {};
  // persistent pass: per-layer step arguments on the device, phase counter
  PassLayer* pass_layers = nullptr;
  unsigned* bar = nullptr;
  int n_phases = 0;
  int pass_mode = STAGE_PASS_KERNELS;
  // failure injection for tests of the bounded waits (stage_debug_inject)
  uint32_t dbg_wait_limit = 0;
  int dbg_fault_item = -1;
  int max_tiles = 0;
  size_t weight_bytes = 0;
  std::string last_error;
};

namespace {

stage_status fail(stage* st, stage_status code, const std::string& msg) {
  if (st) st->last_error = msg;
  return code;
}

#define CK(call)                                                            \
  do {                                                                      \
    cudaError_t e_ = (call);                                                \
    if (e_ != cudaSuccess) return fail(st, STAGE_E_CUDA, cuda_msg(#call, e_)); \
  } while (0)

stage_status dalloc(stage* st, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return STAGE_OK;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    *p = nullptr;
    return fail(st, STAGE_E_OOM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed: " + cudaGetErrorString(e));
  }
  st->allocs.push_back(*p);
  return STAGE_OK;
}

template <typename T>
stage_status dalloc_t(stage* st, T** p, size_t bytes) {
  void* v = nullptr;
  stage_status s = dalloc(st, &v, bytes);
  *p = static_cast<T*>(v);
  return s;
}

void destroy(stage* st) {
  if (!st) return;
  if (st->stream || st->cap) cudaDeviceSynchronize();
  for (auto& row : st->exec)
    for (auto& g : row)
      if (g) cudaGraphExecDestroy(g);
  for (void* p : st->allocs) cudaFree(p);
  if (st->cap) cudaStreamDestroy(st->cap);
  delete st;
}

size_t qbytes(int qt, long long rows, long long cols) { return (size_t)(rows * (cols / 32) * gguf_block_bytes(qt)); }

bool parse_name(const char* name, int* layer, std::string* tag) {
  if (!name || std::strncmp(name, "blk.", 4) != 0) return false;
  const char* p = name + 4;
  char* e = nullptr;
  long v = std::strtol(p, &e, 10);
  if (e == p || *e != '.') return false;
  *layer = (int)v;
  *tag = std::string(e + 1);
  return true;
}

// Upload one GGUF matrix into the staging buffer.
stage_status upload(stage* st, void* staging, const stage_tensor* t) {
  CK(cudaMemcpy(staging, t->data, t->bytes, cudaMemcpyHostToDevice));
  return STAGE_OK;
}

GemvArgs gemv_base(const stage* st) {
  GemvArgs a = {};
  a.partials = st->partials;
  a.counters = st->counters;
  a.err = st->err;
  a.eps = st->cfg.eps;
  a.inv_dim = 1.0f / (float)st->cfg.hidden;
  a.wait_limit = st->dbg_wait_limit;
  a.fault_item = -1;
  return a;
}

void set_workers(const stage* st, GemvArgs& a) { a.workers = gemv_workers(a.tiles, a.chunks, st->sms); }

// Arguments of every step of layer i.
// Arguments of the steps of layer i (both execution paths use these, so they
// run the same units with the same split): in-projection, out-projection,
// gate/up, down, and the mixer between the first two.
PassLayer layer_args(const stage* st, size_t i, int dn_mode = DN_SNAPSHOTS) {
  const stage_config& c = st->cfg;
  const int H = c.hidden, F = c.ffn;
  const Layer& L = st->layers[i];
  const float* next_norm1 = i + 1 < st->layers.size() ? st->layers[i + 1].norm1 : nullptr;
  PassLayer P = {};
  P.attn = L.attn ? 1 : 0;
  // mixer in-projection with the RMSNorm1 scale folded into the epilogue
  GemvArgs a = gemv_base(st);
  a.W = L.w_in;
  a.tiles = L.in_tiles;
  a.chunks = H / kChunkCols;
  a.qx = st->qz;
  a.qx_stride = st->qz_stride;
  a.y = st->y;
  a.y_stride = st->y_stride;
  a.out_valid = L.in_rows;
  a.ss_in = st->ss;
  a.ss_tiles = H / kTileRows;
  a.ss_stride = st->ss_stride;
  set_workers(st, a);
  P.g[0] = a;
  if (!L.attn) {
    DnArgs& d = P.dn;
    d.y = st->y;
    d.y_stride = st->y_stride;
    d.Hk = c.dn_k_heads;
    d.Hv = c.dn_v_heads;
    d.ring = L.ring;
    d.state_elems = st->state_elems;
    d.ring_size = kRing;
    d.cur = st->ctrl + 1 + L.dn_slot;
    d.qo = st->qo;
    d.qo_stride = st->qo_stride;
    d.mode = dn_mode;
  } else {
    AttnArgs& at = P.at;
    at.y = st->y;
    at.y_stride = st->y_stride;
    at.Hq = c.att_q_heads;
    at.Hkv = c.att_kv_heads;
    at.K = L.K;
    at.V = L.V;
    at.max_ctx = c.max_ctx;
    at.kv_len = st->ctrl;
    at.gq = L.qn;
    at.gk = L.kn;
    at.rope = st->rope;
    at.eps = c.eps;
    at.pm = st->pm;
    at.pl = st->pl;
    at.po = st->po;
    at.nchunk = st->nchunk;
    at.qout = st->qo;
    at.qout_stride = st->qo_stride;
  }
  // out-projection + residual; z = h * norm2 (block fixed point) and its tile sums of squares
  a = gemv_base(st);
  a.W = L.w_out;
  a.tiles = packed_tiles(H, false);
  a.chunks = L.out_cols / kChunkCols;
  a.qx = st->qo;
  a.qx_stride = st->qo_stride;
  a.y = st->h;
  a.y_stride = H;
  a.out_valid = H;
  a.gamma_next = L.norm2;
  a.qout = st->qz;
  a.qout_stride = st->qz_stride;
  a.ss_out = st->ss;
  a.ss_out_stride = st->ss_stride;
  set_workers(st, a);
  P.g[1] = a;
  // gate/up with the RMSNorm2 scale and the SwiGLU epilogue
  a = gemv_base(st);
  a.W = L.w_gu;
  a.tiles = packed_tiles(F, true);
  a.chunks = H / kChunkCols;
  a.qx = st->qz;
  a.qx_stride = st->qz_stride;
  a.out_valid = F;
  a.qout = st->qu;
  a.qout_stride = st->qu_stride;
  a.ss_in = st->ss;
  a.ss_tiles = H / kTileRows;
  a.ss_stride = st->ss_stride;
  set_workers(st, a);
  P.g[2] = a;
  // down + residual; z for the next layer's RMSNorm1
  a = gemv_base(st);
  a.W = L.w_down;
  a.tiles = packed_tiles(H, false);
  a.chunks = F / kChunkCols;
  a.qx = st->qu;
  a.qx_stride = st->qu_stride;
  a.y = st->h;
  a.y_stride = H;
  a.out_valid = H;
  if (next_norm1) {
    a.gamma_next = next_norm1;
    a.qout = st->qz;
    a.qout_stride = st->qz_stride;
    a.ss_out = st->ss;
    a.ss_out_stride = st->ss_stride;
  }
  set_workers(st, a);
  P.g[3] = a;
  return P;
}

// Record one pass of n tokens onto stream s (being captured) as a chain of
// kernels: stage input, then per layer in-projection, mixer, out-projection,
// gate/up, down.  Every kernel after the first is a programmatic dependent of
// the one before.
// Every projection streams exactly its packed matrix and writes inside its
// output: checked on the host before a pass is recorded, so a geometry error
// fails the recording instead of reaching the device.
bool gemv_fits(const stage* st, const GemvArgs& a, size_t packed, int out_cap) {
  const size_t streamed = (size_t)a.tiles * a.chunks * item_bytes(st->cfg.qtype);
  return streamed == packed && a.workers >= 1 && a.workers <= st->sms && a.out_valid <= out_cap &&
         a.tiles * (long long)kTileRows >= a.out_valid;
}

// Whether an n-token forward can run as the one persistent kernel: n within
// the instantiated range, one CTA per SM resident, and every mixer unit's
// scratch within the kernel's.
// The reason a pass is not eligible is left in last_error (for diagnosis).
bool pass_eligible(stage* st, int n) {
  if (n > kPassMaxTok || !st->pass_layers) {
    st->last_error = "persistent pass: n_tok above " + std::to_string(kPassMaxTok);
    return false;
  }
  int blocks = 0;
  const cudaError_t e = pass_occupancy(st->cfg.qtype, n, &blocks);
  if (e != cudaSuccess || blocks < 1) {
    (void)cudaGetLastError();
    st->last_error = "persistent pass: " + (e != cudaSuccess ? cuda_msg("occupancy query", e)
                                                             : std::string("no CTA fits on an SM"));
    return false;
  }
  const int rep = st->cfg.att_q_heads / st->cfg.att_kv_heads;
  const int need = std::max({dn_smem_floats(n) * 4, combine_smem_bytes(st->nchunk),
                             st->nchunk ? attn_smem_bytes(std::min(n, kAttGroup), rep) : 0});
  if (need > kPassMixBytes) {
    st->last_error = "persistent pass: mixer scratch " + std::to_string(need) + " bytes";
    return false;
  }
  return true;
}

// One persistent kernel for the whole pass, after zeroing its phase counter.
cudaError_t record_persistent(stage* st, int n, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(st->bar, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
  const stage_config& c = st->cfg;
  PassArgs p = {};
  p.layers = st->pass_layers;
  p.n_layers = (int)st->layers.size();
  p.h = st->h;
  p.H = c.hidden;
  p.gamma0 = st->layers[0].norm1;
  p.qz = st->qz;
  p.qz_stride = st->qz_stride;
  p.ss = st->ss;
  p.ss_stride = st->ss_stride;
  p.kv_len = st->ctrl;
  p.bar = st->bar;
  p.grid = st->sms;
  p.dn_units = c.dn_v_heads * (kDnDim / 32);
  p.Hq = c.att_q_heads;
  p.Hkv = c.att_kv_heads;
  p.err = st->err;
  p.wait_limit = st->dbg_wait_limit;
  return launch_pass(c.qtype, n, p, s);
}

cudaError_t record_pass(stage* st, int n, int kind, cudaStream_t s) {
  const stage_config& c = st->cfg;
  const int qt = c.qtype;
  if (kind == DN_SNAPSHOTS && st->pass_mode == STAGE_PASS_PERSISTENT && st->dbg_fault_item < 0 &&
      pass_eligible(st, n))
    return record_persistent(st, n, s);
  cudaError_t e = launch_stage_input(n, st->h, c.hidden, st->layers[0].norm1, st->qz, st->qz_stride, st->ss,
                                     st->ss_stride, s);
  if (e != cudaSuccess) return e;
  for (size_t i = 0; i < st->layers.size(); ++i) {
    PassLayer P = layer_args(st, i, kind);
    // each projection warms L2 with the next one's first items
    auto chain = [](GemvArgs& a, const GemvArgs& next) {
      a.next_W = next.W;
      a.next_items = next.tiles * next.chunks;
      a.next_workers = next.workers;
    };
    chain(P.g[0], P.g[1]);
    chain(P.g[1], P.g[2]);
    chain(P.g[2], P.g[3]);
    if (i + 1 < st->layers.size()) chain(P.g[3], layer_args(st, i + 1).g[0]);
    if (i == 0) P.g[0].fault_item = st->dbg_fault_item;   // injected failure (tests only)
    const Layer& L = st->layers[i];
    if (!gemv_fits(st, P.g[0], L.in_bytes, st->y_stride) || !gemv_fits(st, P.g[1], L.out_bytes, c.hidden) ||
        !gemv_fits(st, P.g[2], L.gu_bytes, c.ffn) || !gemv_fits(st, P.g[3], L.down_bytes, c.hidden))
      return cudaErrorInvalidValue;
    if ((e = launch_gemv(qt, n, EPI_STORE, P.g[0], P.g[0].workers, s, kUsePdl)) != cudaSuccess) return e;
    if (!P.attn) {
      if ((e = launch_dn_step(n, P.dn, c.dn_v_heads * (kDnDim / 32), s, kUsePdl)) != cudaSuccess) return e;
    } else {
      if ((e = launch_attn_partial(n, P.at, st->nchunk, c.att_kv_heads, s, kUsePdl)) != cudaSuccess) return e;
      if ((e = launch_attn_combine(n, P.at, s, kUsePdl)) != cudaSuccess) return e;
    }
    if ((e = launch_gemv(qt, n, EPI_RESID, P.g[1], P.g[1].workers, s, kUsePdl)) != cudaSuccess) return e;
    if ((e = launch_gemv(qt, n, EPI_SWIGLU, P.g[2], P.g[2].workers, s, kUsePdl)) != cudaSuccess) return e;
    if ((e = launch_gemv(qt, n, EPI_RESID, P.g[3], P.g[3].workers, s, kUsePdl)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

stage_status build_graph(stage* st, int n, int kind) {
  CK(cudaStreamBeginCapture(st->cap, cudaStreamCaptureModeThreadLocal));
  cudaError_t e = record_pass(st, n, kind, st->cap);
  cudaGraph_t g = nullptr;
  cudaError_t e2 = cudaStreamEndCapture(st->cap, &g);
  if (e != cudaSuccess || e2 != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    (void)cudaGetLastError();
    return fail(st, STAGE_E_CUDA, cuda_msg("recording the pass", e != cudaSuccess ? e : e2));
  }
  cudaGraphExec_t ex = nullptr;
  e = cudaGraphInstantiate(&ex, g, 0);
  cudaGraphDestroy(g);
  if (e != cudaSuccess) return fail(st, STAGE_E_CUDA, cuda_msg("cudaGraphInstantiate", e));
  st->exec[kind][n] = ex;
  return STAGE_OK;
}

const Layer* find_layer(const stage* st, int layer) {
  if (layer < st->begin || layer >= st->end) return nullptr;
  return &st->layers[layer - st->begin];
}

}  // namespace

extern "C" {

stage_status stage_load(const stage_config* cfg, const stage_tensor* tensors, int n_tensors, int layer_begin,
                        int layer_end, void* cuda_stream, stage_t** out) {
  if (!out) return STAGE_E_ARG;
  *out = nullptr;
  if (!cfg || (!tensors && n_tensors > 0) || n_tensors < 0) return STAGE_E_ARG;
  const stage_config c = *cfg;
  if (layer_begin < 0 || layer_end <= layer_begin) return STAGE_E_ARG;
  if (c.qtype != STAGE_Q4_0 && c.qtype != STAGE_Q8_0) return STAGE_E_UNSUPPORTED;
  if (c.hidden <= 0 || c.hidden % kChunkCols || c.ffn <= 0 || c.ffn % kChunkCols) return STAGE_E_UNSUPPORTED;
  if (c.dn_dim != kDnDim || c.dn_k_heads <= 0 || c.dn_v_heads <= 0 || c.dn_v_heads % c.dn_k_heads)
    return STAGE_E_UNSUPPORTED;
  if (c.att_dim != kAttDim || c.rope_dims != kRopeDims || c.att_kv_heads <= 0 || c.att_q_heads <= 0 ||
      c.att_q_heads % c.att_kv_heads || c.att_q_heads / c.att_kv_heads > 7)
    return STAGE_E_UNSUPPORTED;
  if (c.attn_every <= 0 || c.max_ctx < kMaxTok || c.max_ctx > kAttMaxCtx || !(c.eps > 0.f) || !(c.rope_theta > 0.0))
    return STAGE_E_ARG;

  stage* st = new (std::nothrow) stage();
  if (!st) return STAGE_E_OOM;
  st->cfg = c;
  st->begin = layer_begin;
  st->end = layer_end;
  st->stream = static_cast<cudaStream_t>(cuda_stream);
  auto bail = [&](stage_status s) {
    // the stage is gone: its message stays readable through qhl_last_error()
    set_last_error(st->last_error.empty() ? "stage_load failed" : st->last_error);
    destroy(st);
    return s;
  };

  // --- tensor table ------------------------------------------------------
  std::unordered_map<std::string, const stage_tensor*> by_name;
  for (int i = 0; i < n_tensors; ++i) {
    if (!tensors[i].name || !tensors[i].data) return bail(STAGE_E_ARG);
    by_name[tensors[i].name] = &tensors[i];
  }
  const int H = c.hidden, F = c.ffn, qt = c.qtype;
  const int dn_in = 2 * c.dn_k_heads * kDnDim + c.dn_v_heads * kDnDim + 2 * c.dn_v_heads;
  const int dn_o = c.dn_v_heads * kDnDim;
  const int at_in = 2 * c.att_q_heads * kAttDim + 2 * c.att_kv_heads * kAttDim;
  const int at_o = c.att_q_heads * kAttDim;
  auto need = [&](int layer, const char* tag, size_t bytes, const stage_tensor** t) -> bool {
    auto it = by_name.find("blk." + std::to_string(layer) + "." + tag);
    if (it == by_name.end()) {
      st->last_error = std::string("missing tensor blk.") + std::to_string(layer) + "." + tag;
      return false;
    }
    if (it->second->bytes != bytes) {
      st->last_error = std::string("tensor blk.") + std::to_string(layer) + "." + tag + " has " +
                       std::to_string(it->second->bytes) + " bytes, expected " + std::to_string(bytes);
      return false;
    }
    *t = it->second;
    return true;
  };
  bool any_attn = false;
  size_t max_q = 0;
  for (int l = layer_begin; l < layer_end; ++l) {
    const bool attn = l % c.attn_every == c.attn_every - 1;
    any_attn |= attn;
    const stage_tensor* t;
    if (!need(l, "norm1", (size_t)H * 4, &t) || !need(l, "norm2", (size_t)H * 4, &t)) return bail(STAGE_E_FORMAT);
    if (attn) {
      if (!need(l, "attn_in", qbytes(qt, at_in, H), &t) || !need(l, "attn_out", qbytes(qt, H, at_o), &t) ||
          !need(l, "attn_q_norm", (size_t)kAttDim * 4, &t) || !need(l, "attn_k_norm", (size_t)kAttDim * 4, &t))
        return bail(STAGE_E_FORMAT);
      max_q = std::max({max_q, qbytes(qt, at_in, H), qbytes(qt, H, at_o)});
    } else {
      if (!need(l, "dn_in", qbytes(qt, dn_in, H), &t) || !need(l, "dn_out", qbytes(qt, H, dn_o), &t))
        return bail(STAGE_E_FORMAT);
      max_q = std::max({max_q, qbytes(qt, dn_in, H), qbytes(qt, H, dn_o)});
    }
    if (!need(l, "ffn_gate", qbytes(qt, F, H), &t) || !need(l, "ffn_up", qbytes(qt, F, H), &t) ||
        !need(l, "ffn_down", qbytes(qt, H, F), &t))
      return bail(STAGE_E_FORMAT);
    max_q = std::max({max_q, qbytes(qt, F, H), qbytes(qt, H, F)});
  }

  // --- device setup ------------------------------------------------------
  cudaError_t e;
  if ((e = cudaGetDevice(&st->device)) != cudaSuccess) return bail(fail(st, STAGE_E_CUDA, cuda_msg("cudaGetDevice", e)));
  if ((e = cudaDeviceGetAttribute(&st->sms, cudaDevAttrMultiProcessorCount, st->device)) != cudaSuccess)
    return bail(fail(st, STAGE_E_CUDA, cuda_msg("cudaDeviceGetAttribute", e)));
  if ((e = cudaStreamCreateWithFlags(&st->cap, cudaStreamNonBlocking)) != cudaSuccess)
    return bail(fail(st, STAGE_E_CUDA, cuda_msg("cudaStreamCreate", e)));
  if ((e = gemv_prepare(qt)) != cudaSuccess) return bail(fail(st, STAGE_E_CUDA, cuda_msg("gemv_prepare", e)));
  if ((e = mixers_prepare(c.att_q_heads / c.att_kv_heads)) != cudaSuccess)
    return bail(fail(st, STAGE_E_CUDA, cuda_msg("mixers_prepare", e)));
  if ((e = cudaDeviceSynchronize()) != cudaSuccess) return bail(fail(st, STAGE_E_CUDA, cuda_msg("sync", e)));

  uint8_t *stage_a = nullptr, *stage_b = nullptr;
  stage_status s;
  if ((s = dalloc_t(st, &stage_a, max_q)) != STAGE_OK) return bail(s);
  if ((s = dalloc_t(st, &stage_b, max_q)) != STAGE_OK) return bail(s);

  st->state_elems = (long long)c.dn_v_heads * kDnDim * kDnDim;
  const size_t kv_elems = (size_t)c.att_kv_heads * c.max_ctx * kAttDim;
  for (int l = layer_begin; l < layer_end; ++l) {
    Layer L;
    L.index = l;
    L.attn = l % c.attn_every == c.attn_every - 1;
    auto T = [&](const char* tag) { return by_name["blk." + std::to_string(l) + "." + tag]; };
    auto qmat = [&](const stage_tensor* t, int rows, int cols, uint8_t** dst, size_t* bytes) -> stage_status {
      stage_status r;
      const size_t pb = packed_bytes(qt, rows, cols, false);
      *bytes = pb;
      if ((r = dalloc_t(st, dst, pb)) != STAGE_OK) return r;
      if ((r = upload(st, stage_a, t)) != STAGE_OK) return r;
      cudaError_t ee = launch_repack(qt, stage_a, nullptr, rows, cols, *dst, nullptr);
      if (ee != cudaSuccess) return fail(st, STAGE_E_CUDA, cuda_msg("repack", ee));
      if ((ee = cudaDeviceSynchronize()) != cudaSuccess) return fail(st, STAGE_E_CUDA, cuda_msg("repack sync", ee));
      st->weight_bytes += pb;
      return STAGE_OK;
    };
    auto vec = [&](const stage_tensor* t, float** dst) -> stage_status {
      stage_status r;
      if ((r = dalloc_t(st, dst, t->bytes)) != STAGE_OK) return r;
      CK(cudaMemcpy(*dst, t->data, t->bytes, cudaMemcpyHostToDevice));
      return STAGE_OK;
    };
    if ((s = vec(T("norm1"), &L.norm1)) != STAGE_OK || (s = vec(T("norm2"), &L.norm2)) != STAGE_OK) return bail(s);
    if (L.attn) {
      L.in_rows = at_in;
      L.out_cols = at_o;
      if ((s = qmat(T("attn_in"), at_in, H, &L.w_in, &L.in_bytes)) != STAGE_OK) return bail(s);
      if ((s = qmat(T("attn_out"), H, at_o, &L.w_out, &L.out_bytes)) != STAGE_OK) return bail(s);
      if ((s = vec(T("attn_q_norm"), &L.qn)) != STAGE_OK || (s = vec(T("attn_k_norm"), &L.kn)) != STAGE_OK)
        return bail(s);
      if ((s = dalloc_t(st, &L.K, kv_elems * 2)) != STAGE_OK || (s = dalloc_t(st, &L.V, kv_elems * 2)) != STAGE_OK)
        return bail(s);
      if ((e = cudaMemset(L.K, 0, kv_elems * 2)) != cudaSuccess || (e = cudaMemset(L.V, 0, kv_elems * 2)) != cudaSuccess)
        return bail(fail(st, STAGE_E_CUDA, cuda_msg("cudaMemset", e)));
    } else {
      L.in_rows = dn_in;
      L.out_cols = dn_o;
      if ((s = qmat(T("dn_in"), dn_in, H, &L.w_in, &L.in_bytes)) != STAGE_OK) return bail(s);
      if ((s = qmat(T("dn_out"), H, dn_o, &L.w_out, &L.out_bytes)) != STAGE_OK) return bail(s);
      const size_t rb = (size_t)kRing * st->state_elems * 4;
      if ((s = dalloc_t(st, &L.ring, rb)) != STAGE_OK) return bail(s);
      if ((e = cudaMemset(L.ring, 0, rb)) != cudaSuccess) return bail(fail(st, STAGE_E_CUDA, cuda_msg("cudaMemset", e)));
      L.dn_slot = st->n_dn++;
    }
    L.in_tiles = packed_tiles(L.in_rows, false);
    {
      // gate and up, interleaved tile by tile for the SwiGLU epilogue
      const size_t pb = packed_bytes(qt, F, H, true);
      L.gu_bytes = pb;
      if ((s = dalloc_t(st, &L.w_gu, pb)) != STAGE_OK) return bail(s);
      if ((s = upload(st, stage_a, T("ffn_gate"))) != STAGE_OK) return bail(s);
      if ((s = upload(st, stage_b, T("ffn_up"))) != STAGE_OK) return bail(s);
      if ((e = launch_repack(qt, stage_a, stage_b, F, H, L.w_gu, nullptr)) != cudaSuccess ||
          (e = cudaDeviceSynchronize()) != cudaSuccess)
        return bail(fail(st, STAGE_E_CUDA, cuda_msg("repack gate/up", e)));
      st->weight_bytes += pb;
    }
    if ((s = qmat(T("ffn_down"), H, F, &L.w_down, &L.down_bytes)) != STAGE_OK) return bail(s);
    st->layers.push_back(L);
  }
  // staging no longer needed
  cudaFree(stage_a);
  cudaFree(stage_b);
  st->allocs.erase(std::remove_if(st->allocs.begin(), st->allocs.end(),
                                  [&](void* p) { return p == stage_a || p == stage_b; }),
                   st->allocs.end());

  // --- activations and scratch --------------------------------------------
  const int y_rows = std::max(dn_in, at_in);
  st->y_stride = (y_rows + 63) / 64 * 64;
  st->ss_stride = H / kTileRows;
  st->qz_stride = (int)qact_row_bytes(H);
  st->qo_stride = (int)qact_row_bytes(std::max(dn_o, at_o));
  st->qu_stride = (int)qact_row_bytes(F);
  if ((s = dalloc_t(st, &st->h, (size_t)kMaxTok * H * 4)) != STAGE_OK ||
      (s = dalloc_t(st, &st->ss, (size_t)kMaxTok * st->ss_stride * 4)) != STAGE_OK ||
      (s = dalloc_t(st, &st->y, (size_t)kMaxTok * st->y_stride * 4)) != STAGE_OK ||
      (s = dalloc_t(st, &st->qz, (size_t)kMaxTok * st->qz_stride)) != STAGE_OK ||
      (s = dalloc_t(st, &st->qo, (size_t)kMaxTok * st->qo_stride)) != STAGE_OK ||
      (s = dalloc_t(st, &st->qu, (size_t)kMaxTok * st->qu_stride)) != STAGE_OK)
    return bail(s);
  if (any_attn) {
    st->nchunk = (c.max_ctx + kAttChunk - 1) / kAttChunk;
    const size_t np = (size_t)kMaxTok * c.att_q_heads * st->nchunk;
    if ((s = dalloc_t(st, &st->pm, np * 4)) != STAGE_OK || (s = dalloc_t(st, &st->pl, np * 4)) != STAGE_OK ||
        (s = dalloc_t(st, &st->po, np * kAttDim * 4)) != STAGE_OK ||
        (s = dalloc_t(st, &st->rope, (size_t)c.max_ctx * (kRopeDims / 2) * sizeof(float2))) != STAGE_OK)
      return bail(s);
    if ((e = launch_rope_table(st->rope, c.max_ctx, c.rope_dims, c.rope_theta, nullptr)) != cudaSuccess)
      return bail(fail(st, STAGE_E_CUDA, cuda_msg("rope table", e)));
  }
  const int max_tiles = std::max({packed_tiles(y_rows, false), packed_tiles(F, true), H / kTileRows});
  st->max_tiles = max_tiles;
  if ((s = dalloc_t(st, &st->partials, (size_t)2 * st->sms * kMaxTok * kTileRows * 4)) != STAGE_OK ||
      (s = dalloc_t(st, &st->counters, (size_t)max_tiles * 4)) != STAGE_OK ||
      (s = dalloc_t(st, &st->err, 16)) != STAGE_OK ||
      (s = dalloc_t(st, &st->ctrl, (size_t)(1 + st->n_dn) * 4)) != STAGE_OK)
    return bail(s);
  if ((e = cudaMemset(st->counters, 0, (size_t)max_tiles * 4)) != cudaSuccess ||
      (e = cudaMemset(st->err, 0, 16)) != cudaSuccess ||
      (e = cudaMemset(st->ctrl, 0, (size_t)(1 + st->n_dn) * 4)) != cudaSuccess ||
      (e = cudaMemset(st->h, 0, (size_t)kMaxTok * H * 4)) != cudaSuccess)
    return bail(fail(st, STAGE_E_CUDA, cuda_msg("cudaMemset", e)));
  st->cur.assign(st->n_dn, 0);

  // --- persistent pass: step arguments of every layer, phase numbering -------
  if ((e = pass_prepare(qt)) != cudaSuccess) return bail(fail(st, STAGE_E_CUDA, cuda_msg("pass_prepare", e)));
  {
    std::vector<PassLayer> pl(st->layers.size());
    int phase = 1;   // phase 0: stage input
    for (size_t i = 0; i < pl.size(); ++i) {
      pl[i] = layer_args(st, i);
      pl[i].phase_in = phase;
      phase += pl[i].attn ? 6 : 5;   // in-proj, mixer (attention: partials + combine), out, gate/up, down
    }
    st->n_phases = phase;
    if ((s = dalloc_t(st, &st->pass_layers, pl.size() * sizeof(PassLayer))) != STAGE_OK ||
        (s = dalloc_t(st, &st->bar, 16)) != STAGE_OK)
      return bail(s);
    if ((e = cudaMemcpy(st->pass_layers, pl.data(), pl.size() * sizeof(PassLayer), cudaMemcpyHostToDevice)) !=
        cudaSuccess)
      return bail(fail(st, STAGE_E_CUDA, cuda_msg("cudaMemcpy pass layers", e)));
  }
  if ((e = cudaDeviceSynchronize()) != cudaSuccess) return bail(fail(st, STAGE_E_CUDA, cuda_msg("load sync", e)));
  *out = st;
  return STAGE_OK;
}

// Checks shared by both forward entries; builds the n_tok graph on first use.
static stage_status forward_begin(stage_t* st, const void* hidden_dev, int n_tok, int pos, int kind = DN_SNAPSHOTS) {
  if (!st) return STAGE_E_ARG;
  if (!hidden_dev) return fail(st, STAGE_E_ARG, "hidden buffer is NULL");
  if (n_tok < 1 || n_tok > kMaxTok) return fail(st, STAGE_E_ARG, "n_tok must be in 1..16");
  if (st->pending_n) return fail(st, STAGE_E_STATE, "a pass is pending: commit or roll back first");
  if (pos != st->committed) return fail(st, STAGE_E_STATE, "pos must equal the committed length");
  if (pos + n_tok > st->cfg.max_ctx) return fail(st, STAGE_E_ARG, "pass would overflow max_ctx");
  if (!st->exec[kind][n_tok]) return build_graph(st, n_tok, kind);
  return STAGE_OK;
}

stage_status stage_forward(stage_t* st, float* hidden_dev, int n_tok, int pos) {
  stage_status s = forward_begin(st, hidden_dev, n_tok, pos);
  if (s != STAGE_OK) return s;
  const size_t bytes = (size_t)n_tok * st->cfg.hidden * 4;
  CK(cudaMemcpyAsync(st->h, hidden_dev, bytes, cudaMemcpyDeviceToDevice, st->stream));
  CK(cudaGraphLaunch(st->exec[DN_SNAPSHOTS][n_tok], st->stream));
  CK(cudaMemcpyAsync(hidden_dev, st->h, bytes, cudaMemcpyDeviceToDevice, st->stream));
  st->pending_n = n_tok;
  st->pending_pos = pos;
  return STAGE_OK;
}

stage_status stage_forward_host(stage_t* st, const float* hidden_in_host, float* hidden_out_host, int n_tok,
                                int pos) {
  if (st && !hidden_out_host) return fail(st, STAGE_E_ARG, "hidden_out_host is NULL");
  stage_status s = forward_begin(st, hidden_in_host, n_tok, pos);
  if (s != STAGE_OK) return s;
  const size_t bytes = (size_t)n_tok * st->cfg.hidden * 4;
  CK(cudaMemcpyAsync(st->h, hidden_in_host, bytes, cudaMemcpyHostToDevice, st->stream));
  CK(cudaGraphLaunch(st->exec[DN_SNAPSHOTS][n_tok], st->stream));
  CK(cudaMemcpyAsync(hidden_out_host, st->h, bytes, cudaMemcpyDeviceToHost, st->stream));
  st->pending_n = n_tok;
  st->pending_pos = pos;
  return STAGE_OK;
}

stage_status stage_forward_f16(stage_t* st, void* hidden_dev, int n_tok, int pos) {
  if (st && reinterpret_cast<uintptr_t>(hidden_dev) % 2) return fail(st, STAGE_E_ARG, "hidden_dev must be 2-byte aligned");
  stage_status s = forward_begin(st, hidden_dev, n_tok, pos);
  if (s != STAGE_OK) return s;
  const int n = n_tok * st->cfg.hidden;
  CK(launch_hidden_from_f16(hidden_dev, st->h, n, st->stream));
  CK(cudaGraphLaunch(st->exec[DN_SNAPSHOTS][n_tok], st->stream));
  CK(launch_hidden_to_f16(st->h, hidden_dev, n, st->stream));
  st->pending_n = n_tok;
  st->pending_pos = pos;
  return STAGE_OK;
}

stage_status stage_prefill(stage_t* st, float* hidden_dev, int n_tok, int pos, int mode) {
  if (st && mode != STAGE_PREFILL_EXACT && mode != STAGE_PREFILL_CHUNKED)
    return fail(st, STAGE_E_ARG, "mode must be STAGE_PREFILL_EXACT or STAGE_PREFILL_CHUNKED");
  const int kind = mode == STAGE_PREFILL_CHUNKED ? DN_CHUNKED : DN_FINAL;
  stage_status s = forward_begin(st, hidden_dev, n_tok, pos, kind);
  if (s != STAGE_OK) return s;
  const size_t bytes = (size_t)n_tok * st->cfg.hidden * 4;
  CK(cudaMemcpyAsync(st->h, hidden_dev, bytes, cudaMemcpyDeviceToDevice, st->stream));
  CK(cudaGraphLaunch(st->exec[kind][n_tok], st->stream));
  CK(cudaMemcpyAsync(hidden_dev, st->h, bytes, cudaMemcpyDeviceToDevice, st->stream));
  // the chunk is committed whole: each DeltaNet layer's final state sits in
  // ring slot (cur + n_tok), the slot commit(n_tok) selects
  CK(launch_commit(st->ctrl, n_tok, st->n_dn, kRing, st->stream));
  st->committed = pos + n_tok;
  for (int& v : st->cur) v = (v + n_tok) % kRing;
  return STAGE_OK;
}

stage_status stage_commit(stage_t* st, int n_accepted) {
  if (!st) return STAGE_E_ARG;
  if (!st->pending_n) return fail(st, STAGE_E_STATE, "no pending pass");
  if (n_accepted < 0 || n_accepted > st->pending_n) return fail(st, STAGE_E_ARG, "n_accepted out of range");
  if (n_accepted > 0) CK(launch_commit(st->ctrl, n_accepted, st->n_dn, kRing, st->stream));
  st->committed = st->pending_pos + n_accepted;
  for (int& v : st->cur) v = (v + n_accepted) % kRing;
  st->pending_n = 0;
  return STAGE_OK;
}

stage_status stage_rollback(stage_t* st) { return stage_commit(st, 0); }

stage_status stage_reset(stage_t* st) {
  if (!st) return STAGE_E_ARG;
  if (st->pending_n) return fail(st, STAGE_E_STATE, "a pass is pending");
  CK(cudaMemsetAsync(st->ctrl, 0, (size_t)(1 + st->n_dn) * 4, st->stream));
  for (const Layer& L : st->layers)
    if (!L.attn) CK(cudaMemsetAsync(L.ring, 0, (size_t)st->state_elems * 4, st->stream));
  st->committed = 0;
  std::fill(st->cur.begin(), st->cur.end(), 0);
  return STAGE_OK;
}

stage_status stage_sync(stage_t* st) {
  if (!st) return STAGE_E_ARG;
  CK(cudaStreamSynchronize(st->stream));
  unsigned err = 0;
  CK(cudaMemcpy(&err, st->err, sizeof(err), cudaMemcpyDeviceToHost));
  if (err) {
    // a kernel that gave up may have left stream-K tile counters part-way:
    // clear them with the error word, so the next pass starts clean
    CK(cudaMemset(st->err, 0, sizeof(err)));
    CK(cudaMemset(st->counters, 0, (size_t)st->max_tiles * sizeof(int)));
    return fail(st, STAGE_E_DEVICE, "device error word " + std::to_string(err) + " (bounded wait timed out)");
  }
  return STAGE_OK;
}

int stage_committed_len(const stage_t* st) { return st ? st->committed : -1; }
int stage_pending(const stage_t* st) { return st ? st->pending_n : -1; }

static stage_status dn_state_io(stage_t* st, int layer, void* host, size_t bytes, bool to_host) {
  if (!st) return STAGE_E_ARG;
  const Layer* L = find_layer(st, layer);
  if (!L || L->attn) return fail(st, STAGE_E_ARG, "not a DeltaNet layer of this stage");
  if (!host || bytes != (size_t)st->state_elems * 4) return fail(st, STAGE_E_ARG, "bad buffer or size");
  if (st->pending_n) return fail(st, STAGE_E_STATE, "a pass is pending");
  CK(cudaStreamSynchronize(st->stream));
  float* dev = L->ring + (size_t)st->cur[L->dn_slot] * st->state_elems;
  if (to_host)
    CK(cudaMemcpy(host, dev, bytes, cudaMemcpyDeviceToHost));
  else
    CK(cudaMemcpy(dev, host, bytes, cudaMemcpyHostToDevice));
  return STAGE_OK;
}

stage_status stage_get_dn_state(stage_t* st, int layer, float* host_dst, size_t bytes) {
  return dn_state_io(st, layer, host_dst, bytes, true);
}
stage_status stage_set_dn_state(stage_t* st, int layer, const float* host_src, size_t bytes) {
  return dn_state_io(st, layer, const_cast<float*>(host_src), bytes, false);
}

static stage_status kv_io(stage_t* st, int layer, uint16_t* k, uint16_t* v, size_t bytes, bool to_host) {
  if (!st) return STAGE_E_ARG;
  const Layer* L = find_layer(st, layer);
  if (!L || !L->attn) return fail(st, STAGE_E_ARG, "not an attention layer of this stage");
  const size_t need = (size_t)st->cfg.att_kv_heads * st->cfg.max_ctx * kAttDim * 2;
  if (!k || !v || bytes != need) return fail(st, STAGE_E_ARG, "bad buffer or size");
  if (st->pending_n) return fail(st, STAGE_E_STATE, "a pass is pending");
  CK(cudaStreamSynchronize(st->stream));
  if (to_host) {
    CK(cudaMemcpy(k, L->K, bytes, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(v, L->V, bytes, cudaMemcpyDeviceToHost));
  } else {
    CK(cudaMemcpy(L->K, k, bytes, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(L->V, v, bytes, cudaMemcpyHostToDevice));
  }
  return STAGE_OK;
}

stage_status stage_get_kv(stage_t* st, int layer, uint16_t* k_host, uint16_t* v_host, size_t bytes_each) {
  return kv_io(st, layer, k_host, v_host, bytes_each, true);
}
stage_status stage_set_kv(stage_t* st, int layer, const uint16_t* k_host, const uint16_t* v_host, size_t bytes_each) {
  return kv_io(st, layer, const_cast<uint16_t*>(k_host), const_cast<uint16_t*>(v_host), bytes_each, false);
}

stage_status stage_set_kv_len(stage_t* st, int kv_len) {
  if (!st) return STAGE_E_ARG;
  if (kv_len < 0 || kv_len >= st->cfg.max_ctx) return fail(st, STAGE_E_ARG, "kv_len out of range");
  if (st->pending_n) return fail(st, STAGE_E_STATE, "a pass is pending");
  CK(launch_set_int(st->ctrl, kv_len, st->stream));
  CK(cudaStreamSynchronize(st->stream));
  st->committed = kv_len;
  return STAGE_OK;
}

stage_status stage_debug_dequant(stage_t* st, const char* tensor, int row, float* host_dst, size_t dst_elems) {
  if (!st) return STAGE_E_ARG;
  int layer;
  std::string tag;
  if (!host_dst || !parse_name(tensor, &layer, &tag)) return fail(st, STAGE_E_ARG, "bad tensor name or buffer");
  const Layer* L = find_layer(st, layer);
  if (!L) return fail(st, STAGE_E_ARG, "layer not in this stage");
  const int H = st->cfg.hidden, F = st->cfg.ffn;
  const uint8_t* P = nullptr;
  int rows = 0, cols = 0, paired = 0, r = row;
  if ((tag == "dn_in" && !L->attn) || (tag == "attn_in" && L->attn)) {
    P = L->w_in; rows = L->in_rows; cols = H;
  } else if ((tag == "dn_out" && !L->attn) || (tag == "attn_out" && L->attn)) {
    P = L->w_out; rows = H; cols = L->out_cols;
  } else if (tag == "ffn_gate" || tag == "ffn_up") {
    P = L->w_gu; rows = F; cols = H; paired = 1;
    if (tag == "ffn_up") r = row + F;
  } else if (tag == "ffn_down") {
    P = L->w_down; rows = H; cols = F;
  } else {
    return fail(st, STAGE_E_ARG, "not a quantised tensor of this layer");
  }
  if (row < 0 || row >= rows) return fail(st, STAGE_E_ARG, "row out of range");
  if (dst_elems < (size_t)cols)
    return fail(st, STAGE_E_ARG, "host_dst holds " + std::to_string(dst_elems) + " floats; the row has " +
                                     std::to_string(cols));
  float* tmp = nullptr;
  cudaError_t e = cudaMalloc(&tmp, (size_t)cols * 4);
  if (e != cudaSuccess) return fail(st, STAGE_E_OOM, cuda_msg("cudaMalloc", e));
  e = launch_dequant(st->cfg.qtype, P, rows, cols, paired, r, 1, tmp, st->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st->stream);
  if (e == cudaSuccess) e = cudaMemcpy(host_dst, tmp, (size_t)cols * 4, cudaMemcpyDeviceToHost);
  cudaFree(tmp);
  if (e != cudaSuccess) return fail(st, STAGE_E_CUDA, cuda_msg("dequant", e));
  return STAGE_OK;
}

// Drop every recorded graph (the next forward of each token count records
// it again with the current settings).
static stage_status drop_graphs(stage_t* st) {
  CK(cudaStreamSynchronize(st->stream));
  for (auto& row : st->exec)
    for (auto& g : row)
      if (g) {
        CK(cudaGraphExecDestroy(g));
        g = nullptr;
      }
  return STAGE_OK;
}

stage_status stage_set_pass_mode(stage_t* st, int mode) {
  if (!st) return STAGE_E_ARG;
  if (mode != STAGE_PASS_KERNELS && mode != STAGE_PASS_PERSISTENT) return fail(st, STAGE_E_ARG, "unknown pass mode");
  if (st->pending_n) return fail(st, STAGE_E_STATE, "a pass is pending");
  if (mode == st->pass_mode) return STAGE_OK;
  stage_status s = drop_graphs(st);
  if (s != STAGE_OK) return s;
  st->pass_mode = mode;
  return STAGE_OK;
}

int stage_pass_persistent(stage_t* st, int n_tok) {
  if (!st || n_tok < 1 || n_tok > kMaxTok) return -1;
  return st->pass_mode == STAGE_PASS_PERSISTENT && st->dbg_fault_item < 0 && pass_eligible(st, n_tok) ? 1 : 0;
}

stage_status stage_debug_inject(stage_t* st, int fault_item, unsigned wait_limit) {
  if (!st) return STAGE_E_ARG;
  if (st->pending_n) return fail(st, STAGE_E_STATE, "a pass is pending");
  if (fault_item < -1) return fail(st, STAGE_E_ARG, "fault_item must be -1 or a local item index");
  stage_status s = drop_graphs(st);
  if (s != STAGE_OK) return s;
  st->dbg_fault_item = fault_item;
  st->dbg_wait_limit = wait_limit;
  return STAGE_OK;
}

size_t stage_weight_bytes(const stage_t* st) { return st ? st->weight_bytes : 0; }

const char* stage_last_error(const stage_t* st) { return st ? st->last_error.c_str() : "null stage"; }

void stage_free(stage_t* st) { destroy(st); }

}  // extern "C"

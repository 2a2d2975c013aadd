// Kernel-level C entry points (qhl_*): one hot-path kernel per call, no stage.
#include <cuda_runtime.h>

#include <atomic>
#include <deque>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/qhl_stage.h"
#include "launch.h"

using namespace qhl;

namespace qhl {
thread_local std::string g_last_error;
void set_last_error(const std::string& s) { g_last_error = s; }
unsigned noalloc_take_error(int dev);   // noalloc.cu: read and clear the static scratch's error word
}  // namespace qhl

namespace {

int err(int code, const std::string& msg) {
  set_last_error(msg);
  return code;
}

int cuda_err(const char* what, cudaError_t e) {
  return err(STAGE_E_CUDA, std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
}

// Per-device scratch of qhl_qgemv: the input in block fixed point, stream-K
// partials for up to 16 tokens and one counter per tile, allocated on first
// use and grown on demand.  Entries live in a deque, so a pointer to one stays
// valid while another host thread adds a device.
struct GemvScratch {
  bool ready = false;
  int sms = 0;
  uint8_t* qx = nullptr;
  size_t qx_cap = 0;
  float* partials = nullptr;
  int* counters = nullptr;
  int counter_cap = 0;
  unsigned* err = nullptr;
  bool prepared[9] = {};
};
std::mutex g_mu;
std::deque<GemvScratch> g_scratch;

// Failure injection for qhl_qgemv (qhl_debug_inject): applies to later calls.
std::atomic<int> g_fault_item{-1};
std::atomic<unsigned> g_wait_limit{0};

// What one call needs from the scratch, copied out under the lock.
struct ScratchView {
  int sms;
  uint8_t* qx;
  float* partials;
  int* counters;
  unsigned* err;
};

int get_scratch(int tiles, int qt, size_t qx_bytes, ScratchView* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err("cudaGetDevice", e);
  std::lock_guard<std::mutex> lk(g_mu);
  if ((int)g_scratch.size() <= dev) g_scratch.resize(dev + 1);
  GemvScratch& s = g_scratch[dev];
  if (!s.ready) {
    if ((e = cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_err("cudaDeviceGetAttribute", e);
    if ((e = cudaMalloc(&s.partials, (size_t)2 * s.sms * 16 * kTileRows * 4)) != cudaSuccess)
      return cuda_err("cudaMalloc", e);
    if ((e = cudaMalloc(&s.err, 16)) != cudaSuccess) return cuda_err("cudaMalloc", e);
    if ((e = cudaMemset(s.err, 0, 16)) != cudaSuccess) return cuda_err("cudaMemset", e);
    s.ready = true;
  }
  if (tiles > s.counter_cap) {
    int* c = nullptr;
    if ((e = cudaMalloc(&c, (size_t)tiles * 4)) != cudaSuccess) return cuda_err("cudaMalloc", e);
    if ((e = cudaMemset(c, 0, (size_t)tiles * 4)) != cudaSuccess) return cuda_err("cudaMemset", e);
    if (s.counters) {
      cudaDeviceSynchronize();
      cudaFree(s.counters);
    }
    s.counters = c;
    s.counter_cap = tiles;
  }
  if (qx_bytes > s.qx_cap) {
    uint8_t* q = nullptr;
    if ((e = cudaMalloc(&q, qx_bytes)) != cudaSuccess) return cuda_err("cudaMalloc", e);
    if ((e = cudaMemset(q, 0, qx_bytes)) != cudaSuccess) return cuda_err("cudaMemset", e);
    if (s.qx) {
      cudaDeviceSynchronize();
      cudaFree(s.qx);
    }
    s.qx = q;
    s.qx_cap = qx_bytes;
  }
  if (!s.prepared[qt]) {
    if ((e = gemv_prepare(qt)) != cudaSuccess) return cuda_err("gemv_prepare", e);
    s.prepared[qt] = true;
  }
  *out = ScratchView{s.sms, s.qx, s.partials, s.counters, s.err};
  return 0;
}

bool valid_qt(int qt) { return qt == kQ4_0 || qt == kQ8_0; }

}  // namespace

extern "C" {

size_t qhl_packed_bytes(int qtype, int rows, int cols, int paired) {
  if (!valid_qt(qtype)) return 0;
  return packed_bytes(qtype, rows, cols, paired != 0);
}

int qhl_repack(int qtype, int rows, int cols, const void* gguf_dev, const void* gguf_b_dev, void* packed_dev,
               void* stream) {
  if (!valid_qt(qtype) || !gguf_dev || !packed_dev || rows <= 0 || cols <= 0 || cols % kChunkCols)
    return err(STAGE_E_ARG, "qhl_repack: bad argument");
  if (reinterpret_cast<uintptr_t>(packed_dev) % 16) return err(STAGE_E_ARG, "qhl_repack: packed_dev not 16-byte aligned");
  cudaError_t e = launch_repack(qtype, static_cast<const uint8_t*>(gguf_dev), static_cast<const uint8_t*>(gguf_b_dev),
                                rows, cols, static_cast<uint8_t*>(packed_dev), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? 0 : cuda_err("repack", e);
}

int qhl_dequant(int qtype, int rows, int cols, const void* packed_dev, int paired, int row0, int nrows,
                float* out_dev, void* stream) {
  const int total = paired ? 2 * rows : rows;
  if (!valid_qt(qtype) || !packed_dev || !out_dev || rows <= 0 || cols <= 0 || cols % kChunkCols || row0 < 0 ||
      nrows < 0 || row0 + nrows > total)
    return err(STAGE_E_ARG, "qhl_dequant: bad argument");
  if (reinterpret_cast<uintptr_t>(packed_dev) % 16) return err(STAGE_E_ARG, "qhl_dequant: packed_dev not 16-byte aligned");
  cudaError_t e = launch_dequant(qtype, static_cast<const uint8_t*>(packed_dev), rows, cols, paired ? 1 : 0, row0,
                                 nrows, out_dev, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? 0 : cuda_err("dequant", e);
}

int qhl_qgemv(int qtype, int rows, int cols, const void* packed_dev, const float* x_dev, int n_tok, float* y_dev,
              void* stream) {
  if (!valid_qt(qtype) || !packed_dev || !x_dev || !y_dev || rows <= 0 || cols <= 0 || cols % kChunkCols ||
      n_tok < 1 || n_tok > 16)
    return err(STAGE_E_ARG, "qhl_qgemv: bad argument");
  if (reinterpret_cast<uintptr_t>(packed_dev) % 16 || reinterpret_cast<uintptr_t>(x_dev) % 16)
    return err(STAGE_E_ARG, "qhl_qgemv: packed_dev and x_dev must be 16-byte aligned");
  if ((long long)packed_tiles(rows, false) * (cols / kChunkCols) >= (1LL << 31))
    return err(STAGE_E_ARG, "qhl_qgemv: more than 2^31 - 1 packed items");
  const int tiles = packed_tiles(rows, false);
  ScratchView s;
  int rc = get_scratch(tiles, qtype, (size_t)n_tok * qact_row_bytes(cols), &s);
  if (rc) return rc;
  cudaError_t e = launch_quantize_rows(x_dev, n_tok, cols, s.qx, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_err("quantize launch", e);
  GemvArgs a = {};
  a.W = static_cast<const uint8_t*>(packed_dev);
  a.tiles = tiles;
  a.chunks = cols / kChunkCols;
  a.qx = s.qx;
  a.qx_stride = (int)qact_row_bytes(cols);
  a.y = y_dev;
  a.y_stride = rows;
  a.out_valid = rows;
  a.inv_dim = 1.f;
  a.eps = 0.f;
  a.partials = s.partials;
  a.counters = s.counters;
  a.err = s.err;
  a.workers = gemv_workers(a.tiles, a.chunks, s.sms);
  a.fault_item = g_fault_item.load();
  a.wait_limit = g_wait_limit.load();
  e = launch_gemv(qtype, n_tok, EPI_STORE, a, a.workers, static_cast<cudaStream_t>(stream), true);
  return e == cudaSuccess ? 0 : cuda_err("qgemv launch", e);
}

int qhl_deltanet_step(int Hk, int Hv, const float* y_dev, int n_tok, const float* s_in_dev, float* snaps_dev,
                      float* o_dev, void* stream) {
  if (Hk <= 0 || Hv <= 0 || Hv % Hk || !y_dev || !s_in_dev || !snaps_dev || !o_dev || n_tok < 1 || n_tok > 16)
    return err(STAGE_E_ARG, "qhl_deltanet_step: bad argument");
  if (reinterpret_cast<uintptr_t>(y_dev) % 16 || reinterpret_cast<uintptr_t>(s_in_dev) % 16 ||
      reinterpret_cast<uintptr_t>(snaps_dev) % 16)
    return err(STAGE_E_ARG, "qhl_deltanet_step: y_dev, s_in_dev and snaps_dev must be 16-byte aligned");
  DnArgs d = {};
  d.y = y_dev;
  d.y_stride = 2 * Hk * kDnDim + Hv * kDnDim + 2 * Hv;
  if (d.y_stride % 4) return err(STAGE_E_UNSUPPORTED, "qhl_deltanet_step: row width must be a multiple of 4");
  d.Hk = Hk;
  d.Hv = Hv;
  d.ring = snaps_dev;
  d.state_elems = (long long)Hv * kDnDim * kDnDim;
  d.ring_size = n_tok;
  d.cur = nullptr;
  d.s_in = s_in_dev;
  d.o = o_dev;
  d.o_stride = Hv * kDnDim;
  cudaError_t e = launch_dn_step(n_tok, d, Hv * (kDnDim / 32), static_cast<cudaStream_t>(stream), false);
  return e == cudaSuccess ? 0 : cuda_err("deltanet launch", e);
}

int qhl_debug_inject(int fault_item, unsigned wait_limit) {
  if (fault_item < -1) return err(STAGE_E_ARG, "qhl_debug_inject: fault_item must be -1 or a local item index");
  g_fault_item.store(fault_item);
  g_wait_limit.store(wait_limit);
  return 0;
}

int qhl_sync(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_err("cudaStreamSynchronize", e);
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_err("cudaGetDevice", e);
  unsigned word = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if ((int)g_scratch.size() > dev && g_scratch[dev].ready) {
      GemvScratch& s = g_scratch[dev];
      unsigned w = 0;
      if ((e = cudaMemcpy(&w, s.err, sizeof(w), cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_err("cudaMemcpy", e);
      if (w) {
        // a kernel that gave up may have left tile counters part-way
        if ((e = cudaMemset(s.err, 0, sizeof(w))) != cudaSuccess) return cuda_err("cudaMemset", e);
        if (s.counters && (e = cudaMemset(s.counters, 0, (size_t)s.counter_cap * 4)) != cudaSuccess)
          return cuda_err("cudaMemset", e);
      }
      word |= w;
    }
  }
  word |= noalloc_take_error(dev);
  if (word) return err(STAGE_E_DEVICE, "device error word " + std::to_string(word) + " (bounded wait timed out)");
  return 0;
}

const char* qhl_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"

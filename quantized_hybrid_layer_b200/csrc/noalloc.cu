// qhl_qgemv_noalloc: the quantised GEMV without any device allocation.
//
// Some callers cannot allocate device memory when they call the GEMV: a
// process whose memory pool already owns the whole GPU (a framework's caching
// allocator that has reserved everything), or a latency-critical loop that
// must not pay for cudaMalloc / cudaFree, which can synchronise the device.
// qhl_qgemv allocates its scratch (the stream-K partial sums, the tile
// counters and the input in block fixed point) on first use and grows it on
// demand; this variant keeps that scratch in one file-scope device array whose
// size is fixed when the library is loaded, so a call never allocates.
//
// The array lives on every GPU that loads the library until the process
// exits.  Its size bounds the problems this entry point accepts (see
// qhl_stage.h); larger ones are rejected before any device work.
#include <cuda_runtime.h>

#include <deque>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/qhl_stage.h"
#include "launch.h"

using namespace qhl;

namespace qhl {
void set_last_error(const std::string& s);   // kernel_abi.cu
}

namespace {

// Regions of the scratch array (bytes).
constexpr size_t kPartialBytes = (size_t)5 << 19;     // 2.5 MiB: 2 * SMs * 16 tokens * 128 rows f32, SMs <= 160
constexpr size_t kCounterBytes = (size_t)64 << 10;    // 64 KiB: one int per 128-row tile (16384 tiles)
constexpr size_t kQxBytes = (size_t)9 << 18;          // 2.25 MiB: the input in block fixed point
constexpr size_t kErrBytes = 256;
constexpr size_t kScratchBytes = kPartialBytes + kCounterBytes + kQxBytes + kErrBytes;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

struct DeviceScratch {
  bool ready = false;
  unsigned char* base = nullptr;   // device address of g_scratch on this device
  int sms = 0;
  bool prepared[9] = {};
};

// Entries live in a deque: references to one stay valid while another host
// thread adds a device.  Callers still copy what they need under the lock.
std::mutex g_mu;
std::deque<DeviceScratch> g_dev;

int fail(int code, const std::string& msg) {
  set_last_error("qhl_qgemv_noalloc: " + msg);
  return code;
}

}  // namespace

extern "C" int qhl_qgemv_noalloc(int qtype, int rows, int cols, const void* packed_dev, const float* x_dev, int n_tok,
                                 float* y_dev, void* stream) {
  if ((qtype != kQ4_0 && qtype != kQ8_0) || !packed_dev || !x_dev || !y_dev || rows <= 0 || cols <= 0 ||
      cols % kChunkCols || n_tok < 1 || n_tok > 16)
    return fail(STAGE_E_ARG, "bad argument");
  if (reinterpret_cast<uintptr_t>(packed_dev) % 16 || reinterpret_cast<uintptr_t>(x_dev) % 16)
    return fail(STAGE_E_ARG, "packed_dev and x_dev must be 16-byte aligned");
  if ((long long)packed_tiles(rows, false) * (cols / kChunkCols) >= (1LL << 31))
    return fail(STAGE_E_ARG, "more than 2^31 - 1 packed items");
  const int tiles = packed_tiles(rows, false);
  const size_t qx_bytes = (size_t)n_tok * qact_row_bytes(cols);
  if (qx_bytes > kQxBytes)
    return fail(STAGE_E_ARG, "n_tok * cols/256 * 2048 = " + std::to_string(qx_bytes) + " bytes exceeds the " +
                                 std::to_string(kQxBytes) + "-byte input region of the static scratch");
  if ((size_t)tiles * sizeof(int) > kCounterBytes)
    return fail(STAGE_E_ARG, "rows exceed the static scratch's tile counters (at most " +
                                 std::to_string(kCounterBytes / sizeof(int) * kTileRows) + " rows)");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(STAGE_E_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  unsigned char* base = nullptr;
  int sms = 0;
  {
    // once per device, with that device current: the scratch array's device
    // address (a host-side use of g_scratch would be a host stand-in, not it)
    std::lock_guard<std::mutex> lk(g_mu);
    if ((int)g_dev.size() <= dev) g_dev.resize(dev + 1);
    DeviceScratch& ds = g_dev[dev];
    if (!ds.ready) {
      void* p = nullptr;
      if ((e = cudaGetSymbolAddress(&p, g_scratch)) != cudaSuccess)
        return fail(STAGE_E_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      if ((e = cudaDeviceGetAttribute(&ds.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return fail(STAGE_E_CUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
      ds.base = static_cast<unsigned char*>(p);
      ds.ready = true;
    }
    if (!ds.prepared[qtype]) {
      if ((e = gemv_prepare(qtype)) != cudaSuccess)
        return fail(STAGE_E_CUDA, std::string("gemv_prepare: ") + cudaGetErrorString(e));
      ds.prepared[qtype] = true;
    }
    base = ds.base;
    sms = ds.sms;
  }
  if ((size_t)2 * sms * 16 * kTileRows * sizeof(float) > kPartialBytes)
    return fail(STAGE_E_UNSUPPORTED, "this device has more SMs than the static stream-K region holds");

  float* partials = reinterpret_cast<float*>(base);
  int* counters = reinterpret_cast<int*>(base + kPartialBytes);
  uint8_t* qx = base + kPartialBytes + kCounterBytes;
  unsigned* err = reinterpret_cast<unsigned*>(base + kPartialBytes + kCounterBytes + kQxBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // the array keeps the previous call's contents: the tile counters must start at zero
  if ((e = cudaMemsetAsync(counters, 0, (size_t)tiles * sizeof(int), s)) != cudaSuccess)
    return fail(STAGE_E_CUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));
  if ((e = launch_quantize_rows(x_dev, n_tok, cols, qx, s)) != cudaSuccess)
    return fail(STAGE_E_CUDA, std::string("quantize launch: ") + cudaGetErrorString(e));
  GemvArgs a = {};
  a.W = static_cast<const uint8_t*>(packed_dev);
  a.tiles = tiles;
  a.chunks = cols / kChunkCols;
  a.qx = qx;
  a.qx_stride = (int)qact_row_bytes(cols);
  a.y = y_dev;
  a.y_stride = rows;
  a.out_valid = rows;
  a.inv_dim = 1.f;
  a.partials = partials;
  a.counters = counters;
  a.err = err;
  a.workers = gemv_workers(a.tiles, a.chunks, sms);
  a.fault_item = -1;
  if ((e = launch_gemv(qtype, n_tok, EPI_STORE, a, a.workers, s, true)) != cudaSuccess)
    return fail(STAGE_E_CUDA, std::string("qgemv launch: ") + cudaGetErrorString(e));
  return 0;
}

namespace qhl {
// The static scratch's error word on device `dev` (current), read and cleared
// with the tile counters; 0 if the array was never used there.  For qhl_sync.
unsigned noalloc_take_error(int dev) {
  unsigned char* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if ((int)g_dev.size() > dev && g_dev[dev].ready) base = g_dev[dev].base;
  }
  if (!base) return 0;
  unsigned* err = reinterpret_cast<unsigned*>(base + kPartialBytes + kCounterBytes + kQxBytes);
  unsigned w = 0;
  if (cudaMemcpy(&w, err, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return 0;
  if (w) {
    cudaMemset(err, 0, sizeof(w));
    cudaMemset(base + kPartialBytes, 0, kCounterBytes);
  }
  return w;
}
}  // namespace qhl

// Instantiations and launch of the persistent pass (pass.cuh): both weight
// types, n_tok 1..kPassMaxTok.
#include "launch.h"

namespace qhl {
namespace {

template <int QT, int NT>
cudaError_t prep_one() {
  cudaError_t e = cudaFuncSetAttribute(stage_pass_kernel<QT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       pass_smem_bytes<QT, NT>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(stage_pass_kernel<QT, NT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  return e;
}

template <int QT, int NT>
cudaError_t occupancy_one(int* blocks) {
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, stage_pass_kernel<QT, NT>, kPassThreads,
                                                       pass_smem_bytes<QT, NT>());
}

template <int QT, int NT>
cudaError_t launch_one(const PassArgs& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kPassThreads);
  cfg.dynamicSmemBytes = pass_smem_bytes<QT, NT>();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA co-resident: the phase counter relies on it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stage_pass_kernel<QT, NT>, p);
}

#define QHL_PASS_CASES(X) X(1) X(2) X(3) X(4)

template <int QT>
cudaError_t prepare_qt() {
  cudaError_t e = cudaSuccess;
#define P(N) if (e == cudaSuccess) e = prep_one<QT, N>();
  QHL_PASS_CASES(P)
#undef P
  return e;
}

}  // namespace

cudaError_t pass_prepare(int qt) {
  if (qt == kQ4_0) return prepare_qt<kQ4_0>();
  if (qt == kQ8_0) return prepare_qt<kQ8_0>();
  return cudaErrorInvalidValue;
}

cudaError_t pass_occupancy(int qt, int nt, int* blocks) {
  *blocks = 0;
  switch (qt * 100 + nt) {
#define C(N)                                               \
  case kQ4_0 * 100 + N: return occupancy_one<kQ4_0, N>(blocks); \
  case kQ8_0 * 100 + N: return occupancy_one<kQ8_0, N>(blocks);
    QHL_PASS_CASES(C)
#undef C
    default: return cudaSuccess;
  }
}

cudaError_t launch_pass(int qt, int nt, const PassArgs& p, cudaStream_t s) {
  switch (qt * 100 + nt) {
#define C(N)                                            \
  case kQ4_0 * 100 + N: return launch_one<kQ4_0, N>(p, s); \
  case kQ8_0 * 100 + N: return launch_one<kQ8_0, N>(p, s);
    QHL_PASS_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qhl

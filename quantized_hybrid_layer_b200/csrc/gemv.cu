// Instantiations and launch dispatch of the dequant-GEMV: both weight types,
// NT = 1..16, three epilogues, one translation unit.
#include "launch.h"

namespace qhl {
namespace {

template <int QT, int NT, int EPI>
cudaError_t one(const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_ex(qgemv_kernel<QT, NT, EPI>, dim3(grid), dim3(GemvCfg<QT, NT>::kThreads), (size_t)gemv_smem_bytes<QT, NT>(), s,
                   pdl, a);
}

// Every stage kernel asks for the full shared-memory carveout, so consecutive
// kernels never need the SM reconfigured and can share it under programmatic
// dependent launch.
template <typename K>
cudaError_t set_attrs(K k, int smem) {
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}

template <int QT, int NT>
cudaError_t prep() {
  const int smem = gemv_smem_bytes<QT, NT>();
  cudaError_t e = set_attrs(qgemv_kernel<QT, NT, EPI_STORE>, smem);
  if (e == cudaSuccess) e = set_attrs(qgemv_kernel<QT, NT, EPI_SWIGLU>, smem);
  if (e == cudaSuccess) e = set_attrs(qgemv_kernel<QT, NT, EPI_RESID>, smem);
  return e;
}

template <int QT, int NT>
cudaError_t by_epi(int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
  switch (epi) {
    case EPI_STORE: return one<QT, NT, EPI_STORE>(a, grid, s, pdl);
    case EPI_SWIGLU: return one<QT, NT, EPI_SWIGLU>(a, grid, s, pdl);
    case EPI_RESID: return one<QT, NT, EPI_RESID>(a, grid, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

#define QHL_NT_CASES(X) X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16)

template <int QT>
cudaError_t prepare_qt() {
  cudaError_t e = cudaSuccess;
#define P(N) if (e == cudaSuccess) e = prep<QT, N>();
  QHL_NT_CASES(P)
#undef P
  return e;
}

template <int QT>
cudaError_t launch_qt(int nt, int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
  switch (nt) {
#define C(N) case N: return by_epi<QT, N>(epi, a, grid, s, pdl);
    QHL_NT_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

template <int QT>
int smem_qt(int nt) {
  switch (nt) {
#define C(N) case N: return gemv_smem_bytes<QT, N>();
    QHL_NT_CASES(C)
#undef C
    default: return 0;
  }
}

}  // namespace

cudaError_t gemv_prepare(int qt) {
  if (qt == kQ4_0) return prepare_qt<kQ4_0>();
  if (qt == kQ8_0) return prepare_qt<kQ8_0>();
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemv(int qt, int nt, int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
  if (qt == kQ4_0) return launch_qt<kQ4_0>(nt, epi, a, grid, s, pdl);
  if (qt == kQ8_0) return launch_qt<kQ8_0>(nt, epi, a, grid, s, pdl);
  return cudaErrorInvalidValue;
}

int gemv_smem(int qt, int nt) { return qt == kQ4_0 ? smem_qt<kQ4_0>(nt) : (qt == kQ8_0 ? smem_qt<kQ8_0>(nt) : 0); }

}  // namespace qhl

// Instantiations of the dequant-GEMV for kQ4_0 (NT = 1..16, three epilogues).
#include "launch.h"

namespace qhl {
namespace {

// Every stage kernel asks for the full shared-memory carveout, so consecutive
// kernels never need the SM reconfigured and can share it under programmatic
// dependent launch.
template <typename K>
cudaError_t set_carveout(K k, cudaFuncAttribute, int smem) {
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}

template <int NT, int EPI>
cudaError_t one(const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
  return launch_ex(qgemv_kernel<kQ4_0, NT, EPI>, dim3(grid), dim3(kGemvCtaThreads),
                   (size_t)gemv_smem_bytes<kQ4_0, NT>(), s, pdl, a);
}

template <int NT>
cudaError_t prep() {
  const int smem = gemv_smem_bytes<kQ4_0, NT>();
  cudaError_t e = set_carveout(qgemv_kernel<kQ4_0, NT, EPI_STORE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = set_carveout(qgemv_kernel<kQ4_0, NT, EPI_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = set_carveout(qgemv_kernel<kQ4_0, NT, EPI_RESID>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}

template <int NT>
cudaError_t by_epi(int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
  switch (epi) {
    case EPI_STORE: return one<NT, EPI_STORE>(a, grid, s, pdl);
    case EPI_SWIGLU: return one<NT, EPI_SWIGLU>(a, grid, s, pdl);
    case EPI_RESID: return one<NT, EPI_RESID>(a, grid, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

#define QHL_NT_CASES(X) X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16)

cudaError_t gemv_prepare_4() {
  cudaError_t e = cudaSuccess;
#define P(N) if (e == cudaSuccess) e = prep<N>();
  QHL_NT_CASES(P)
#undef P
  return e;
}

cudaError_t launch_gemv_4(int nt, int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
  switch (nt) {
#define C(N) case N: return by_epi<N>(epi, a, grid, s, pdl);
    QHL_NT_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

int gemv_smem_4(int nt) {
  switch (nt) {
#define C(N) case N: return gemv_smem_bytes<kQ4_0, N>();
    QHL_NT_CASES(C)
#undef C
    default: return 0;
  }
}

}  // namespace qhl

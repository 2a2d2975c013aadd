// The whole layer-stage pass in one persistent, cooperative kernel.
//
// The pages submit one command buffer per token (SwarmLLM README, paragraph
// after the peer diagram); this takes that one step further on B200: instead
// of a chain of kernels (each paying launch, ramp-up and tail), one grid of
// two CTAs per SM runs every phase of the pass -- stage input, then per layer the mixer in-projection,
// the DeltaNet step or the attention partials + combine, the out-projection,
// gate/up and down -- separated by grid-wide barriers (a monotonic counter in
// global memory; every wait is bounded).
//
// Each CTA's producer warp knows the whole pass's weight schedule (the CTA's
// stream-K items of every projection, in order) and keeps the shared-memory
// ring full across phase boundaries: while the consumers wait at a barrier or
// run a mixer, the next projection's weights are already streaming in.  Only
// an item's x columns wait for the barrier that makes them ready (consumer
// thread 0 acquires the counter and hands the phase to the producer through
// shared memory; the producer fences the async proxy before the bulk copy).  Consumers run the same device functions as the separate kernels of
// the graph path (gemv_consume, dn_unit, attn_unit, combine_unit, input_unit)
// with the same stream-K split, so both paths give the same bits.  Data written
// earlier in the pass is read through L2 (ld.cg) or bulk copies, never L1.
#pragma once

#include "attention.cuh"
#include "deltanet.cuh"
#include "input.cuh"
#include "qgemv.cuh"

namespace qhl {

struct PassLayer {
  int attn;            // 1: full-attention layer, 0: gated DeltaNet
  int phase_in;        // phase index of the mixer in-projection
  GemvArgs g[4];       // in-projection, out-projection, gate/up, down
  DnArgs dn;
  AttnArgs at;
};

struct PassArgs {
  const PassLayer* layers;
  int n_layers;
  const float* h;      // stage input [NT][H]
  int H;
  const float* gamma0; // first layer's RMSNorm1 weight
  uint8_t* qz;
  int qz_stride;
  float* ss;
  int ss_stride;
  const int* kv_len;   // position of token 0
  unsigned* bar;       // grid barrier counter, zero at launch
  int grid;            // CTAs (all co-resident)
  int dn_units;        // Hv * 4
  int Hq, Hkv;
  unsigned* err;
  // optional phase trace, [grid][n_phases][2] global-timer ns: when this CTA's
  // consumers start the phase (past the barrier) and when they finish it
  unsigned long long* trace;
  int n_phases;
};

QHL_DEV unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Shared memory: the ring of item stages, then one scratch area shared by the
// mixer units (attention / combine / DeltaNet / stage input, used by the
// consumer warps during their phases) and the GEMV tile hand-off (reduction
// buffers + final tile, used during projection phases), then rstd, mbarriers
// and flags; within 113 KB so two CTAs share an SM.
template <int QT, int NT>
struct PassCfg {
  static constexpr int kIB = QLayout<QT>::kItemBytes;
  static constexpr int kSB = kIB + NT * kQChunkBytes;
  static constexpr int kMixUnits = 12 * 1024 + NT * 8 * 1024;
  static constexpr int kTileBytes = TileRing<NT>::kBytes + NT * 64 * 4;
  static constexpr int kMix = kMixUnits > kTileBytes ? kMixUnits : kTileBytes;
  static constexpr int kFixed = kMix + 16 * 4 + 2 * TileRing<NT>::kBufs * 8 + 16;
  static constexpr int kRaw = (113 * 1024 - kFixed) / (kSB + 16);
  static constexpr int kStages = kRaw > 16 ? 16 : kRaw;
  static constexpr int kMixOff = kStages * kSB;                     // 16-byte aligned: kSB is a multiple of 16
  static constexpr int kRstdOff = kMixOff + kMix;
  static constexpr int kBarOff = kRstdOff + 16 * 4;
  static constexpr int kFlagOff = kBarOff + (2 * kStages + 2 * TileRing<NT>::kBufs) * 8;
  static constexpr int kSmem = kFlagOff + 16;
  // A deep enough ring and two CTAs per SM (Q8_0 at 4 tokens does not fit:
  // that pass runs as separate kernels).
  static constexpr bool kFits = kRaw >= 3 && kSmem <= 113 * 1024;
};

// Token counts the persistent pass is instantiated for (two CTAs per SM fit).
constexpr int kPassMaxTok = 4;

QHL_DEV unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Order global data acquired through the generic proxy before later bulk
// copies (async proxy) that read it.
QHL_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
// Wait (suspended, at most about `ns` nanoseconds) for the phase with the
// given parity to complete; true once it has.
QHL_DEV bool mbar_wait_for(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Spin bound of every grid-barrier and ring wait (seconds: far beyond any
// legitimate wait, short of a hung GPU).
constexpr uint32_t kSpinLimit = 1u << 24;

// Grid-barrier arrival: add 1 with release semantics (the CTA's writes,
// ordered before this thread by the preceding barrier, become visible with it).
QHL_DEV void red_add_release(unsigned* p) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p) : "memory");
}

QHL_DEV unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// The phase count this CTA's consumers have seen complete, handed to the
// producer thread through shared memory (release / acquire at CTA scope), so
// only one thread per CTA polls the global counter.
QHL_DEV void st_release_cta(unsigned* p, unsigned v) {
  asm volatile("st.release.cta.shared.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
QHL_DEV unsigned ld_acquire_cta(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// Error path: once any CTA has recorded an error, every wait of the pass gives
// up and the CTAs leave (after drain_inflight_copies).
QHL_DEV void pass_drain() { drain_inflight_copies(); }

// Consumers: wait until phases 0 .. ph-1 are complete on every CTA, then tell
// this CTA's producer.  False if the pass is aborted (an error recorded
// anywhere, or this wait ran out).  Thread 0 polls with relaxed loads and
// acquires once the count is reached.
QHL_DEV bool grid_wait(const PassArgs& p, int ph, int* sflag, unsigned* ready) {
  if (threadIdx.x == 0) {
    const unsigned target = (unsigned)ph * (unsigned)p.grid;
    int ok = 1;
    for (uint32_t i = 0; ld_relaxed(p.bar) < target; ++i) {
      __nanosleep(64);   // keep the polling of the counter's L2 line light
      if ((i & 63u) == 63u && ld_relaxed(p.err)) {
        ok = 0;
        break;
      }
      if (i == kSpinLimit) {
        atomicOr(p.err, ERR_WAIT_TIMEOUT);
        ok = 0;
        break;
      }
    }
    (void)ld_acquire(p.bar);
    if (ok) st_release_cta(ready, (unsigned)ph);
    if (p.trace) p.trace[((size_t)blockIdx.x * p.n_phases + ph) * 2] = global_ns();
    *sflag = ok;
  }
  named_sync(1, 256);
  return *sflag != 0;
}

// Consumers: this CTA finished its share of the current phase.  Every thread
// orders its global writes before later bulk copies (async proxy) that other
// CTAs make of them; thread 0 then releases the arrival.
QHL_DEV void grid_arrive(const PassArgs& p, int ph) {
  fence_proxy_async_global();
  named_sync(1, 256);
  if (threadIdx.x == 0) {
    if (p.trace) p.trace[((size_t)blockIdx.x * p.n_phases + ph) * 2 + 1] = global_ns();
    red_add_release(p.bar);
  }
}

// Producer (one thread): stream every projection item of this CTA, in pass
// order, into the ring; issue each item's x copies once its phase is ready.
template <int QT, int NT, int S>
QHL_DEV void pass_producer(const PassArgs& p, int cta, uint8_t* stages, uint64_t* bars, const unsigned* ready_sm) {
  constexpr int IB = PassCfg<QT, NT>::kIB;
  constexpr int SB = PassCfg<QT, NT>::kSB;
  const uint64_t pol = policy_evict_first();
  struct XJob {
    const uint8_t* src;    // token 0's chunk
    int stride;
    int slot;
    int phase;
  };
  XJob q[S];
  int qh = 0, qn = 0;
  unsigned ready = 0;      // phases known complete
  auto service = [&]() {
    while (qn > 0) {
      const XJob& j = q[qh];
      if ((unsigned)j.phase > ready) {
        const unsigned done = ld_acquire_cta(ready_sm);
        if (done <= ready) return;
        ready = done;
        fence_proxy_async_global();
        if ((unsigned)j.phase > ready) return;
      }
      const uint32_t full = smem_u32(&bars[j.slot]);
      for (int t = 0; t < NT; ++t)
        bulk_g2s_plain(smem_u32(stages + j.slot * SB + IB + t * kQChunkBytes), j.src + (size_t)t * j.stride,
                       kQChunkBytes, full);
      qh = qh + 1 == S ? 0 : qh + 1;
      --qn;
    }
  };
  long long k = 0;          // items issued so far (all projections of the pass)
  int slot = 0;             // k % S
  uint32_t round = 0;       // k / S
  for (int l = 0; l < p.n_layers; ++l) {
    const PassLayer& L = p.layers[l];
    const int ph_out = L.phase_in + (L.attn ? 3 : 2);
    const int phases[4] = {L.phase_in, ph_out, ph_out + 1, ph_out + 2};
    for (int gi = 0; gi < 4; ++gi) {
      const GemvArgs& a = L.g[gi];
      if (cta >= a.workers) continue;
      const StreamK sk(a.tiles * a.chunks, a.workers);
      const int i0 = sk.begin(cta), i1 = sk.begin(cta + 1);
      int c = i0 % a.chunks;
      for (int it = i0; it < i1; ++it, ++k) {
        if (round > 0) {
          const uint32_t empty = smem_u32(&bars[S + slot]);
          const uint32_t par = (round - 1) & 1u;
          for (uint32_t spins = 0; !mbar_wait_for(empty, par, 256); ++spins) {
            service();
            if ((spins & 63u) == 63u && ld_relaxed(p.err)) {
              pass_drain();
              return;
            }
            if (spins == kSpinLimit) {
              atomicOr(p.err, ERR_WAIT_TIMEOUT);
              pass_drain();
              return;
            }
          }
        }
        const uint32_t full = smem_u32(&bars[slot]);
        mbar_arrive_expect_tx(full, SB);
        bulk_g2s(smem_u32(stages + slot * SB), a.W + (size_t)it * IB, IB, full, pol);
        int qt = qh + qn;
        if (qt >= S) qt -= S;
        q[qt] = XJob{a.qx + (size_t)c * kQChunkBytes, a.qx_stride, slot, phases[gi]};
        ++qn;
        if (++c == a.chunks) c = 0;
        if (++slot == S) {
          slot = 0;
          ++round;
        }
        service();
      }
    }
  }
  for (uint32_t spins = 0; qn > 0; ++spins) {
    service();
    __nanosleep(128);
    if ((spins & 63u) == 63u && ld_relaxed(p.err)) break;
    if (spins == kSpinLimit) {
      atomicOr(p.err, ERR_WAIT_TIMEOUT);
      break;
    }
  }
  if (qn > 0) pass_drain();
}

// The epilogue warp's arrival at the grid barrier after its share of a
// projection phase: every lane orders its global writes before later bulk
// copies that other CTAs make of them, lane 0 releases the arrival.
QHL_DEV void epilogue_arrive(const PassArgs& p, int ph) {
  fence_proxy_async_global();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    if (p.trace) p.trace[((size_t)blockIdx.x * p.n_phases + ph) * 2 + 1] = global_ns();
    red_add_release(p.bar);
  }
}

// Epilogue warp: wait until this CTA's consumers have seen phase `ph` open
// (so the previous step's outputs, the RMS partials among them, are visible).
// False if the pass is aborted.
QHL_DEV bool epilogue_wait(const PassArgs& p, int ph, const unsigned* ready_sm) {
  for (uint32_t i = 0; ld_acquire_cta(ready_sm) < (unsigned)ph; ++i) {
    if ((i & 63u) == 63u && ld_relaxed(p.err)) return false;
    if (i == kSpinLimit) {
      atomicOr(p.err, ERR_WAIT_TIMEOUT);
      return false;
    }
    __nanosleep(128);
  }
  return true;
}

// Epilogue warp over the whole pass: finishes every projection's tiles of this
// CTA and arrives at the barrier that closes each projection phase.
template <int NT>
QHL_DEV void pass_epilogue(const PassArgs& p, int cta, const TileSync& ts, float* fin, float* rstd,
                           const unsigned* ready_sm) {
  uint32_t tc = 0;
  bool timed_out = false;
  for (int l = 0; l < p.n_layers; ++l) {
    const PassLayer& L = p.layers[l];
    const int ph_out = L.phase_in + (L.attn ? 3 : 2);
    if (!epilogue_wait(p, L.phase_in, ready_sm)) break;
    gemv_finish<EPI_STORE, NT>(L.g[0], cta, ts, fin, rstd, tc, timed_out);
    epilogue_arrive(p, L.phase_in);
    if (!epilogue_wait(p, ph_out, ready_sm)) break;
    gemv_finish<EPI_RESID, NT>(L.g[1], cta, ts, fin, rstd, tc, timed_out);
    epilogue_arrive(p, ph_out);
    if (!epilogue_wait(p, ph_out + 1, ready_sm)) break;
    gemv_finish<EPI_SWIGLU, NT>(L.g[2], cta, ts, fin, rstd, tc, timed_out);
    epilogue_arrive(p, ph_out + 1);
    if (!epilogue_wait(p, ph_out + 2, ready_sm)) break;
    gemv_finish<EPI_RESID, NT>(L.g[3], cta, ts, fin, rstd, tc, timed_out);
    epilogue_arrive(p, ph_out + 2);
  }
}

template <int QT, int NT>
__global__ void __launch_bounds__(kGemvCtaThreads, 2) stage_pass_kernel(const PassArgs p) {
  using C = PassCfg<QT, NT>;
  constexpr int S = C::kStages;
  constexpr int RB = TileRing<NT>::kBufs;
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* stages = smem;
  uint8_t* mix = smem + C::kMixOff;                                   // mixer scratch / tile hand-off
  float* rstd = reinterpret_cast<float*>(smem + C::kRstdOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);   // full[S], empty[S], tile full[RB], tile free[RB]
  const TileSync ts{reinterpret_cast<float*>(mix), bars + 2 * S, bars + 2 * S + RB};
  float* fin = reinterpret_cast<float*>(mix + TileRing<NT>::kBytes);
  int* flag = reinterpret_cast<int*>(smem + C::kFlagOff);
  int* abort_flag = flag + 1;
  unsigned* ready_sm = reinterpret_cast<unsigned*>(flag + 2);         // phases seen complete

  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[S + s]), kConsumerWarps);
    }
    for (int b = 0; b < RB; ++b) {
      mbar_init(smem_u32(&ts.full[b]), kConsumerWarps * 32);
      mbar_init(smem_u32(&ts.free_[b]), 32);
    }
    fence_mbar_init();
    *ready_sm = 0;
  }
  __syncthreads();
  if (warp == kProducerWarp) {
    if ((tid & 31) == 0) pass_producer<QT, NT, S>(p, cta, stages, bars, ready_sm);
    return;
  }
  if (warp == kEpilogueWarp) {
    pass_epilogue<NT>(p, cta, ts, fin, rstd, ready_sm);
    return;
  }

  // ---- consumers: items of every projection, and the mixer / input units ----
  int slot = 0;
  uint32_t parity = 0, tc = 0;
  bool timed_out = false;
  int ph = 0;
  if (p.trace && tid == 0) p.trace[(size_t)cta * p.n_phases * 2] = global_ns();
  for (int u = cta; u < p.H / 64; u += p.grid)
    input_unit<NT>(p.h, p.H, p.gamma0, p.qz, p.qz_stride, p.ss, p.ss_stride, u, reinterpret_cast<float*>(mix));
  grid_arrive(p, 0);
  ++ph;
#define QHL_PASS_WAIT()                                 \
  if (!grid_wait(p, ph++, abort_flag, ready_sm)) {      \
    if (tid == 0) pass_drain();                         \
    return;                                             \
  }
  for (int l = 0; l < p.n_layers; ++l) {
    const PassLayer& L = p.layers[l];
    QHL_PASS_WAIT();
    gemv_consume<QT, NT, S>(L.g[0], cta, stages, bars, ts, slot, parity, tc, timed_out);   // the epilogue warp arrives
    if (!L.attn) {
      QHL_PASS_WAIT();
      for (int u = cta; u < p.dn_units; u += p.grid) dn_unit<NT>(L.dn, u, reinterpret_cast<float*>(mix));
      grid_arrive(p, ph - 1);
    } else {
      QHL_PASS_WAIT();
      const int pos = *p.kv_len;
      constexpr int kGroups = (NT + kAttGroup - 1) / kAttGroup;
      const int units = (pos + NT + kAttChunk - 1) / kAttChunk * p.Hkv * kGroups;
      for (int u = cta; u < units; u += p.grid) {
        const int grp = u % kGroups, rest = u / kGroups, t0 = grp * kAttGroup;
        const int c = rest / p.Hkv, g = rest % p.Hkv;
        if (c * kAttChunk < pos + t0 + min(kAttGroup, NT - t0)) attn_unit<NT>(L.at, c, g, pos, t0, mix);
      }
      grid_arrive(p, ph - 1);
      QHL_PASS_WAIT();
      for (int u = cta; u < NT * p.Hq; u += p.grid)
        combine_unit<NT>(L.at, u / p.Hq, u % p.Hq, pos, reinterpret_cast<float*>(mix));
      grid_arrive(p, ph - 1);
    }
    QHL_PASS_WAIT();
    gemv_consume<QT, NT, S>(L.g[1], cta, stages, bars, ts, slot, parity, tc, timed_out);
    QHL_PASS_WAIT();
    gemv_consume<QT, NT, S>(L.g[2], cta, stages, bars, ts, slot, parity, tc, timed_out);
    QHL_PASS_WAIT();
    gemv_consume<QT, NT, S>(L.g[3], cta, stages, bars, ts, slot, parity, tc, timed_out);
  }
#undef QHL_PASS_WAIT
  if (timed_out && tid == 0) pass_drain();
}

// Host side, per weight type; explicitly instantiated in pass_q4.cu / pass_q8.cu.
template <int QT>
struct PassOps {
  // shared-memory limit and carveout of every instantiation
  static cudaError_t prepare();
  // co-resident CTAs per SM of the nt-token kernel (0: not instantiated)
  static cudaError_t occupancy(int nt, int* blocks);
  // bytes of mixer scratch the nt-token kernel offers
  static int mix_bytes(int nt);
  // cooperative launch of p.grid CTAs
  static cudaError_t launch(int nt, const PassArgs& p, cudaStream_t s);
};

template <int QT, int NT>
cudaError_t pass_prepare_one() {
  if constexpr (PassCfg<QT, NT>::kFits) {
    cudaError_t e = cudaFuncSetAttribute(stage_pass_kernel<QT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         PassCfg<QT, NT>::kSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(stage_pass_kernel<QT, NT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    return e;
  } else {
    return cudaSuccess;
  }
}

template <int QT, int NT>
cudaError_t pass_occupancy_one(int* blocks) {
  *blocks = 0;
  if constexpr (PassCfg<QT, NT>::kFits)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, stage_pass_kernel<QT, NT>, kGemvCtaThreads,
                                                         PassCfg<QT, NT>::kSmem);
  else
    return cudaSuccess;
}

template <int QT, int NT>
cudaError_t pass_launch_one(const PassArgs& p, cudaStream_t s) {
  if constexpr (PassCfg<QT, NT>::kFits) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(kGemvCtaThreads);
    cfg.dynamicSmemBytes = PassCfg<QT, NT>::kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs co-resident: the grid barriers rely on it
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, stage_pass_kernel<QT, NT>, p);
  } else {
    return cudaErrorInvalidValue;
  }
}

template <int QT>
cudaError_t PassOps<QT>::prepare() {
  cudaError_t e = pass_prepare_one<QT, 1>();
  if (e == cudaSuccess) e = pass_prepare_one<QT, 2>();
  if (e == cudaSuccess) e = pass_prepare_one<QT, 3>();
  if (e == cudaSuccess) e = pass_prepare_one<QT, 4>();
  return e;
}

template <int QT>
cudaError_t PassOps<QT>::occupancy(int nt, int* blocks) {
  switch (nt) {
    case 1: return pass_occupancy_one<QT, 1>(blocks);
    case 2: return pass_occupancy_one<QT, 2>(blocks);
    case 3: return pass_occupancy_one<QT, 3>(blocks);
    case 4: return pass_occupancy_one<QT, 4>(blocks);
    default: *blocks = 0; return cudaSuccess;
  }
}

template <int QT>
int PassOps<QT>::mix_bytes(int nt) {
  switch (nt) {
    case 1: return PassCfg<QT, 1>::kMix;
    case 2: return PassCfg<QT, 2>::kMix;
    case 3: return PassCfg<QT, 3>::kMix;
    case 4: return PassCfg<QT, 4>::kMix;
    default: return 0;
  }
}

template <int QT>
cudaError_t PassOps<QT>::launch(int nt, const PassArgs& p, cudaStream_t s) {
  switch (nt) {
    case 1: return pass_launch_one<QT, 1>(p, s);
    case 2: return pass_launch_one<QT, 2>(p, s);
    case 3: return pass_launch_one<QT, 3>(p, s);
    case 4: return pass_launch_one<QT, 4>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qhl

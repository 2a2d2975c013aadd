// The whole layer-stage pass in one persistent, cooperative kernel.
//
// The pages submit one command buffer per token (SwarmLLM README, paragraph
// after the peer diagram), and every token reads all of the weights once.
// Here one grid of one CTA per SM runs every phase of the pass -- the stage
// input, then per layer the mixer in-projection, the DeltaNet step or the
// attention partials + combine, the out-projection, gate/up and down -- with
// the phases separated by a grid-wide arrival counter.  What a chain of
// kernels cannot do, this does: the weight stream never stops at a phase
// boundary.  The producer thread knows the pass's whole schedule of items
// and keeps both rings full across phases; only an item's x columns wait for
// the phase that writes them, and the unpack warps turn the next
// projection's weights into MMA operands while the previous phase finishes.
//
// Warp roles of the CTA (14 warps):
//   0..3    update (the GEMV role of qgemv.cuh, thread = tile row) during the
//           projection phases, and with 4..7 the mixer units (stage input,
//           DeltaNet step, attention partials and combine, the same device
//           functions as the separate kernels) during the mixer phases
//   4..7    mixer units only
//   8       producer (one thread): bulk copies of every projection's items
//   9       MMA issuer (one thread) and tensor-memory owner
//   10..13  unpack
// The update and the mixer phases of a layer are strictly ordered, so one set
// of warps serves both; fourteen warps of up to 128 registers fit the
// register file of an SM's four sub-partitions (at most four warps each).
// Each CTA arrives once per phase (the update warps for a projection, the
// mixer warps for a mixer phase); phase p may start once the counter reaches
// p * grid.  Every wait is bounded; any recorded error makes every wait of
// the pass give up.
#pragma once

#include "attention.cuh"
#include "deltanet.cuh"
#include "input.cuh"
#include "qgemv.cuh"

namespace qhl {

struct PassLayer {
  int attn;            // 1: full-attention layer, 0: gated DeltaNet
  int phase_in;        // phase of the mixer in-projection
  GemvArgs g[4];       // in-projection, out-projection, gate/up, down
  DnArgs dn;
  AttnArgs at;
};

struct PassArgs {
  const PassLayer* layers;
  int n_layers;
  const float* h;      // stage input [NT][H]
  int H;
  const float* gamma0; // first layer's RMSNorm weight
  uint8_t* qz;
  int qz_stride;
  float* ss;
  int ss_stride;
  const int* kv_len;   // position of token 0
  unsigned* bar;       // phase arrival counter, zero at launch
  int grid;            // CTAs (all co-resident)
  int dn_units;        // Hv * 4
  int Hq, Hkv;
  unsigned* err;
  uint32_t wait_limit; // 0: the default cap
};

// Mixer scratch of the persistent kernel: attention at up to 4 tokens with up
// to 7 query heads per KV head, the combine's chunk statistics, the DeltaNet
// unit, the stage input.
constexpr int kPassMixBytes = 40 * 1024;
constexpr int kPassMaxTok = 4;

constexpr int kPassMixWarps = 8;      // warps 0..7; 0..3 are also the update warps
constexpr int kPassProducerWarp = 8;  // weights
constexpr int kPassMmaWarp = 9;
constexpr int kPassUnpackWarp0 = 10;
constexpr int kPassXWarp = 14;
constexpr int kPassMma2Warp = 15;
constexpr int kPassThreads = 16 * 32;

template <int QT, int NT>
struct PassCfg : GemvGeom<QT, NT, 221 * 1024, 8, 4, 4, 12, kPassMixBytes> {
  static constexpr int kUnpackWarps = 4;
  static constexpr int kUpdateWarps = 4;
  static constexpr int kMmaThreads = 2;
  static_assert(PassCfg::kNA % 2 == 0 && PassCfg::kND % 2 == 0 && PassCfg::kSX % 2 == 0, "slots per MMA thread");
};

template <int QT, int NT>
constexpr int pass_smem_bytes() {
  return PassCfg<QT, NT>::kSmem;
}

QHL_DEV unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
QHL_DEV unsigned ld_relaxed_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
QHL_DEV void red_release_gpu(unsigned* p) { asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p) : "memory"); }
// Order this thread's earlier global writes before later async-proxy (bulk
// copy) reads of them, and acquired global data before later bulk copies.
QHL_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// One thread: wait until phase `ph` may start (every CTA arrived for the
// phases before it).  False if an error was recorded anywhere or the wait ran
// out.
QHL_DEV bool phase_wait(const PassArgs& p, int ph) {
  const unsigned target = (unsigned)ph * (unsigned)p.grid;
  const uint32_t limit = wait_limit(p.wait_limit);
  for (uint32_t i = 0;; ++i) {
    if (ld_acquire_gpu(p.bar) >= target) return true;
    if ((i & 63u) == 63u && ld_relaxed_gpu(p.err)) return false;
    if (i >= limit) {
      atomicOr(p.err, ERR_WAIT_TIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
}

// The threads of one role (`nthreads` on named barrier `bar_id`) wait for a
// phase together: thread `leader` polls, all get the same answer.
QHL_DEV bool group_phase_wait(const PassArgs& p, int ph, int bar_id, int nthreads, bool leader) {
  bool ok = true;
  if (leader) ok = phase_wait(p, ph);
  return bar_and(bar_id, nthreads, ok);
}

// The group's arrival for a phase after its writes: every thread orders its
// global writes before later bulk-copy reads by other CTAs, then the leader
// releases the arrival.
QHL_DEV void group_arrive(const PassArgs& p, int bar_id, int nthreads, bool leader) {
  fence_proxy_async_global();
  __threadfence();
  named_sync(bar_id, nthreads);
  if (leader) red_release_gpu(p.bar);
}

// This CTA's projection items in pass order: layer, projection, item and its
// chunk, stepped one item at a time.
struct PassItems {
  int l = 0, gi = -1, it = 0, i1 = 0, c = 0;
  // To the next item; false past the last.
  QHL_DEV bool next(const PassArgs& p, int cta) {
    if (gi >= 0 && ++it < i1) {
      if (++c == p.layers[l].g[gi].chunks) c = 0;
      return true;
    }
    for (;;) {
      if (++gi == 4) {
        gi = 0;
        if (++l >= p.n_layers) return false;
      }
      const GemvArgs& a = p.layers[l].g[gi];
      if (cta >= a.workers) continue;
      const StreamK sk(a.tiles * a.chunks, a.workers);
      it = sk.begin(cta);
      i1 = sk.begin(cta + 1);
      if (it < i1) {
        c = it % a.chunks;
        return true;
      }
    }
  }
  QHL_DEV const GemvArgs& args(const PassArgs& p) const { return p.layers[l].g[gi]; }
  // The phase in which the item's x columns are written (and may be read).
  QHL_DEV int phase(const PassArgs& p) const {
    const PassLayer& L = p.layers[l];
    return gi == 0 ? L.phase_in : L.phase_in + (L.attn ? 3 : 2) + gi - 1;
  }
};

// Weight producer (one thread): every projection item's quants in pass order,
// each as soon as its ring slot is released.  The weights never depend on the
// pass, so the stream runs across phase boundaries.
template <class C>
QHL_DEV bool pass_produce_weights(const PassArgs& p, const GemvSmem<C>& S, int cta) {
  constexpr int SW = C::kSW;
  const uint64_t pol = policy_evict_first();
  PassItems w;
  for (uint32_t K = 0; w.next(p, cta); ++K) {
    if (K >= (uint32_t)SW && !mbar_wait(smem_u32(&S.wempty[K % SW]), ((K / SW) - 1) & 1u, p.err, p.wait_limit))
      return false;
    issue_weights<C>(w.args(p), S, w.it, K, pol);
  }
  return true;
}

// x producer (one thread): every item's block scales and x columns.  Two
// cursors run over the items: the scales go as soon as the item's x slot is
// released (they are weights), the x columns once the phase that writes them
// has completed on every CTA.  The phase counter is polled with relaxed loads
// whose value is read at the next turn, so a poll never stalls the scale
// copies; once the target is seen, one acquiring load and a proxy fence order
// the phase's data before the bulk copies that read it.
template <class C>
QHL_DEV bool pass_produce_x(const PassArgs& p, const GemvSmem<C>& S, int cta) {
  constexpr int SX = C::kSX;
  const uint64_t pol = policy_evict_first();
  const uint32_t limit = wait_limit(p.wait_limit);
  PassItems sc, xc;
  bool s_ok = sc.next(p, cta), x_ok = xc.next(p, cta);
  uint32_t KS = 0, KX = 0;   // items whose scales / x columns are requested
  int ready = 0;             // phases known to have completed before
  unsigned polled = 0;
  bool poll_out = false;
  for (uint32_t spins = 0; x_ok;) {
    bool did = false;
    if (s_ok && (KS < (uint32_t)SX || mbar_test(smem_u32(&S.xempty[KS % SX]), ((KS / SX) - 1) & 1u))) {
      issue_scales<C>(sc.args(p), S, sc.it, KS, pol);
      ++KS;
      s_ok = sc.next(p, cta);
      did = true;
    }
    if (KX < KS) {
      const int ph = xc.phase(p);
      if (ph > ready) {
        if (!poll_out) {
          polled = ld_relaxed_gpu(p.bar);
          poll_out = true;
        } else {
          poll_out = false;
          if (polled >= (unsigned)ph * (unsigned)p.grid) {
            (void)ld_acquire_gpu(p.bar);
            fence_proxy_async_global();
            ready = ph;
          }
        }
      }
      if (ph <= ready) {
        issue_x<C>(xc.args(p), S, xc.c, KX);
        ++KX;
        x_ok = xc.next(p, cta);
        did = true;
      }
    }
    if (did) {
      spins = 0;
      continue;
    }
    if ((++spins & 63u) == 0 && ld_relaxed_gpu(p.err)) return false;
    if (spins >= limit) {
      atomicOr(p.err, ERR_WAIT_TIMEOUT);
      return false;
    }
    __nanosleep(32);
  }
  return true;
}

template <int QT, int NT>
__global__ void __maxnreg__(128) stage_pass_kernel(const PassArgs p) {
  using C = PassCfg<QT, NT>;
  extern __shared__ __align__(16) uint8_t gsmem[];
  const GemvSmem<C> S(gsmem);
  uint8_t* mix = S.extra;
  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == kPassProducerWarp) S.init(lane);
  if (warp == kPassMmaWarp) tmem_alloc(S.tslot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *S.tslot;
  bool ok = true;

  if (warp == kPassProducerWarp) {
    if (lane == 0 && !pass_produce_weights<C>(p, S, cta)) drain_inflight_copies();   // error path
    return;   // the producers take no part in the tensor-memory teardown
  }
  if (warp == kPassXWarp) {
    if (lane == 0 && !pass_produce_x<C>(p, S, cta)) drain_inflight_copies();   // error path
    return;
  }
  uint32_t K = 0;   // this CTA's items so far, over every projection of the pass
  if (warp < kPassMixWarps) {
    // ------------- warps 0..7: projection updates (0..3) and mixer units -----
    const bool upd = warp < 4;
    const bool lead = tid == 0;
    // one projection's update (warps 0..3): wait for its phase, run this
    // CTA's items, arrive
    auto update = [&](const GemvArgs& a, int gi, int ph) -> bool {
      if (!group_phase_wait(p, ph, kBarUpdate, 128, lead)) return false;
      bool good = true;
      if (cta < a.workers) {
        const StreamK sk(a.tiles * a.chunks, a.workers);
        const int i0 = sk.begin(cta), n = sk.begin(cta + 1) - i0;
        load_rstd<C>(a, S, warp & 3, lane);
        switch (gi) {
          case 0: good = update_items<C, EPI_STORE>(a, S, tmem, cta, i0, n, K, warp & 3, lane); break;
          case 1: good = update_items<C, EPI_RESID>(a, S, tmem, cta, i0, n, K, warp & 3, lane); break;
          case 2: good = update_items<C, EPI_SWIGLU>(a, S, tmem, cta, i0, n, K, warp & 3, lane); break;
          default: good = update_items<C, EPI_RESID>(a, S, tmem, cta, i0, n, K, warp & 3, lane); break;
        }
        K += n;
      }
      if (good) group_arrive(p, kBarUpdate, 128, lead);
      return good;
    };
    // phase 0: the stage input (warps 0..3, 128-row tiles)
    if (upd)
      for (int u = cta; u < p.H / kTileRows; u += p.grid)
        input_unit<NT>(p.h, p.H, p.gamma0, p.qz, p.qz_stride, p.ss, p.ss_stride, u, reinterpret_cast<float*>(mix),
                       kBarMix);
    group_arrive(p, kBarMix + 1, 256, lead);
    for (int l = 0; l < p.n_layers; ++l) {
      const PassLayer& L = p.layers[l];
      const int ph = L.phase_in + 1;
      const int ph_out = L.phase_in + (L.attn ? 3 : 2);
      if (upd && ok) ok = update(L.g[0], 0, L.phase_in);
      float4 Sr[4];
      const int u0 = cta;
      if (!L.attn && ok && u0 < p.dn_units) dn_load<NT>(L.dn, u0, Sr);   // the state rows never depend on this pass
      // the eight warps agree on going on before any barrier of the mixer
      if (!(ok = bar_and(kBarMix + 1, 256, ok))) break;
      if (!L.attn) {
        if (!(ok = group_phase_wait(p, ph, kBarMix + 1, 256, lead))) break;
        for (int u = u0; u < p.dn_units; u += p.grid) {
          if (u != u0) dn_load<NT>(L.dn, u, Sr);
          if (L.dn.mode == DN_CHUNKED)
            dn_run_chunked<NT>(L.dn, u, Sr, reinterpret_cast<float*>(mix));
          else
            dn_run<NT>(L.dn, u, Sr, reinterpret_cast<float*>(mix));
        }
        group_arrive(p, kBarMix + 1, 256, lead);
      } else {
        if (!(ok = group_phase_wait(p, ph, kBarMix + 1, 256, lead))) break;
        const int pos = *p.kv_len;
        constexpr int kGroups = (NT + kAttGroup - 1) / kAttGroup;
        const int units = (pos + NT + kAttChunk - 1) / kAttChunk * p.Hkv * kGroups;
        for (int u = cta; u < units; u += p.grid) {
          const int grp = u % kGroups, rest = u / kGroups, t0 = grp * kAttGroup;
          const int c = rest / p.Hkv, g = rest % p.Hkv;
          if (c * kAttChunk < pos + t0 + min(kAttGroup, NT - t0)) attn_unit<NT>(L.at, c, g, pos, t0, mix);
        }
        group_arrive(p, kBarMix + 1, 256, lead);
        if (!(ok = group_phase_wait(p, ph + 1, kBarMix + 1, 256, lead))) break;
        for (int u = cta; u < NT * p.Hq * kCombineParts; u += p.grid)
          combine_unit<NT>(L.at, u / (kCombineParts * p.Hq), (u / kCombineParts) % p.Hq, u % kCombineParts, pos,
                           reinterpret_cast<float*>(mix));
        group_arrive(p, kBarMix + 1, 256, lead);
      }
      // out-projection, gate/up, down (warps 0..3; 4..7 go on to the next
      // layer's agreement, where these four join them)
      if (upd)
        for (int gi = 1; gi < 4 && ok; ++gi) ok = update(L.g[gi], gi, ph_out + gi - 1);
    }
    if (!upd) {
      if (!ok && lane == 0) drain_inflight_copies();
      return;   // warps 4..7 take no part in the tensor-memory teardown
    }
  } else if (warp == kPassMmaWarp || warp == kPassMma2Warp) {
    if (lane == 0) {
      for (int l = 0; l < p.n_layers && ok; ++l)
        for (int gi = 0; gi < 4 && ok; ++gi) {
          const GemvArgs& a = p.layers[l].g[gi];
          if (cta >= a.workers) continue;
          const StreamK sk(a.tiles * a.chunks, a.workers);
          const int n = sk.begin(cta + 1) - sk.begin(cta);
          ok = mma_items<C>(a, S, tmem, n, K, warp == kPassMmaWarp ? 0 : 1);
          K += n;
        }
      // every MMA this thread issued has completed before tensor memory goes
      tc_commit(S.drain);
      if (!mbar_wait(smem_u32(S.drain), 0, p.err, p.wait_limit)) ok = false;
    }
    __syncwarp();
  } else {
    for (int l = 0; l < p.n_layers && ok; ++l)
      for (int gi = 0; gi < 4 && ok; ++gi) {
        const GemvArgs& a = p.layers[l].g[gi];
        if (cta >= a.workers) continue;
        const StreamK sk(a.tiles * a.chunks, a.workers);
        const int n = sk.begin(cta + 1) - sk.begin(cta);
        ok = unpack_items<C>(a, S, tmem, n, K, warp & 3, 0, lane);
        K += n;
      }
  }
  // ---------------- teardown: tensor memory back, after every MMA and load --
  tc_fence_before();
  named_sync(kBarTmem, 10 * 32);   // update 0..3, the two MMA warps, unpack 10..13
  if (warp == kPassMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  if (!ok && lane == 0) drain_inflight_copies();   // error path
}

}  // namespace qhl

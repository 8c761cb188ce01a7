// Fused 4-bit attention forward for sm_100a ("HiFA4: Training-Free 4-bit FlashAttention on
// Ascend HIF4 NPUs for LLM Inference", abstract): QK^T and PV both run as block-scaled
// FP4 tensor-core MMAs (tcgen05 kind::mxf4nvf4, accumulators in TMEM), the online-softmax
// running max m and normaliser l are kept in FP16, P is quantised to the 4-bit P_hat in
// registers, and -- P-Reordering -- the normaliser is summed from that same P_hat by the
// tensor core: an extra MMA of P_hat against a block of ones (N = 16) runs next to the
// PV MMA, so no row sum of P is computed on the ALUs.
//
// Persistent kernel: one CTA per SM walks a list of work units (batch, query head, 128-row
// query tile), longest first, in a snake order over the CTAs; kv tiles of BC keys are
// visited in ascending order.  Warp roles:
//   warp 0      TMA producer: per unit the Q tile (double-buffered, so the next unit's Q
//               arrives early), then K and V^T tiles (+ their scale atoms) into KS / VS-deep
//               shared-memory rings.
//   warp 1      allocates TMEM; issues tcgen05.cp (Q, K scales -> TMEM) and the QK^T MMAs
//               S_j = Q K_j^T into the S buffers.  The next unit's first QK^T overlaps the
//               epilogue.
//   warp 2      issues the PV MMAs: O (+)= P_hat_j V_j and R = P_hat_j * ones.
//   warps 3..   softmax: thread = one query row (TMEM lane).  Per tile: load S row, mask,
//               m_new = max(m, fp16(rowmax(S) * c)), P = E(fma(S, c, -m_new)) quantised to
//               P_hat (codes -> shared memory in the MMA's swizzled layout, scales -> a
//               scale atom), then after PV_{j-1} completed: l = fp16(fma(alpha_{j-1}, l,
//               R)) and O *= alpha_j where m changed.  Epilogue O / l -> bf16.
// Every wait is bounded (wall-clock limit, shared abort flag); on a timeout the kernel
// sets the status word, drains its own copies and MMAs and frees TMEM before exiting.
#pragma once
#include <cuda.h>
#include "method.cuh"

namespace hifa4 {

__host__ __device__ constexpr uint32_t layout_code(int rowbytes) {
  return rowbytes == 32 ? 6u : rowbytes == 64 ? 4u : 2u;   // UMMA SWIZZLE_32B / 64B / 128B
}
__host__ __device__ constexpr uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int D_, int BC_>
struct AttnCfg {
  static constexpr int D = D_, BC = BC_, BR = 128;
  static constexpr int KQ = D / 64;             // 64-wide K chunks of QK^T
  static constexpr int KP = BC / 64;            // 64-wide K chunks of PV
  static constexpr int NAK = BC > 128 ? BC / 128 : 1;   // 128-row scale atoms per K tile
  static constexpr int NAV = (D + 127) / 128;   // 128-channel scale atoms of V^T
  static constexpr int QROW = D / 2, PROW = BC / 2;
  static constexpr int KS = 3, VS = 3;
  static constexpr uint32_t LQ = layout_code(QROW), LP = layout_code(PROW);
  static constexpr uint32_t SZ_Q = BR * QROW, SZ_K = BC * QROW, SZ_V = D * PROW, SZ_P = BR * PROW;
  static constexpr uint32_t SZ_ONES = 16 * PROW;
  static constexpr uint32_t SZ_QSF = KQ * 512, SZ_KSF = NAK * KQ * 512, SZ_VSF = KP * NAV * 512, SZ_PSF = KP * 512;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + 2 * align_up(SZ_Q, 1024);
  static constexpr uint32_t OFF_V = OFF_K + KS * align_up(SZ_K, 1024);
  static constexpr uint32_t OFF_P = OFF_V + VS * align_up(SZ_V, 1024);
  static constexpr uint32_t OFF_ONES = OFF_P + 2 * align_up(SZ_P, 1024);
  static constexpr uint32_t OFF_QSF = OFF_ONES + align_up(SZ_ONES, 1024);
  static constexpr uint32_t OFF_KSF = OFF_QSF + 2 * SZ_QSF;
  static constexpr uint32_t OFF_VSF = OFF_KSF + KS * SZ_KSF;
  static constexpr uint32_t OFF_PSF = OFF_VSF + VS * SZ_VSF;
  static constexpr uint32_t OFF_1SF = OFF_PSF + 2 * SZ_PSF;
  static constexpr uint32_t OFF_RTAB = OFF_1SF + 512;            // 256 x fp32: RN(1/sigma) (fast rule: L(sigma))
  static constexpr uint32_t OFF_XMAX = OFF_RTAB + 1024;          // [2][NSW][128] fp32 partial row maxima
  static constexpr uint32_t OFF_XSUM = OFF_XMAX + 2 * 4 * 128 * 4;   // [2][NSW][128] partial sums of P (ablation)
  static constexpr uint32_t OFF_BAR = OFF_XSUM + 2 * 4 * 128 * 4;
  // barriers: q_full[2], q_empty[2], k_full[KS], k_empty[KS], v_full[VS], v_empty[VS],
  // s_full[2], s_empty[2], p_full[2], o_bar, o_free, drain[2]
  static constexpr int NBAR = 4 + 2 * KS + 2 * VS + 6 + 4;
  static constexpr uint32_t OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;   // + slack for 1024-B alignment
  // TMEM columns.  S is double-buffered when it fits; a single buffer is enough for
  // overlap because the softmax warps release S as soon as it is in their registers.
  static constexpr uint32_t SF_COLS = 4 * KQ + 8 * KQ * NAK + 8 * KP + 8 * KP * NAV + 4;
  static constexpr int SB = (2 * BC + D + 16 + SF_COLS <= 512) ? 2 : 1;
  static constexpr uint32_t T_S = 0, T_O = SB * BC, T_R = T_O + D, T_SFQ = T_R + 16;
  static constexpr uint32_t T_SFK = T_SFQ + 4 * KQ, T_SFP = T_SFK + 8 * KQ * NAK, T_SFV = T_SFP + 8 * KP;
  static constexpr uint32_t T_SF1 = T_SFV + 8 * KP * NAV, T_END = T_SF1 + 4;
  static constexpr uint32_t TMEM_COLS = T_END <= 256 ? 256 : 512;
  static_assert(T_END <= 512, "TMEM budget exceeded");
  static_assert(D == 64 || D == 128 || D == 256, "head dim");
  static_assert(BC == 64 || BC == 128 || BC == 256, "kv tile");
  // softmax warpgroups (at most 4, so that all softmax warps of a lane quarter share one
  // SMSP): each takes CW consecutive score columns of every row and D/NSW columns of O (both
  // at least 32, the width of one tcgen05.ld)
  static constexpr int NSW0 = (BC < D ? BC : D) / 32;
  static constexpr int NSW = NSW0 < 4 ? NSW0 : 4, CW = BC / NSW;
  static_assert(NSW == 2 || NSW == 4, "softmax warpgroups");
  static_assert(CW == 32 || CW == 64 || CW == 128, "column split");
  static constexpr int NTHREADS = 96 + 128 * NSW;   // producer, QK^T issuer, PV issuer, softmax
};

struct AttnParams {
  const uint8_t* qsf;       // Q scale atoms  [B, Hq, N/128, D/64, 512]
  const uint8_t* ksf;       // K scale atoms  [B, Hkv, N/128, D/64, 512]
  const uint8_t* vsf;       // V^T scale atoms [B, Hkv, N/64, ceil(D/128), 512]
  __nv_bfloat16* o;         // [B, Hq, N, D]
  __half* m_out;            // [B, Hq, N] or nullptr
  __half* l_out;            // [B, Hq, N] or nullptr
  int* status;
  int B, Hq, Hkv, N, causal;
  float c;                  // RN(log2(e) / sqrt(D))
  unsigned long long wait_ns;
  int inject;               // 1: the producer never delivers kv tile 1 (timeout test)
  int l_from_p;             // ablation kernels: 1 = l from the unquantised P (inconsistent normaliser)
  // keys per kv head (= N for the square forward); decode / split-KV kernels (DEC): Q holds
  // packed rows (B * Hkv tiles of 128 rows: row r = hi * nq + t, token t of query head
  // g * G + hi, at position Nk - nq + t); unit = (b * Hkv + g, split) over kv tiles
  // [split * tps, ...); partials (unnormalised fp32 O, m, l) go to part_*
  int Nk, nq, G, nsplit, tps;
  float* part_o;            // [B * Hkv * nsplit * 128, D]
  float* part_m;            // [B * Hkv * nsplit * 128]
  float* part_l;
  float* trace;             // ablation kernels: [B*Hq*N][N/BC][2] per (row, tile): sum P_hat, sum P; or nullptr
  // ablation kernels: 1 = two-level P scale, a per-(row, tile) power of two 2^k under the
  // block scales of P, k = max(floor(log2 p_t) - 10, -40), p_t the tile's largest block
  // amax; TMEM then holds O * 2^-k and R * 2^-k
  int two_level;
  float lneg[128];          // fast code rule: L(sigma) = RN(-log2 sigma) per E4M3 scale code (-inf for 0)
};

// Keep the register results of tcgen05.ld from being read before tcgen05.wait::ld.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Bounded wait that also returns early when another role aborted; warp-uniform result.
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort, int* status,
                                         uint64_t ns) {
  bool ok = mbar_wait(bar, parity, abort, status, ns);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait used while draining: ignores the abort flag.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, int* status, uint64_t ns) {
  int never = 0;
  return mbar_wait(bar, parity, &never, status, ns);
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Geometry of work unit u.  Square forward: units (batch * query head, 128-row query tile),
// causal ones longest first; decode: units (batch * kv head, split).
struct UnitGeom {
  int qrow;         // first row of the unit's Q tile in the Q tensor (its scale atom: qrow / 128)
  int kvh;          // global kv head b * Hkv + g
  int j0, nt;       // kv tiles j0 .. j0 + nt - 1
  long long orow;   // output row of TMEM lane 0 (decode: partial slot u * 128)
  int pos0;         // square causal: the key limit of lane 0 (lane r sees keys <= pos0 + r)
};

template <int BC, bool DEC>
__device__ __forceinline__ UnitGeom unit_geom(int u, const AttnParams& p) {
  UnitGeom g;
  if constexpr (DEC) {
    const int bkv = u / p.nsplit, sp = u % p.nsplit, ntile = p.Nk / BC;
    g.qrow = bkv * 128;
    g.kvh = bkv;
    g.j0 = min(sp * p.tps, ntile);
    g.nt = min(p.tps, ntile - g.j0);
    g.orow = (long long)u * 128;
    g.pos0 = 0;
  } else {
    const int BH = p.B * p.Hq, nqt = p.N / 128;
    const int qtile = p.causal ? nqt - 1 - u / BH : u / BH;
    const int bh = u % BH;
    g.qrow = bh * p.N + qtile * 128;
    g.kvh = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / (p.Hq / p.Hkv);
    g.j0 = 0;
    g.nt = p.causal ? ((qtile + 1) * 128 + BC - 1) / BC : p.N / BC;
    g.orow = (long long)bh * p.N + qtile * 128;
    g.pos0 = qtile * 128;
  }
  return g;
}

//
// DEC: the decode / split-KV kernels (packed query rows, a split's tile range, partial
// outputs); the square forward is the DEC = false instance.
// FAST: the approximate P_hat code rule (linear-mantissa exponential in the log domain,
// see phat_pair); the default instances round RN(P * RN(1/sigma)) to E2M1.
template <int D, int BC, bool SUMP = false, bool DEC = false, bool FAST = false>
__global__ void __launch_bounds__(AttnCfg<D, BC>::NTHREADS, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<D, BC>;
  static_assert(!(FAST && (SUMP || DEC)), "the fast code rule exists for the plain forward only");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sOnes = smem + C::OFF_ONES;
  uint8_t* s1sf = smem + C::OFF_1SF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 2;
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + C::KS;
  uint64_t* v_full = k_empty + C::KS;
  uint64_t* v_empty = v_full + C::VS;
  uint64_t* s_full = v_empty + C::VS;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* o_bar = p_full + 2;
  uint64_t* o_free = o_bar + 1;
  uint64_t* drain_bar = o_free + 1;   // [0] QK^T issuer, [1] PV issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  auto sQ = [&](int s) { return smem + C::OFF_Q + s * align_up(C::SZ_Q, 1024); };
  auto sQsf = [&](int s) { return smem + C::OFF_QSF + s * C::SZ_QSF; };
  auto sK = [&](int s) { return smem + C::OFF_K + s * align_up(C::SZ_K, 1024); };
  auto sV = [&](int s) { return smem + C::OFF_V + s * align_up(C::SZ_V, 1024); };
  auto sP = [&](int s) { return smem + C::OFF_P + s * align_up(C::SZ_P, 1024); };
  auto sKsf = [&](int s) { return smem + C::OFF_KSF + s * C::SZ_KSF; };
  auto sVsf = [&](int s) { return smem + C::OFF_VSF + s * C::SZ_VSF; };
  auto sPsf = [&](int s) { return smem + C::OFF_PSF + s * C::SZ_PSF; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = DEC ? p.B * p.Hkv * p.nsplit : p.B * p.Hq * (p.N / 128);
  // the CTA's i-th unit: rows of gridDim.x units, every other row reversed (snake order),
  // which evens out the per-CTA work of the longest-first causal list
  auto unit_of = [&](int i) {
    return i * (int)gridDim.x + ((i & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBAR; ++i) {
      const bool per_warp = (&bars[i] == &s_empty[0] || &bars[i] == &s_empty[1] || &bars[i] == &p_full[0] ||
                             &bars[i] == &p_full[1] || &bars[i] == o_free);
      mbar_init(&bars[i], per_warp ? 4 * C::NSW : 1);   // one arrival per softmax warp
    }
    *abort = 0;
    fence_mbar_init();
  }
  float* rtab = reinterpret_cast<float*>(smem + C::OFF_RTAB);
  float* xmax = reinterpret_cast<float*>(smem + C::OFF_XMAX);
  float* xsum = reinterpret_cast<float*>(smem + C::OFF_XSUM);
  if (warp >= 3) {
    // the ones operand (E2M1 1.0 = 0b0010 in both nibbles) and its scales (UE4M3 1.0)
    const int t = threadIdx.x - 96, nt2 = 128 * C::NSW;
    for (int i = t; i < (int)C::SZ_ONES / 4; i += nt2) reinterpret_cast<uint32_t*>(sOnes)[i] = 0x22222222u;
    for (int i = t; i < 128; i += nt2) reinterpret_cast<uint32_t*>(s1sf)[i] = 0x38383838u;
    fence_proxy_async_smem();
    if constexpr (FAST) {
      for (int i = t; i < 128; i += nt2) rtab[i] = p.lneg[i];
    } else {
      fill_recip_table(rtab, t, nt2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int nq = 0, nk = 0, nv = 0;   // loads issued (Q per unit, K and V per tile)
      bool ok = true;
      for (int i = 0, u = unit_of(0); ok && u < units; u = unit_of(++i)) {
        const UnitGeom ug = unit_geom<BC, DEC>(u, p);
        const int kvh = ug.kvh;
        const int qb = i & 1;
        if (i >= 2 && !mbar_wait(&q_empty[qb], ((i >> 1) - 1) & 1, abort, p.status, p.wait_ns)) break;
        mbar_arrive_expect_tx(&q_full[qb], C::SZ_Q + C::SZ_QSF);
        tma_load_2d(sQ(qb), &tmQ, 0, ug.qrow, &q_full[qb]);
        bulk_load(sQsf(qb), p.qsf + (long long)(ug.qrow / 128) * C::SZ_QSF, C::SZ_QSF, &q_full[qb]);
        ++nq;
        for (int jj = 0; jj < ug.nt; ++jj) {
          const int j = ug.j0 + jj;
          if (p.inject == 1 && i == 0 && jj == 1) { ok = false; break; }
          const int g = nk, ks = g % C::KS, vs = g % C::VS;
          if (g >= C::KS && !mbar_wait(&k_empty[ks], ((g / C::KS) - 1) & 1, abort, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[ks], C::SZ_K + C::SZ_KSF);
          tma_load_2d(sK(ks), &tmK, 0, kvh * p.Nk + j * BC, &k_full[ks]);
          // the tile's NAK consecutive 128-row atoms (KQ x 512 bytes each) are contiguous
          const int katom = (j * BC) / 128;
          bulk_load(sKsf(ks), p.ksf + ((long long)kvh * (p.Nk / 128) + katom) * (C::KQ * 512), C::SZ_KSF,
                    &k_full[ks]);
          ++nk;
          if (g >= C::VS && !mbar_wait(&v_empty[vs], ((g / C::VS) - 1) & 1, abort, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[vs], C::SZ_V + C::SZ_VSF);
          tma_load_2d(sV(vs), &tmV, j * C::PROW, kvh * D, &v_full[vs]);
          bulk_load(sVsf(vs), p.vsf + ((long long)kvh * (p.Nk / 64) + j * C::KP) * (C::NAV * 512), C::SZ_VSF,
                    &v_full[vs]);
          ++nv;
        }
      }
      // drain: every load this warp issued must have landed before the CTA exits
      auto drain_ring = [&](uint64_t* full, int n, int stages) {
        for (int s = 0; s < stages && s < n; ++s) {
          const int last = s + ((n - 1 - s) / stages) * stages;
          drain_wait(&full[s], (last / stages) & 1, p.status, p.wait_ns);
        }
      };
      drain_ring(q_full, nq, 2);
      drain_ring(k_full, nk, C::KS);
      drain_ring(v_full, nv, C::VS);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ QK^T issuer
    // S_g = Q K_g^T into S buffer g % SB.  Shared-memory descriptors are formed once; a
    // byte offset inside the (256 KB) window adds offset >> 4 to the start-address field.
    constexpr uint32_t ID_QK = idesc_nvf4(128, BC);
    const uint64_t dQ = smem_desc(smem_u32(sQ(0)), 0, 8 * C::QROW, C::LQ);
    const uint64_t dK = smem_desc(smem_u32(sK(0)), 0, 8 * C::QROW, C::LQ);
    const uint64_t dQsf = smem_desc(smem_u32(sQsf(0)), 0, 128, 0);
    const uint64_t dKsf = smem_desc(smem_u32(sKsf(0)), 0, 128, 0);
    bool ok = true;
    int g = 0;   // global tile counter
    for (int i = 0, u = unit_of(0); ok && u < units; u = unit_of(++i)) {
      const UnitGeom ug = unit_geom<BC, DEC>(u, p);
      const int nt = ug.nt;
      const int qb = i & 1;
      ok = wait_all(&q_full[qb], (i >> 1) & 1, abort, p.status, p.wait_ns);
      // the previous unit's QK MMAs (which read the Q scale columns) have completed
      if (ok && i >= 1) ok = wait_all(&q_empty[qb ^ 1], ((i - 1) >> 1) & 1, abort, p.status, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kc = 0; kc < C::KQ; ++kc)
          tmem_cp_sf(tbase + C::T_SFQ + 4 * kc, dQsf + ((qb * C::SZ_QSF + 512 * kc) >> 4));
      }
      __syncwarp();
      const uint64_t dQi = dQ + ((qb * align_up(C::SZ_Q, 1024)) >> 4);
      for (int jj = 0; ok && jj < nt; ++jj, ++g) {
        const int j = ug.j0 + jj;
        const int ks = g % C::KS, sb = g % C::SB;
        ok = wait_all(&k_full[ks], (g / C::KS) & 1, abort, p.status, p.wait_ns);
        if (ok && g >= C::SB) ok = wait_all(&s_empty[sb], ((g / C::SB) - 1) & 1, abort, p.status, p.wait_ns);
        if (!ok) break;
        if (BC == 64 && (j & 1)) {
          // keys 64..127 of the 128-row scale atom: move record words 2,3 into words 0,1
#pragma unroll
          for (int kc = 0; kc < C::KQ; ++kc) {
            uint4* rec = reinterpret_cast<uint4*>(sKsf(ks) + 512 * kc) + lane;
            uint4 w = *rec;
            *rec = make_uint4(w.z, w.w, w.z, w.w);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        tc_fence_after();
        if (lane == 0) {
          // K scale atoms (row atom rt, chunk kc) -> 4 columns at chunk kc's 4*NAK columns + 4 rt
          const uint32_t sfk = tbase + C::T_SFK + (g & 1) * 4 * C::KQ * C::NAK;
          const uint64_t dKsfs = dKsf + ((ks * C::SZ_KSF) >> 4);
#pragma unroll
          for (int rt = 0; rt < C::NAK; ++rt)
#pragma unroll
            for (int kc = 0; kc < C::KQ; ++kc)
              tmem_cp_sf(sfk + 4 * (C::NAK * kc + rt), dKsfs + ((512 * (rt * C::KQ + kc)) >> 4));
          const uint64_t dKs = dK + ((ks * align_up(C::SZ_K, 1024)) >> 4);
#pragma unroll
          for (int kc = 0; kc < C::KQ; ++kc)
            mma_nvf4(tbase + C::T_S + sb * BC, dQi + 2 * kc, dKs + 2 * kc, ID_QK, tbase + C::T_SFQ + 4 * kc,
                     sfk + 4 * C::NAK * kc, kc > 0 ? 1u : 0u);
          tc_commit(&s_full[sb]);
          tc_commit(&k_empty[ks]);
          if (jj == nt - 1) tc_commit(&q_empty[qb]);   // the unit's Q tile and Q scales are free
        }
        __syncwarp();
      }
    }
    // drain: every MMA / copy this warp issued has completed before TMEM is freed
    if (lane == 0) {
      tc_commit(&drain_bar[0]);
      drain_wait(&drain_bar[0], 0, p.status, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ PV issuer
    // O (+)= P_hat_g V_g and R = P_hat_g * ones, once the softmax warps have written
    // P_hat_g and applied alpha to O (p_full).
    constexpr uint32_t ID_PV = idesc_nvf4(128, D), ID_R = idesc_nvf4(128, 16);
    const uint64_t dP = smem_desc(smem_u32(sP(0)), 0, 8 * C::PROW, C::LP);
    const uint64_t dV = smem_desc(smem_u32(sV(0)), 0, 8 * C::PROW, C::LP);
    const uint64_t dOnes = smem_desc(smem_u32(sOnes), 0, 8 * C::PROW, C::LP);
    const uint64_t dPsf = smem_desc(smem_u32(sPsf(0)), 0, 128, 0);
    const uint64_t dVsf = smem_desc(smem_u32(sVsf(0)), 0, 128, 0);
    tc_fence_after();
    if (lane == 0) tmem_cp_sf(tbase + C::T_SF1, smem_desc(smem_u32(s1sf), 0, 128, 0));
    __syncwarp();
    bool ok = true;
    int g = 0;   // global tile counter
    for (int i = 0, u = unit_of(0); ok && u < units; u = unit_of(++i)) {
      const int nt = unit_geom<BC, DEC>(u, p).nt;
      for (int j = 0; ok && j < nt; ++j, ++g) {   // j: the unit's local tile index
        const int vs = g % C::VS, pb = g & 1;
        ok = wait_all(&v_full[vs], (g / C::VS) & 1, abort, p.status, p.wait_ns);
        ok = ok && wait_all(&p_full[pb], (g >> 1) & 1, abort, p.status, p.wait_ns);
        // the previous unit's epilogue must have read O and R before they are overwritten
        if (ok && j == 0 && i >= 1) ok = wait_all(o_free, (i - 1) & 1, abort, p.status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sfv = tbase + C::T_SFV + pb * 4 * C::KP * C::NAV;
          const uint32_t sfp = tbase + C::T_SFP + pb * 4 * C::KP;
          const uint64_t dVsfs = dVsf + ((vs * C::SZ_VSF) >> 4), dPsfs = dPsf + ((pb * C::SZ_PSF) >> 4);
#pragma unroll
          for (int q = 0; q < C::KP * C::NAV; ++q) tmem_cp_sf(sfv + 4 * q, dVsfs + 32 * q);
#pragma unroll
          for (int kc = 0; kc < C::KP; ++kc) tmem_cp_sf(sfp + 4 * kc, dPsfs + 32 * kc);
          const uint64_t dPs = dP + ((pb * align_up(C::SZ_P, 1024)) >> 4);
          const uint64_t dVs = dV + ((vs * align_up(C::SZ_V, 1024)) >> 4);
#pragma unroll
          for (int kc = 0; kc < C::KP; ++kc)
            mma_nvf4(tbase + C::T_O, dPs + 2 * kc, dVs + 2 * kc, ID_PV, sfp + 4 * kc, sfv + 4 * C::NAV * kc,
                     (j > 0 || kc > 0) ? 1u : 0u);
#pragma unroll
          for (int kc = 0; kc < C::KP; ++kc)
            mma_nvf4(tbase + C::T_R, dPs + 2 * kc, dOnes + 2 * kc, ID_R, sfp + 4 * kc, tbase + C::T_SF1,
                     kc > 0 ? 1u : 0u);
          tc_commit(o_bar);
          tc_commit(&v_empty[vs]);
        }
        __syncwarp();
      }
    }
    if (lane == 0) {
      tc_commit(&drain_bar[1]);
      drain_wait(&drain_bar[1], 0, p.status, p.wait_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    // warps w, w+4, ... share TMEM lane quarter q4 (the same 32 query rows); warpgroup
    // wg takes score columns [wg*CW, wg*CW + CW) and O columns [wg*D/NSW, ...).
    constexpr int CW = C::CW, NB = CW / 16, OW = D / C::NSW;
    const int sw = warp - 3, wg = sw >> 2;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lrow = (uint32_t)(q4 * 32) << 16;
    const int col0 = wg * CW;
    const float c = p.c;
    const float c7 = c * 0.0078125f;
    // this thread's byte offsets in a P_hat buffer (swizzled K-major rows) and in its scale atoms
    uint32_t p_off[CW / 32];
#pragma unroll
    for (int q = 0; q < CW / 32; ++q) p_off[q] = swz_offset(row, col0 / 32 + q, C::PROW);
    // one scale atom per 64 columns: CW / 64 atoms (CW = 128), or a part of one
    constexpr int NATOM = CW >= 64 ? CW / 64 : 1;
    const uint32_t psf_off = 512 * (col0 / 64) + sf_atom_offset(row, (col0 % 64) / 16);
    // Epilogue of a unit whose last tile is gl: read R and O of that tile's PV, release
    // them (o_free), then O / l -> bf16 (decode: the unnormalised fp32 O and l of the
    // split's partial).  It runs after the next unit's first tile, which touches neither O
    // nor R, so that tile's work overlaps the last PV.
    const int ntmax = p.N / BC;
    auto epilogue = [&](int gl, long long orow, float l_e, float alpha_e, float rsum_e, int jl, float kpow_e) -> bool {
      if (!wait_all(o_bar, gl & 1, abort, p.status, p.wait_ns)) return false;
      tc_fence_after();
      uint32_t rr[1] = {tmem_ld1(tbase + lrow + C::T_R)};
      tmem_wait_ld();
      reg_fence(rr);
      float r_use = __uint_as_float(rr[0]);
      if constexpr (SUMP) {
        r_use = __fmul_rn(r_use, kpow_e);   // two-level: R * 2^-k -> sum P_hat (exact)
        if (p.trace && wg == 0) {
          float* t = p.trace + (orow * ntmax + jl) * 2;
          t[0] = r_use;
          t[1] = rsum_e;
        }
        if (p.l_from_p) r_use = rsum_e;
      }
      const float l_fin = f16_round(__fmaf_rn(alpha_e, l_e, r_use));
      if constexpr (DEC) {
        float4* pdst = reinterpret_cast<float4*>(p.part_o + orow * D);
#pragma unroll 1
        for (int c0 = wg * OW; c0 < wg * OW + OW; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tbase + lrow + C::T_O + c0, o);
          tmem_wait_ld();
          reg_fence(o);
          if (c0 + 32 == wg * OW + OW) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
          }
#pragma unroll
          for (int q = 0; q < 8; ++q)
            pdst[c0 / 4 + q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                           __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
        }
        if (wg == 0) p.part_l[orow] = l_fin;
        return true;
      }
      float inv = (l_fin > 0.0f) ? __frcp_rn(l_fin) : 0.0f;
      if constexpr (SUMP) inv = __fmul_rn(inv, kpow_e);   // O in TMEM is O * 2^-k
      uint4* dst = reinterpret_cast<uint4*>(p.o + orow * D);
#pragma unroll 1
      for (int c0 = wg * OW; c0 < wg * OW + OW; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tbase + lrow + C::T_O + c0, o);
        tmem_wait_ld();
        reg_fence(o);
        if (c0 + 32 == wg * OW + OW) {
          // every TMEM read of this unit is done: the next unit's first PV may overwrite O, R
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free);
        }
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          __nv_bfloat162 v2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(o[2 * q]), inv),
                                                    __fmul_rn(__uint_as_float(o[2 * q + 1]), inv));
          pk[q] = *reinterpret_cast<uint32_t*>(&v2);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[c0 / 8 + q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      if (wg == 0 && p.l_out) p.l_out[orow] = __float2half_rn(l_fin);
      return true;
    };
    bool ok = true;
    long long pend_row = 0;                  // the previous unit's output row, l and alpha
    float pend_l = 0.0f, pend_alpha = 0.0f;
    float pend_rsum = 0.0f;                  // ablation kernels: its last tile's sum of P and index
    int pend_j = 0;
    float pend_kpow = 1.0f;                  // two-level: 2^k of that tile
    int g = 0;   // global tile counter
    for (int i = 0, u = unit_of(0); ok && u < units; u = unit_of(++i)) {
      const UnitGeom ug = unit_geom<BC, DEC>(u, p);
      const int nt = ug.nt;
      // the last key this thread's row sees, and the smallest such limit of the unit's rows:
      // tiles ending at or below it need no mask
      int pos, pos_min;
      if constexpr (DEC) {
        pos = row < p.G * p.nq ? p.Nk - p.nq + row % p.nq : p.Nk - 1;
        pos_min = p.Nk - p.nq;
      } else {
        pos = p.causal ? ug.pos0 + row : 0x7FFFFFFF;
        pos_min = p.causal ? ug.pos0 : 0x7FFFFFFF;
      }
      float m_run = -INFINITY, l_run = 0.0f, alpha_prev = 0.0f;
      float rsum_prev = 0.0f;                // ablation kernels: the previous tile's sum of P
      int k_prev = 0;                        // two-level: the previous tile's k and 2^k
      float kpow_prev = 1.0f;
      for (int jj = 0; jj < nt; ++jj, ++g) {
        const int j = ug.j0 + jj;
        const int sb = g % C::SB, pb = g & 1;
        ok = wait_all(&s_full[sb], (g / C::SB) & 1, abort, p.status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        float s[CW];
        {
          uint32_t r[CW];
#pragma unroll
          for (int c0 = 0; c0 < CW; c0 += 32)
            tmem_ld32(tbase + lrow + C::T_S + sb * BC + col0 + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[c0]));
          tmem_wait_ld();
          reg_fence(r);
#pragma unroll
          for (int q = 0; q < CW; ++q) s[q] = __uint_as_float(r[q]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
        if ((j + 1) * BC - 1 > pos_min) {
#pragma unroll
          for (int q = 0; q < CW; ++q)
            if (j * BC + col0 + q > pos) s[q] = -INFINITY;
        }
        // block maxima as a 3-input-max tree (depth 3), then the row part over the blocks
        float bmax[NB];
#pragma unroll
        for (int bl = 0; bl < NB; ++bl) {
          const float* x = s + bl * 16;
          const float u0 = fmax3(fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], x[5]), fmax3(x[6], x[7], x[8]));
          const float u1 = fmax3(fmax3(x[9], x[10], x[11]), fmax3(x[12], x[13], x[14]), x[15]);
          bmax[bl] = fmaxf(u0, u1);
        }
        float lmax = bmax[0];
        if constexpr (NB == 4) {
          lmax = fmaxf(fmax3(bmax[0], bmax[1], bmax[2]), bmax[3]);
        } else {
#pragma unroll
          for (int bl = 1; bl < NB; ++bl) lmax = fmaxf(lmax, bmax[bl]);
        }
        // combine the partial row maxima of the NSW warpgroups (double-buffered by parity)
        float* xm = xmax + (g & 1) * (C::NSW * 128);
        xm[wg * 128 + row] = lmax;
        named_bar(1 + q4, 32 * C::NSW);
        float rmax;
        if constexpr (C::NSW == 4) {
          rmax = fmaxf(fmax3(xm[row], xm[128 + row], xm[256 + row]), xm[384 + row]);
        } else {
          rmax = fmaxf(xm[row], xm[128 + row]);
        }
        // m_new = max(m, fp16(RN(rowmax * c))); a row with no visible key keeps m (-inf * c
        // rounds to -inf)
        const float mnew = fmaxf(m_run, f16_round(__fmul_rn(rmax, c)));
        // alpha = E(m - m_new), without branches: on the first tile m = -inf and the argument
        // is -inf (or NaN when m_new is -inf too), which E clamps to -127, so alpha = E(-127) = 0;
        // when the max is unchanged the argument is 0 and alpha = E(0) = 1 exactly
        const float alpha = exp2_own(__fsub_rn(m_run, mnew));
        const float negm = -mnew;
        const float2 c2 = make_float2(c, c), negm2 = make_float2(negm, negm);
        // O is rescaled by alpha_o: alpha, times 2^(k_prev - k) with the two-level scale
        float alpha_o = alpha, kinv = 1.0f, kpow = 1.0f;
        int k2 = 0;
        if constexpr (SUMP) {
          if (p.two_level) {
            // p_t = E(fma(rowmax S, c, -m_new)), the largest block amax of P (E monotone)
            const float pt = exp2_own(__fmaf_rn(rmax, c, negm));
            k2 = (int)((__float_as_uint(pt) >> 23) & 0xFFu) - 127 - 10;
            k2 = k2 < -40 ? -40 : k2;
            kinv = __uint_as_float((uint32_t)(127 - k2) << 23);
            kpow = __uint_as_float((uint32_t)(127 + k2) << 23);
            alpha_o = __fmul_rn(alpha, __uint_as_float((uint32_t)(127 + k_prev - k2) << 23));
          }
        }
        // block amax of P = E(fma(block max of S, c, -m_new)), two blocks per packed call
        float pmax[NB];
#pragma unroll
        for (int bl = 0; bl < NB; bl += 2) {
          const float2 e2 = exp2_own2(__ffma2_rn(make_float2(bmax[bl], bmax[bl + 1]), c2, negm2));
          pmax[bl] = e2.x;
          pmax[bl + 1] = e2.y;
        }
        uint32_t words[CW / 8];
        uint64_t sfw = 0;                    // the NB scale bytes, block bl in byte bl
        float part = 0.0f;                   // ablation kernels: this warpgroup's sum of P
        // the blocks' scales and codes
        {
#pragma unroll
          for (int bl = 0; bl < NB; ++bl) {
            float sarg = __fmul_rn(pmax[bl], kSixth);
            if constexpr (SUMP) sarg = __fmul_rn(sarg, kinv);
            const uint32_t sc = cvt_e4m3(sarg);
            sfw |= (uint64_t)sc << (8 * bl);
            if constexpr (FAST) {
              // B = (L(sigma) - m + 125) / 128; L(0) = -inf makes every code of the block 0
              const float B = __fmul_rn(__fadd_rn(__fsub_rn(rtab[sc], mnew), 125.0f), 0.0078125f);
#pragma unroll
              for (int h8 = 0; h8 < 2; ++h8) {
                float2 y[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int e = bl * 16 + h8 * 8 + 2 * k;
                  y[k] = phat_pair(make_float2(fma_sat(s[e], c7, B), fma_sat(s[e + 1], c7, B)));
                }
                words[2 * bl + h8] = encode8_pairs(y);
              }
            } else {
              // code = E2M1_RN(RN(P * R)), R = RN(1/sigma) (0 for sigma = 0); with the
              // two-level scale R = RN(1/(sigma 2^k)) = RN(1/sigma) 2^-k, exact
              float R = rtab[sc];
              if constexpr (SUMP) R = __fmul_rn(R, kinv);
              const float2 R2 = make_float2(R, R);
#pragma unroll
              for (int h8 = 0; h8 < 2; ++h8) {
                float2 y[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int e = bl * 16 + h8 * 8 + 2 * k;
                  const float2 x2 = __ffma2_rn(make_float2(s[e], s[e + 1]), c2, negm2);
                  const float2 e2 = exp2_own2(x2);
                  if constexpr (SUMP) part = __fadd_rn(__fadd_rn(part, e2.x), e2.y);
                  y[k] = __fmul2_rn(e2, R2);
                }
                words[2 * bl + h8] = encode8_pairs(y);
              }
            }
          }
        }
        float rsum = 0.0f;
        if constexpr (SUMP) {
          float* xs = xsum + (g & 1) * (C::NSW * 128);
          xs[wg * 128 + row] = part;
          named_bar(1 + q4, 32 * C::NSW);
          rsum = xs[row];
#pragma unroll
          for (int w2 = 1; w2 < C::NSW; ++w2) rsum = __fadd_rn(rsum, xs[w2 * 128 + row]);
        }
        uint8_t* pbuf = sP(pb);
#pragma unroll
        for (int q = 0; q < CW / 32; ++q)
          *reinterpret_cast<uint4*>(pbuf + p_off[q]) =
              make_uint4(words[4 * q], words[4 * q + 1], words[4 * q + 2], words[4 * q + 3]);
#pragma unroll
        for (int a = 0; a < NATOM; ++a) {
          uint8_t* atom = sPsf(pb) + psf_off + 512 * a;
          if (NB >= 4) *reinterpret_cast<uint32_t*>(atom) = (uint32_t)(sfw >> (32 * a));
          else *reinterpret_cast<uint16_t*>(atom) = (uint16_t)sfw;
        }
        fence_proxy_async_smem();
        if (jj > 0) {
          ok = wait_all(o_bar, (g - 1) & 1, abort, p.status, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          uint32_t rr[1] = {tmem_ld1(tbase + lrow + C::T_R)};
          tmem_wait_ld();
          reg_fence(rr);
          float r_use = __uint_as_float(rr[0]);
          if constexpr (SUMP) {
            r_use = __fmul_rn(r_use, kpow_prev);
            if (p.trace && wg == 0) {
              float* t = p.trace + ((ug.orow + row) * ntmax + (j - 1)) * 2;
              t[0] = r_use;
              t[1] = rsum_prev;
            }
            if (p.l_from_p) r_use = rsum_prev;
          }
          l_run = f16_round(__fmaf_rn(alpha_prev, l_run, r_use));
          if (__any_sync(0xffffffffu, alpha_o != 1.0f)) {
#pragma unroll 1
            for (int c0 = wg * OW; c0 < wg * OW + OW; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(tbase + lrow + C::T_O + c0, o);
              tmem_wait_ld();
              reg_fence(o);
              const float2 a2 = make_float2(alpha_o, alpha_o);
#pragma unroll
              for (int q = 0; q < 32; q += 2) {
                const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[q]), __uint_as_float(o[q + 1])), a2);
                o[q] = __float_as_uint(v.x);
                o[q + 1] = __float_as_uint(v.y);
              }
              tmem_st32(tbase + lrow + C::T_O + c0, o);
            }
            tmem_wait_st();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pb]);
        alpha_prev = alpha;
        m_run = mnew;
        rsum_prev = rsum;
        k_prev = k2;
        kpow_prev = kpow;
        if (jj == 0 && i > 0) {
          ok = epilogue(g - 1, pend_row, pend_l, pend_alpha, pend_rsum, pend_j, pend_kpow);
          if (!ok) break;
        }
      }
      if (!ok) break;
      pend_row = ug.orow + row;
      pend_l = l_run;
      pend_alpha = alpha_prev;
      pend_rsum = rsum_prev;
      pend_j = ug.j0 + nt - 1;
      pend_kpow = kpow_prev;
      if (wg == 0) {
        if constexpr (DEC) p.part_m[pend_row] = m_run;
        else if (p.m_out) p.m_out[pend_row] = __float2half_rn(m_run);
      }
    }
    if (ok && g > 0) ok = epilogue(g - 1, pend_row, pend_l, pend_alpha, pend_rsum, pend_j, pend_kpow);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- decode merge
// Merge of the split partials of one packed decode row per CTA (thread x = output channel
// x): m = max_s m_s, w_s = E(m_s - m) (0 when m_s = -inf), L = fma(w_s, l_s, L) and
// O = fma(w_s, O_s, O) over the splits in order, out = bf16(O * RN(1/L)), m and fp16(L)
// out.  o: [B, Hq, nq, D]; rows r = hi * nq + t of kv head g are token t of head g * G + hi.
struct DecodeMergeArgs {
  const float* part_o;
  const float* part_m;
  const float* part_l;
  __nv_bfloat16* o;
  __half* m_out;
  __half* l_out;
  int Hkv, G, nq, nsplit;
};

template <int D>
__global__ void __launch_bounds__(D) k_decode_merge(const DecodeMergeArgs a) {
  const int rows = a.G * a.nq;
  const int bkv = blockIdx.x / rows, r = blockIdx.x % rows, x = threadIdx.x;
  float m = -INFINITY;
  for (int s = 0; s < a.nsplit; ++s) m = fmaxf(m, a.part_m[((long long)bkv * a.nsplit + s) * 128 + r]);
  float L = 0.0f, O = 0.0f;
  for (int s = 0; s < a.nsplit; ++s) {
    const long long slot = ((long long)bkv * a.nsplit + s) * 128 + r;
    const float ms = a.part_m[slot];
    const float w = (ms == -INFINITY) ? 0.0f : exp2_own(__fsub_rn(ms, m));
    L = __fmaf_rn(w, a.part_l[slot], L);
    O = __fmaf_rn(w, a.part_o[slot * D + x], O);
  }
  const float inv = (L > 0.0f) ? __frcp_rn(L) : 0.0f;
  const int b = bkv / a.Hkv, g = bkv % a.Hkv, hi = r / a.nq, t = r % a.nq;
  const long long orow = ((long long)b * a.Hkv * a.G + g * a.G + hi) * a.nq + t;
  a.o[orow * D + x] = __float2bfloat16_rn(__fmul_rn(O, inv));
  if (x == 0) {
    if (a.m_out) a.m_out[orow] = __float2half_rn(m);
    if (a.l_out) a.l_out[orow] = __float2half_rn(L);
  }
}

#ifdef HIFA4_TEST_HOOKS
// ---------------------------------------------------------------- single-tile probes

// S = Q_hat K_hat^T of one 128 x BC tile through the same TMA / tcgen05.cp / MMA path as
// the attention kernel (QK half only), written out as fp32 [128][BC].
template <int D, int BC>
__global__ void __launch_bounds__(128, 1)
    k_probe_qk(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const uint8_t* qsf, const uint8_t* ksf, float* S, int* status, unsigned long long wait_ns) {
  using C = AttnCfg<D, BC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + align_up(C::SZ_Q, 1024);
  uint8_t* sQsf = sK + align_up(C::SZ_K, 1024);
  uint8_t* sKsf = sQsf + C::SZ_QSF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKsf + C::SZ_KSF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(bars + 3);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bars[0], C::SZ_Q + C::SZ_K + C::SZ_QSF + C::SZ_KSF);
    tma_load_2d(sQ, &tmQ, 0, 0, &bars[0]);
    tma_load_2d(sK, &tmK, 0, 0, &bars[0]);
    bulk_load(sQsf, qsf, C::SZ_QSF, &bars[0]);
    bulk_load(sKsf, ksf, C::SZ_KSF, &bars[0]);
  }
  bool ok = wait_all(&bars[0], 0, abort, status, wait_ns);
  if (ok && warp == 0) {
    tc_fence_after();
    if (lane == 0) {
      const uint32_t T_SFQ = BC, T_SFK = BC + 4 * C::KQ;
      for (int kc = 0; kc < C::KQ; ++kc) {
        tmem_cp_sf_atom(tbase + T_SFQ + 4 * kc, sQsf + 512 * kc);
        tmem_cp_sf_atom(tbase + T_SFK + 4 * kc, sKsf + 512 * kc);
      }
      for (int kc = 0; kc < C::KQ; ++kc)
        mma_nvf4(tbase, smem_desc(smem_u32(sQ) + 32 * kc, 0, 8 * C::QROW, C::LQ),
                 smem_desc(smem_u32(sK) + 32 * kc, 0, 8 * C::QROW, C::LQ), idesc_nvf4(128, BC),
                 tbase + T_SFQ + 4 * kc, tbase + T_SFK + 4 * kc, kc > 0 ? 1u : 0u);
      tc_commit(&bars[1]);
    }
    __syncwarp();
  }
  if (ok) ok = wait_all(&bars[1], 0, abort, status, wait_ns);
  if (ok) {
    tc_fence_after();
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    for (int c0 = 0; c0 < BC; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tbase + lrow + c0, r);
      tmem_wait_ld();
      reg_fence(r);
      for (int i = 0; i < 32; ++i) S[(warp * 32 + lane) * BC + c0 + i] = __uint_as_float(r[i]);
    }
  } else if (threadIdx.x == 0) {
    drain_wait(&bars[0], 0, status, wait_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

// O = P_hat V_hat (fp32 [128][D]) and R = P_hat * ones (fp32 [128]) of one tile through
// the attention kernel's PV path; P_hat arrives by TMA from a [128][BC/2] code tile.
template <int D, int BC>
__global__ void __launch_bounds__(128, 1)
    k_probe_pv(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmV, const uint8_t* psf,
               const uint8_t* vsf, float* O, float* Rout, int* status, unsigned long long wait_ns) {
  using C = AttnCfg<D, BC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sP = smem;
  uint8_t* sV = sP + align_up(C::SZ_P, 1024);
  uint8_t* sOnes = sV + align_up(C::SZ_V, 1024);
  uint8_t* sPsf = sOnes + align_up(C::SZ_ONES, 1024);
  uint8_t* sVsf = sPsf + C::SZ_PSF;
  uint8_t* s1sf = sVsf + C::SZ_VSF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s1sf + 512);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(bars + 3);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < (int)C::SZ_ONES / 4; i += 128) reinterpret_cast<uint32_t*>(sOnes)[i] = 0x22222222u;
  for (int i = threadIdx.x; i < 128; i += 128) reinterpret_cast<uint32_t*>(s1sf)[i] = 0x38383838u;
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  constexpr uint32_t T_O = 0, T_R = D, T_SFP = D + 16, T_SFV = T_SFP + 4 * C::KP, T_SF1 = T_SFV + 4 * C::KP * C::NAV;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bars[0], C::SZ_P + C::SZ_V + C::SZ_PSF + C::SZ_VSF);
    tma_load_2d(sP, &tmP, 0, 0, &bars[0]);
    tma_load_2d(sV, &tmV, 0, 0, &bars[0]);
    bulk_load(sPsf, psf, C::SZ_PSF, &bars[0]);
    bulk_load(sVsf, vsf, C::SZ_VSF, &bars[0]);
  }
  bool ok = wait_all(&bars[0], 0, abort, status, wait_ns);
  if (ok && warp == 0) {
    tc_fence_after();
    if (lane == 0) {
      for (int i = 0; i < C::KP; ++i) tmem_cp_sf_atom(tbase + T_SFP + 4 * i, sPsf + 512 * i);
      for (int i = 0; i < C::KP * C::NAV; ++i) tmem_cp_sf_atom(tbase + T_SFV + 4 * i, sVsf + 512 * i);
      tmem_cp_sf_atom(tbase + T_SF1, s1sf);
      for (int kc = 0; kc < C::KP; ++kc)
        mma_nvf4(tbase + T_O, smem_desc(smem_u32(sP) + 32 * kc, 0, 8 * C::PROW, C::LP),
                 smem_desc(smem_u32(sV) + 32 * kc, 0, 8 * C::PROW, C::LP), idesc_nvf4(128, D),
                 tbase + T_SFP + 4 * kc, tbase + T_SFV + 4 * C::NAV * kc, kc > 0 ? 1u : 0u);
      for (int kc = 0; kc < C::KP; ++kc)
        mma_nvf4(tbase + T_R, smem_desc(smem_u32(sP) + 32 * kc, 0, 8 * C::PROW, C::LP),
                 smem_desc(smem_u32(sOnes) + 32 * kc, 0, 8 * C::PROW, C::LP), idesc_nvf4(128, 16),
                 tbase + T_SFP + 4 * kc, tbase + T_SF1, kc > 0 ? 1u : 0u);
      tc_commit(&bars[1]);
    }
    __syncwarp();
  }
  if (ok) ok = wait_all(&bars[1], 0, abort, status, wait_ns);
  if (ok) {
    tc_fence_after();
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tbase + lrow + T_O + c0, r);
      tmem_wait_ld();
      reg_fence(r);
      for (int i = 0; i < 32; ++i) O[(warp * 32 + lane) * D + c0 + i] = __uint_as_float(r[i]);
    }
    uint32_t rr[1] = {tmem_ld1(tbase + lrow + T_R)};
    tmem_wait_ld();
    reg_fence(rr);
    Rout[warp * 32 + lane] = __uint_as_float(rr[0]);
  } else if (threadIdx.x == 0) {
    drain_wait(&bars[0], 0, status, wait_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int D, int BC>
constexpr uint32_t probe_qk_smem() {
  using C = AttnCfg<D, BC>;
  return align_up(C::SZ_Q, 1024) + align_up(C::SZ_K, 1024) + C::SZ_QSF + C::SZ_KSF + 64 + 1024;
}
template <int D, int BC>
constexpr uint32_t probe_pv_smem() {
  using C = AttnCfg<D, BC>;
  return align_up(C::SZ_P, 1024) + align_up(C::SZ_V, 1024) + align_up(C::SZ_ONES, 1024) + C::SZ_PSF + C::SZ_VSF +
         512 + 64 + 1024;
}

// P_hat of 16-key blocks by the attention kernel's device steps: block b holds the scores
// S[16b .. 16b+15] of a row whose running max after the tile is m[b] (an FP16 value).  The
// block scale comes from E(fma(block max, c, -m)), the codes from the default rule
// E2M1_RN(RN(E(RN(fma(S, c, -m))) * RN(1/sigma))) or, with FAST, from the fast entry
// point's linear-mantissa rule.  Writes the E4M3 scale code and 16 E2M1 codes (one per
// byte) per block.
struct PhatProbeArgs {
  const float* S;
  const float* m;
  int nblk;
  float c;
  float lneg[128];
  uint8_t* codes;
  uint8_t* scales;
};

template <bool FAST>
__global__ void k_probe_phat(const PhatProbeArgs a) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < a.nblk; b += gridDim.x * blockDim.x) {
    float s[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) s[e] = a.S[16 * b + e];
    float bm = s[0];
#pragma unroll
    for (int e = 1; e < 15; e += 2) bm = fmax3(bm, s[e], s[e + 1]);
    bm = fmaxf(bm, s[15]);
    const float mnew = a.m[b], negm = -mnew;
    const float c = a.c, c7 = c * 0.0078125f;
    const float2 c2 = make_float2(c, c), negm2 = make_float2(negm, negm);
    const float pmax = exp2_own2(__ffma2_rn(make_float2(bm, bm), c2, negm2)).x;
    const uint32_t sc = cvt_e4m3(__fmul_rn(pmax, kSixth));
    uint32_t words[2];
    if constexpr (FAST) {
      const float B = __fmul_rn(__fadd_rn(__fsub_rn(a.lneg[sc], mnew), 125.0f), 0.0078125f);
#pragma unroll
      for (int h8 = 0; h8 < 2; ++h8) {
        float2 y[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = h8 * 8 + 2 * k;
          y[k] = phat_pair(make_float2(fma_sat(s[e], c7, B), fma_sat(s[e + 1], c7, B)));
        }
        words[h8] = encode8_pairs(y);
      }
    } else {
      const float sv = e4m3_value(sc);
      const float R = (sv > 0.0f && sv <= 448.0f) ? __frcp_rn(sv) : 0.0f;
      const float2 R2 = make_float2(R, R);
#pragma unroll
      for (int h8 = 0; h8 < 2; ++h8) {
        float2 y[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = h8 * 8 + 2 * k;
          y[k] = __fmul2_rn(exp2_own2(__ffma2_rn(make_float2(s[e], s[e + 1]), c2, negm2)), R2);
        }
        words[h8] = encode8_pairs(y);
      }
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) a.codes[16 * b + e] = (uint8_t)((words[e >> 3] >> (4 * (e & 7))) & 0xFu);
    a.scales[b] = (uint8_t)sc;
  }
}

// Elementwise codec check: the device E2M1 / E4M3 conversions and the exp2 on given inputs.
__global__ void k_probe_codec(const float* x, int n, uint8_t* e2m1, uint8_t* e4m3, float* ex2) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float v = x[i];
    e2m1[i] = (uint8_t)(cvt_e2m1x2(0.0f, v) & 0xF);
    e4m3[i] = (uint8_t)cvt_e4m3(fabsf(v));
    ex2[i] = exp2_own(v);
  }
}

#endif  // HIFA4_TEST_HOOKS

#ifdef HIFA4_TEST_HOOKS
// The same conversions on the n consecutive fp32 bit patterns start, start + 1, ...
// (inputs generated on the device, so a whole range needs no input buffer).
__global__ void k_probe_codec_range(uint32_t start, long long n, uint8_t* e2m1, uint8_t* e4m3) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = __uint_as_float(start + (uint32_t)i);
    e2m1[i] = (uint8_t)(cvt_e2m1x2(0.0f, v) & 0xF);
    e4m3[i] = (uint8_t)cvt_e4m3(fabsf(v));
  }
}
#endif  // HIFA4_TEST_HOOKS

}  // namespace hifa4

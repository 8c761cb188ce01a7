// Decode / split-KV attention with the keys on the MMA's M dimension ("transposed" form)
// for head dim 128 and at most 16 packed query rows (G * nq <= 16).
//
// The split-KV tile loop of k_attn_fwd<.., DEC = true> computes S = Q_hat K_hat^T with the
// 128 packed query rows on M: with one new token per sequence only G of those rows hold
// queries, and every softmax warp still works through a full 128-row tile.  Here the same
// per-row recursion runs on the transposed products:
//   S^T = K_hat_j Q_hat^T       (M = 128 keys, N = 16 query rows, K = d)
//   O^T += V_hat_j^T P_hat^T    (M = d = 128 channels, N = 16, K = 128 keys)
//   R^T  = 1 P_hat^T            (ones on M: every TMEM lane receives the row sums of P_hat)
// so a softmax thread holds one key (S^T) and one channel (O^T) for NQ query rows.  The
// 4-bit products and their accumulation per 64-wide K step are the same as in the
// untransposed MMA, and every other step (m, alpha, block scales, P_hat codes, the FP16 l
// recursion, the partial outputs) follows the k_attn_fwd definitions with a 128-key tile,
// so the results equal that kernel's at kv_tile = 128.
//
// Roles (224 threads): warp 0 TMA producer, warp 1 QK^T issuer and TMEM owner, warp 2 PV
// issuer, warps 3..6 softmax (warp w reads TMEM lane quarter w & 3: keys 32 (w & 3) ..
// +31 of S^T, channels 32 (w & 3) .. +31 of O^T).  Per tile a softmax warp takes the
// column maxima of its 32 keys with one integer max-reduction per query row, combines
// the four warps' maxima through shared memory, forms the 16-key block maxima with four
// shuffle rounds, and packs the codes of neighbouring keys into bytes of the P_hat^T
// operand; each of these steps runs over all NQ rows before the next, so the rows'
// dependency chains overlap.  With so little work per tile, latency is hidden by running
// three CTAs per SM (73 KB of shared memory and 128 TMEM columns each).  Every wait is
// bounded, as in k_attn_fwd.
#pragma once
#include "attn.cuh"

namespace hifa4 {

struct DecTCfg {
  static constexpr int D = 128, BC = 128, NMMA = 16;
  static constexpr int KQ = D / 64, KP = BC / 64;
  static constexpr int QROW = D / 2, PROW = BC / 2;                 // 64-byte operand rows
  static constexpr uint32_t LQ = layout_code(QROW), LP = layout_code(PROW);
  static constexpr int KS = 3, VS = 3;
  static constexpr uint32_t SZ_Q = NMMA * QROW, SZ_K = BC * QROW, SZ_V = D * PROW, SZ_P = NMMA * PROW;
  static constexpr uint32_t SZ_ONES = 128 * PROW;
  static constexpr uint32_t SZ_QSF = KQ * 512, SZ_KSF = KQ * 512, SZ_VSF = KP * 512, SZ_PSF = KP * 512;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + 2 * 1024;
  static constexpr uint32_t OFF_V = OFF_K + KS * SZ_K;
  static constexpr uint32_t OFF_P = OFF_V + VS * SZ_V;
  static constexpr uint32_t OFF_ONES = OFF_P + 2 * 1024;
  static constexpr uint32_t OFF_QSF = OFF_ONES + SZ_ONES;
  static constexpr uint32_t OFF_KSF = OFF_QSF + 2 * SZ_QSF;
  static constexpr uint32_t OFF_VSF = OFF_KSF + KS * SZ_KSF;
  static constexpr uint32_t OFF_PSF = OFF_VSF + VS * SZ_VSF;
  static constexpr uint32_t OFF_1SF = OFF_PSF + 2 * SZ_PSF;
  static constexpr uint32_t OFF_RTAB = OFF_1SF + 512;               // 128 x fp32 RN(1/sigma)
  static constexpr uint32_t OFF_XMAX = OFF_RTAB + 512;              // [2][4 warps][16] fp32 column maxima
  static constexpr uint32_t OFF_BAR = OFF_XMAX + 2 * 4 * 16 * 4;
  // barriers: q_full[2], q_empty[2], k_full[KS], k_empty[KS], v_full[VS], v_empty[VS],
  // s_full[2], s_empty[2], p_full[2], o_bar, o_free, drain[2]
  static constexpr int NBAR = 4 + 2 * KS + 2 * VS + 6 + 4;
  static constexpr uint32_t OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;             // + slack for 1024-B alignment
  // TMEM columns: S^T double-buffered, O^T, R^T, scale factors
  static constexpr uint32_t T_S = 0, T_O = 2 * NMMA, T_R = T_O + NMMA, T_SFQ = T_R + NMMA;
  static constexpr uint32_t T_SFK = T_SFQ + 4 * KQ, T_SFV = T_SFK + 2 * 4 * KQ, T_SFP = T_SFV + 2 * 4 * KP;
  static constexpr uint32_t T_SF1 = T_SFP + 2 * 4 * KP, T_END = T_SF1 + 4;
  static constexpr uint32_t TMEM_COLS = 128;
  static_assert(T_END <= TMEM_COLS, "TMEM budget exceeded");
  static constexpr int NTHREADS = 96 + 128;
};

// 32 lanes x N consecutive 32-bit TMEM columns -> N registers per thread (N = 4, 8, 16).
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else {
    static_assert(N == 16, "tmem_ldn width");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  }
}

template <int N>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 4) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
  } else {
    static_assert(N == 16, "tmem_stn width");
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
  }
}

// Maximum of x over the 32 lanes of the warp (-inf allowed; no NaN), through the
// order-preserving map of fp32 bit patterns onto int32 and one integer max-reduction.
__device__ __forceinline__ float warp_max_f32(float x) {
  int k = __float_as_int(x);
  k ^= (k >> 31) & 0x7FFFFFFF;
  int r;
  asm volatile("redux.sync.max.s32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(k));
  r ^= (r >> 31) & 0x7FFFFFFF;
  return __int_as_float(r);
}

template <int NQ>
__global__ void __launch_bounds__(DecTCfg::NTHREADS, NQ == 16 ? 2 : 3)
    k_attn_decode_t(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = DecTCfg;
  constexpr int D = C::D, BC = C::BC;
  static_assert(NQ == 4 || NQ == 8 || NQ == 16, "query columns");
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
  auto sQ = [&](int s) { return smem + C::OFF_Q + s * 1024; };
  auto sQsf = [&](int s) { return smem + C::OFF_QSF + s * C::SZ_QSF; };
  auto sK = [&](int s) { return smem + C::OFF_K + s * C::SZ_K; };
  auto sV = [&](int s) { return smem + C::OFF_V + s * C::SZ_V; };
  auto sP = [&](int s) { return smem + C::OFF_P + s * 1024; };
  auto sKsf = [&](int s) { return smem + C::OFF_KSF + s * C::SZ_KSF; };
  auto sVsf = [&](int s) { return smem + C::OFF_VSF + s * C::SZ_VSF; };
  auto sPsf = [&](int s) { return smem + C::OFF_PSF + s * C::SZ_PSF; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = p.B * p.Hkv * p.nsplit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBAR; ++i) {
      const bool per_warp = (&bars[i] == &s_empty[0] || &bars[i] == &s_empty[1] || &bars[i] == &p_full[0] ||
                             &bars[i] == &p_full[1] || &bars[i] == o_free);
      mbar_init(&bars[i], per_warp ? 4 : 1);   // one arrival per softmax warp
    }
    *abort = 0;
    fence_mbar_init();
  }
  float* rtab = reinterpret_cast<float*>(smem + C::OFF_RTAB);
  float* xmax = reinterpret_cast<float*>(smem + C::OFF_XMAX);
  if (warp >= 3) {
    // the ones operand (E2M1 1.0 in both nibbles) and its scales (UE4M3 1.0); the P_hat^T
    // buffers and their scale atoms start at zero (rows NQ..15 stay zero)
    const int t = threadIdx.x - 96;
    for (int i = t; i < (int)C::SZ_ONES / 4; i += 128) reinterpret_cast<uint32_t*>(sOnes)[i] = 0x22222222u;
    for (int i = t; i < 128; i += 128) reinterpret_cast<uint32_t*>(s1sf)[i] = 0x38383838u;
    for (int i = t; i < 2 * 1024 / 4; i += 128) reinterpret_cast<uint32_t*>(smem + C::OFF_P)[i] = 0u;
    for (int i = t; i < 2 * (int)C::SZ_PSF / 4; i += 128) reinterpret_cast<uint32_t*>(smem + C::OFF_PSF)[i] = 0u;
    fence_proxy_async_smem();
    for (int i = t; i < 128; i += 128) {   // RN(1/sigma) per E4M3 scale code (0 for sigma = 0)
      const float sv = e4m3_value((uint32_t)i);
      rtab[i] = (sv > 0.0f && sv <= 448.0f) ? __frcp_rn(sv) : 0.0f;
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
      int nq = 0, nk = 0, nv = 0;
      bool ok = true;
      for (int i = 0, u = blockIdx.x; ok && u < units; u += gridDim.x, ++i) {
        const UnitGeom ug = unit_geom<BC, true>(u, p);
        const int kvh = ug.kvh;
        const int qb = i & 1;
        if (i >= 2 && !mbar_wait(&q_empty[qb], ((i >> 1) - 1) & 1, abort, p.status, p.wait_ns)) break;
        mbar_arrive_expect_tx(&q_full[qb], C::SZ_Q + C::SZ_QSF);
        tma_load_2d(sQ(qb), &tmQ, 0, ug.qrow, &q_full[qb]);
        bulk_load(sQsf(qb), p.qsf + (long long)(ug.qrow / 128) * C::SZ_QSF, C::SZ_QSF, &q_full[qb]);
        ++nq;
        for (int jj = 0; jj < ug.nt; ++jj) {
          const int j = ug.j0 + jj;
          const int g = nk, ks = g % C::KS, vs = g % C::VS;
          if (g >= C::KS && !mbar_wait(&k_empty[ks], ((g / C::KS) - 1) & 1, abort, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[ks], C::SZ_K + C::SZ_KSF);
          tma_load_2d(sK(ks), &tmK, 0, kvh * p.Nk + j * BC, &k_full[ks]);
          bulk_load(sKsf(ks), p.ksf + ((long long)kvh * (p.Nk / 128) + j) * (C::KQ * 512), C::SZ_KSF, &k_full[ks]);
          ++nk;
          if (g >= C::VS && !mbar_wait(&v_empty[vs], ((g / C::VS) - 1) & 1, abort, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[vs], C::SZ_V + C::SZ_VSF);
          tma_load_2d(sV(vs), &tmV, j * C::PROW, kvh * D, &v_full[vs]);
          bulk_load(sVsf(vs), p.vsf + ((long long)kvh * (p.Nk / 64) + j * C::KP) * 512, C::SZ_VSF, &v_full[vs]);
          ++nv;
        }
      }
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
    // S^T_g = K_hat_g Q_hat^T into S buffer g & 1 (A = the K tile, B = the 16 query rows)
    constexpr uint32_t ID = idesc_nvf4(128, C::NMMA);
    const uint64_t dQ = smem_desc(smem_u32(sQ(0)), 0, 8 * C::QROW, C::LQ);
    const uint64_t dK = smem_desc(smem_u32(sK(0)), 0, 8 * C::QROW, C::LQ);
    const uint64_t dQsf = smem_desc(smem_u32(sQsf(0)), 0, 128, 0);
    const uint64_t dKsf = smem_desc(smem_u32(sKsf(0)), 0, 128, 0);
    bool ok = true;
    int g = 0;
    for (int i = 0, u = blockIdx.x; ok && u < units; u += gridDim.x, ++i) {
      const int nt = unit_geom<BC, true>(u, p).nt;
      const int qb = i & 1;
      ok = wait_all(&q_full[qb], (i >> 1) & 1, abort, p.status, p.wait_ns);
      if (ok && i >= 1) ok = wait_all(&q_empty[qb ^ 1], ((i - 1) >> 1) & 1, abort, p.status, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kc = 0; kc < C::KQ; ++kc)
          tmem_cp_sf(tbase + C::T_SFQ + 4 * kc, dQsf + ((qb * C::SZ_QSF + 512 * kc) >> 4));
      }
      __syncwarp();
      const uint64_t dQi = dQ + ((qb * 1024) >> 4);
      for (int jj = 0; ok && jj < nt; ++jj, ++g) {
        const int ks = g % C::KS, sb = g & 1;
        ok = wait_all(&k_full[ks], (g / C::KS) & 1, abort, p.status, p.wait_ns);
        if (ok && g >= 2) ok = wait_all(&s_empty[sb], ((g >> 1) - 1) & 1, abort, p.status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sfk = tbase + C::T_SFK + (g & 1) * 4 * C::KQ;
          const uint64_t dKsfs = dKsf + ((ks * C::SZ_KSF) >> 4);
#pragma unroll
          for (int kc = 0; kc < C::KQ; ++kc) tmem_cp_sf(sfk + 4 * kc, dKsfs + ((512 * kc) >> 4));
          const uint64_t dKs = dK + ((ks * C::SZ_K) >> 4);
#pragma unroll
          for (int kc = 0; kc < C::KQ; ++kc)
            mma_nvf4(tbase + C::T_S + sb * C::NMMA, dKs + 2 * kc, dQi + 2 * kc, ID, sfk + 4 * kc,
                     tbase + C::T_SFQ + 4 * kc, kc > 0 ? 1u : 0u);
          tc_commit(&s_full[sb]);
          tc_commit(&k_empty[ks]);
          if (jj == nt - 1) tc_commit(&q_empty[qb]);
        }
        __syncwarp();
      }
    }
    if (lane == 0) {
      tc_commit(&drain_bar[0]);
      drain_wait(&drain_bar[0], 0, p.status, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ PV issuer
    // O^T (+)= V_hat_g^T P_hat_g^T and R^T = 1 P_hat_g^T once the softmax warps have
    // written P_hat_g and rescaled O^T (p_full)
    constexpr uint32_t ID = idesc_nvf4(128, C::NMMA);
    const uint64_t dP = smem_desc(smem_u32(sP(0)), 0, 8 * C::PROW, C::LP);
    const uint64_t dV = smem_desc(smem_u32(sV(0)), 0, 8 * C::PROW, C::LP);
    const uint64_t dOnes = smem_desc(smem_u32(sOnes), 0, 8 * C::PROW, C::LP);
    const uint64_t dPsf = smem_desc(smem_u32(sPsf(0)), 0, 128, 0);
    const uint64_t dVsf = smem_desc(smem_u32(sVsf(0)), 0, 128, 0);
    tc_fence_after();
    if (lane == 0) tmem_cp_sf(tbase + C::T_SF1, smem_desc(smem_u32(s1sf), 0, 128, 0));
    __syncwarp();
    bool ok = true;
    int g = 0;
    for (int i = 0, u = blockIdx.x; ok && u < units; u += gridDim.x, ++i) {
      const int nt = unit_geom<BC, true>(u, p).nt;
      for (int jj = 0; ok && jj < nt; ++jj, ++g) {
        const int vs = g % C::VS, pb = g & 1;
        ok = wait_all(&v_full[vs], (g / C::VS) & 1, abort, p.status, p.wait_ns);
        ok = ok && wait_all(&p_full[pb], (g >> 1) & 1, abort, p.status, p.wait_ns);
        if (ok && jj == 0 && i >= 1) ok = wait_all(o_free, (i - 1) & 1, abort, p.status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sfv = tbase + C::T_SFV + pb * 4 * C::KP;
          const uint32_t sfp = tbase + C::T_SFP + pb * 4 * C::KP;
          const uint64_t dVsfs = dVsf + ((vs * C::SZ_VSF) >> 4), dPsfs = dPsf + ((pb * C::SZ_PSF) >> 4);
#pragma unroll
          for (int kc = 0; kc < C::KP; ++kc) {
            tmem_cp_sf(sfv + 4 * kc, dVsfs + 32 * kc);
            tmem_cp_sf(sfp + 4 * kc, dPsfs + 32 * kc);
          }
          const uint64_t dPs = dP + ((pb * 1024) >> 4);
          const uint64_t dVs = dV + ((vs * C::SZ_V) >> 4);
#pragma unroll
          for (int kc = 0; kc < C::KP; ++kc)
            mma_nvf4(tbase + C::T_O, dVs + 2 * kc, dPs + 2 * kc, ID, sfv + 4 * kc, sfp + 4 * kc,
                     (jj > 0 || kc > 0) ? 1u : 0u);
#pragma unroll
          for (int kc = 0; kc < C::KP; ++kc)
            mma_nvf4(tbase + C::T_R, dOnes + 2 * kc, dPs + 2 * kc, ID, tbase + C::T_SF1, sfp + 4 * kc,
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
    const int q4 = warp & 3;                        // TMEM lane quarter
    const uint32_t lrow = (uint32_t)(q4 * 32) << 16;
    const int b8 = 2 * q4 + (lane >> 4);            // this lane's 16-key block of the tile
    const float c = p.c;
    const int nv = p.G * p.nq;                      // query rows in use
    // the last key query column q sees: the decode position of its token; unused columns
    // see every key (their Q rows are zero), which keeps their arithmetic finite
    int qpos[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) qpos[q] = q < nv ? p.Nk - p.nq + q % p.nq : p.Nk - 1;
    const int pos_min = p.Nk - p.nq;
    bool ok = true;
    int g = 0;
    for (int i = 0, u = blockIdx.x; ok && u < units; u += gridDim.x, ++i) {
      const UnitGeom ug = unit_geom<BC, true>(u, p);
      float m_run[NQ], l_run[NQ], a_prev[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        m_run[q] = -INFINITY;
        l_run[q] = 0.0f;
        a_prev[q] = 0.0f;
      }
      for (int jj = 0; jj < ug.nt; ++jj, ++g) {
        const int j = ug.j0 + jj;
        const int sb = g & 1, pb = g & 1;
        ok = wait_all(&s_full[sb], (g >> 1) & 1, abort, p.status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        float s[NQ];
        {
          uint32_t r[NQ];
          tmem_ldn<NQ>(tbase + lrow + C::T_S + sb * C::NMMA, r);
          tmem_wait_ld();
          reg_fence(r);
#pragma unroll
          for (int q = 0; q < NQ; ++q) s[q] = __uint_as_float(r[q]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
        const int key = j * BC + q4 * 32 + lane;
        if ((j + 1) * BC - 1 > pos_min) {
#pragma unroll
          for (int q = 0; q < NQ; ++q)
            if (key > qpos[q]) s[q] = -INFINITY;
        }
        // column (query row) maxima: this warp's 32 keys, then the four warps
        float* xm = xmax + (g & 1) * (4 * 16);
        {
          float wm[NQ];
#pragma unroll
          for (int q = 0; q < NQ; ++q) wm[q] = warp_max_f32(s[q]);
          if (lane == 0) {
#pragma unroll
            for (int q = 0; q < NQ; q += 4)
              *reinterpret_cast<float4*>(xm + q4 * 16 + q) = make_float4(wm[q], wm[q + 1], wm[q + 2], wm[q + 3]);
          }
        }
        named_bar(1, 128);
        float mnew[NQ], alpha[NQ];
#pragma unroll
        for (int q = 0; q < NQ; q += 4) {
          float4 r4 = *reinterpret_cast<const float4*>(xm + q);
#pragma unroll
          for (int w2 = 1; w2 < 4; ++w2) {
            const float4 t = *reinterpret_cast<const float4*>(xm + w2 * 16 + q);
            r4 = make_float4(fmaxf(r4.x, t.x), fmaxf(r4.y, t.y), fmaxf(r4.z, t.z), fmaxf(r4.w, t.w));
          }
          const float rm[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int qq = q + e;
            // branch-free: a row with no visible key keeps m (-inf * c rounds to -inf); E clamps
            // the first tile's argument (-inf, or NaN when m_new is -inf too) to -127, so
            // alpha = 0 there, and alpha = E(0) = 1 exactly when the max is unchanged
            const float mn = fmaxf(m_run[qq], f16_round(__fmul_rn(rm[e], c)));
            mnew[qq] = mn;
            alpha[qq] = exp2_own(__fsub_rn(m_run[qq], mn));
          }
        }
        // P_hat^T: per query row q the 16-key block of this lane (lanes 0-15 / 16-31); even
        // lanes pack the codes of keys k, k + 1 into one byte.  Each step runs over all rows
        // before the next, so the rows' dependency chains overlap.
        uint8_t* pbuf = sP(pb);
        uint8_t* patom = sPsf(pb) + 512 * (b8 >> 2);
        float bm[NQ];
#pragma unroll
        for (int q = 0; q < NQ; ++q) bm[q] = s[q];
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) {
#pragma unroll
          for (int q = 0; q < NQ; ++q) bm[q] = fmaxf(bm[q], __shfl_xor_sync(0xffffffffu, bm[q], off));
        }
        float y[NQ];
        uint32_t sc[NQ];
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float pmax = exp2_own(__fmaf_rn(bm[q], c, -mnew[q]));
          sc[q] = cvt_e4m3(__fmul_rn(pmax, kSixth));
        }
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          // code = E2M1_RN(RN(P * RN(1/sigma))), P = E(RN(fma(S, c, -m_new))); sigma = 0
          // has R = 0, so every code of that block is 0
          y[q] = __fmul_rn(exp2_own(__fmaf_rn(s[q], c, -mnew[q])), rtab[sc[q]]);
        }
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float yn = __shfl_xor_sync(0xffffffffu, y[q], 1);   // the next key's value
          if ((lane & 1) == 0) pbuf[swz_offset(q, q4, C::PROW) + (lane >> 1)] = (uint8_t)cvt_e2m1x2(yn, y[q]);
          if ((lane & 15) == 0) patom[sf_atom_offset(q, b8 & 3)] = (uint8_t)sc[q];
        }
        fence_proxy_async_smem();
        if (jj > 0) {
          ok = wait_all(o_bar, (g - 1) & 1, abort, p.status, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          // l from R^T of PV_{j-1} (every lane holds the row sums), then O^T *= alpha
          uint32_t rr[NQ];
          tmem_ldn<NQ>(tbase + lrow + C::T_R, rr);
          tmem_wait_ld();
          reg_fence(rr);
#pragma unroll
          for (int q = 0; q < NQ; ++q) l_run[q] = f16_round(__fmaf_rn(a_prev[q], l_run[q], __uint_as_float(rr[q])));
          bool resc = false;
#pragma unroll
          for (int q = 0; q < NQ; ++q) resc |= alpha[q] != 1.0f;
          if (resc) {
            uint32_t o[NQ];
            tmem_ldn<NQ>(tbase + lrow + C::T_O, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int q = 0; q < NQ; ++q) o[q] = __float_as_uint(__fmul_rn(__uint_as_float(o[q]), alpha[q]));
            tmem_stn<NQ>(tbase + lrow + C::T_O, o);
            tmem_wait_st();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pb]);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          a_prev[q] = alpha[q];
          m_run[q] = mnew[q];
        }
      }
      if (!ok) break;
      // the unit's partial: unnormalised fp32 O^T, m and l of its rows in use
      ok = wait_all(o_bar, (g - 1) & 1, abort, p.status, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      uint32_t rr[NQ], o[NQ];
      tmem_ldn<NQ>(tbase + lrow + C::T_R, rr);
      tmem_ldn<NQ>(tbase + lrow + C::T_O, o);
      tmem_wait_ld();
      reg_fence(rr);
      reg_fence(o);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
      const int ch = q4 * 32 + lane;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        if (q < nv) {
          const long long orow = ug.orow + q;
          p.part_o[orow * D + ch] = __uint_as_float(o[q]);
          if (q4 == 0 && lane == 0) {
            p.part_m[orow] = m_run[q];
            p.part_l[orow] = f16_round(__fmaf_rn(a_prev[q], l_run[q], __uint_as_float(rr[q])));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace hifa4

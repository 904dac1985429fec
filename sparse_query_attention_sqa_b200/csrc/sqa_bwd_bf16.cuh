// sqa_bwd_bf16.cuh -- Sparse Query Attention backward for head dims 64 and 128
// (bf16 gradient MMAs; the dh = 128 larger-model shapes), as two kernels:
//
//   sqa_bwd_kernel    dK and dV, key-major (this file, first half)
//   sqa_bwd_q_kernel  dQ, query-major (second half)
//
// dQ is not accumulated by the key-major kernel: each (Q tile, key tile) pair
// would add a 128 x dh fp32 tile to dQ through L2 reductions, |dQ| times the
// number of key tiles in all (137 GB at B = 2, N = 65536, dh = 128), and the
// reductions, not the tensor core, then set the pace.  The query-major kernel
// recomputes S and dP for its Q tile (two more MMAs per pair) and keeps dQ in
// TMEM, so no gradient goes through atomics at these head dims.
//
// ---------------------------------------------------------------------------
// sqa_bwd_kernel<DH, LO>: work item, one CTA each, a 128-key tile of one (batch,
// KV head).  K and V stay in shared memory; the stacked Q tiles that see the
// keys (the g query heads of the group, row r = t * g + head) stream through
// two Q / dO stages.  Because a Q tile holds every head of the group, dV +=
// P^T dO and dK += dS^T Q contract over (token, head) rows at once: the
// reduction of dK and dV over the query-head group happens inside the
// tensor-core accumulation in TMEM (GQA summary, "The idea": the heads of a
// group share one key and one value head).
//
//   TMEM  [0, 128)    S^T (fp32), rewritten in place as P^T (bf16 pairs; for
//                     groups of kBwdSplitGroup or more also the remainders,
//                     in the columns the packed pairs leave)
//         [128, 256)  dP^T (fp32), rewritten in place as dS^T (bf16 pairs, the
//                     same way)
//         [256, ...)  dV, then dK (fp32, dh columns each)
//
//   Per Q tile i, in the issuing thread's order (MMAs of one thread run in
//   order, so a later MMA never overtakes an earlier one's reads):
//     dV += P^T_i dO_i, in two halves of 64 query rows, each as soon as the
//         softmax warps have written that half of P^T (p_ready)
//     S^T_{i+1} = K Q_{i+1}^T into the columns P^T_i leaves -> s_full
//     dK += dS^T_i Q_i  (after ds_ready)
//     dP^T_{i+1} = V dO_{i+1}^T into the columns dS^T_i leaves -> dp_full
//   so the tensor core always has the next product while the softmax warps
//   compute P^T (during dP^T) and dS^T (during dV and S^T).
//
// Roles (384 threads):
//   warp 0      TMA producer: K and V once; Q / dO tiles into two stages; the
//               tile's softmax statistics (-lse * log2 e and -D) into one buffer
//               each, refilled as soon as the previous tile's warps are done
//   warp 1      TMEM allocator and MMA issuer (the whole warp runs the loop; one
//               elected lane issues)
//   warps 2-3   idle
//   warps 4-11  two warpgroups: for each half of 64 query rows, warpgroup w
//               takes 32 of them (one key per TMEM lane); the dK / dV epilogue
#pragma once

#include "sqa_bwd.cuh"
#include "sqa_tmem_wide.cuh"

namespace sqa {

// From this group size on, the dK / dV kernel carries P^T and dS^T as bf16
// pairs hi + lo (split_bf16x2) and issues each dV / dK MMA twice.  Each dV or
// dK element sums g rows of every Q tile, and under a causal mask the first
// keys of a sequence take P near 1 from all g heads of the first tokens: with
// P rounded once to bf16 (relative error up to 2^-9) the largest dV errors
// below magnitude 4 grow with g, 0.014 at g = 6 and 0.020 at g = 7 (dh 64)
// and 0.032 at g = 16 (dh 128); the remainder brings them to the 1e-5 range,
// for 1.5 times the tensor work of this kernel.
constexpr int kBwdSplitGroup = 6;

template <int DH>
struct BwdBf16Traits {
  static_assert(DH == 64 || DH == 128, "bf16 backward handles dh 64 and 128");
  static constexpr int BM = kBwdTile, NK = kBwdTile;
  static constexpr int PANEL = 64;  // bf16 elements per 128-byte swizzled row segment
  static constexpr int NPANEL = DH / PANEL;
  static constexpr int ROWB = 128;
  static constexpr uint32_t LAYOUT = 2u;     // 128-byte swizzle
  static constexpr int TILE = 128 * DH * 2;  // one Q, dO, K or V tile
  static constexpr int QS = 2;               // Q / dO stages
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;
  static constexpr int OFF_DO = OFF_Q + QS * TILE;
  static constexpr int OFF_LSE = OFF_DO + QS * TILE;  // -lse2 of the current tile's 128 rows
  static constexpr int OFF_D = OFF_LSE + 512;         // -D of the current tile's rows
  static constexpr int OFF_RTOK = OFF_D + 512;        // row -> token offset inside a Q tile
  static constexpr int OFF_BAR = OFF_RTOK + 512;
  // kv_full, qd_full[2], qd_empty[2], lse_full, d_full, s_full, dp_full, p_ready[2],
  // ds_ready, dkv_final, drain
  static constexpr int B_KV = 0, B_QF = 1, B_QE = 3, B_LSE = 5, B_D = 6, B_S = 7, B_DP = 8, B_P = 9, B_DS = 11,
                       B_FIN = 12, B_DRAIN = 13, N_BARS = 14;
  static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
  // At least 120 KB so that one CTA, which holds all 512 TMEM columns, is
  // resident per SM; plus slack to align the base to 1024 bytes.
  static constexpr int SMEM_BYTES = (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) + 1024;
  static constexpr uint32_t TM_ST = 0, TM_DPT = 128, TM_DV = 256, TM_DK = 256 + DH;
  static constexpr int THREADS = 384;
  static constexpr int WARP_PRODUCER = 0, WARP_MMA = 1, WARP_SOFTMAX0 = 4;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(TM_DK + DH <= 512, "TMEM budget");
};

template <int DH, bool LO>
__global__ void __launch_bounds__(384, 1)
    sqa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const BwdParams p) {
  using Tr = BwdBf16Traits<DH>;
  using namespace dev;
  constexpr int BM = Tr::BM, NK = Tr::NK, ROWB = Tr::ROWB, PANEL = Tr::PANEL, QS = Tr::QS;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Under a causal mask the first key tiles see the most Q tiles: they go first.
  const int kt = static_cast<int>(blockIdx.x / p.n_bh);
  const int bh = blockIdx.x % p.n_bh;
  const int b = bh / p.Hkv, kvh = bh % p.Hkv;
  const int k0 = kt * NK;
  const int qt_first = p.causal ? k0 / p.T : 0;
  const int nq = p.n_qt - qt_first;

  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  const uint32_t kv_full = bar0 + 8u * Tr::B_KV;
  auto qd_full = [&](int s) { return bar0 + 8u * (Tr::B_QF + s); };
  auto qd_empty = [&](int s) { return bar0 + 8u * (Tr::B_QE + s); };
  const uint32_t lse_full = bar0 + 8u * Tr::B_LSE, d_full = bar0 + 8u * Tr::B_D;
  const uint32_t s_full = bar0 + 8u * Tr::B_S, dp_full = bar0 + 8u * Tr::B_DP;
  auto p_ready = [&](int hh) { return bar0 + 8u * (Tr::B_P + hh); };
  const uint32_t ds_ready = bar0 + 8u * Tr::B_DS;
  const uint32_t dkv_final = bar0 + 8u * Tr::B_FIN, drain = bar0 + 8u * Tr::B_DRAIN;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* rtok = reinterpret_cast<int*>(smem + Tr::OFF_RTOK);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(qd_full(s), 1);
      mbar_init(qd_empty(s), 1);
    }
    mbar_init(lse_full, 1);
    mbar_init(d_full, 1);
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready(0), 256);
    mbar_init(p_ready(1), 256);
    mbar_init(ds_ready, 256);
    mbar_init(dkv_final, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 128) rtok[threadIdx.x] = threadIdx.x < p.rows ? threadIdx.x / p.g : (1 << 30);
  if (p.rows < BM) {  // stacked rows the TMA box does not cover stay zero
    const int pad_bytes = (BM - p.rows) * ROWB;
    for (int s = 0; s < QS; ++s)
      for (int which = 0; which < 2; ++which)
        for (int pn = 0; pn < Tr::NPANEL; ++pn) {
          uint8_t* base = smem + (which ? Tr::OFF_DO : Tr::OFF_Q) + s * Tr::TILE + pn * BM * ROWB + p.rows * ROWB;
          for (int i = threadIdx.x * 16; i < pad_bytes; i += Tr::THREADS * 16)
            *reinterpret_cast<uint4*>(base + i) = make_uint4(0, 0, 0, 0);
        }
    fence_async_smem();
  }
  if (warp == Tr::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == Tr::WARP_PRODUCER) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmDO);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      const size_t slot0 = (static_cast<size_t>(bh) * p.n_qt + qt_first) * kBwdTile;
      mbar_expect_tx(kv_full, 2u * Tr::TILE);
      for (int pn = 0; pn < Tr::NPANEL; ++pn) {
        tma_load_4d(sbase + Tr::OFF_K + pn * NK * ROWB, &tmK, kv_full, pn * PANEL, kvh, k0, b);
        tma_load_4d(sbase + Tr::OFF_V + pn * NK * ROWB, &tmV, kv_full, pn * PANEL, kvh, k0, b);
      }
      mbar_expect_tx(lse_full, 512);
      bulk_load(sbase + Tr::OFF_LSE, p.lse2 + slot0, 512, lse_full);
      mbar_expect_tx(d_full, 512);
      bulk_load(sbase + Tr::OFF_D, p.D + slot0, 512, d_full);
      const uint32_t qd_bytes = 2u * p.rows * ROWB * Tr::NPANEL;
      auto load_qd = [&](int i) {
        const int s = i % QS, qt = qt_first + i;
        mbar_expect_tx(qd_full(s), qd_bytes);
        for (int pn = 0; pn < Tr::NPANEL; ++pn) {
          tma_load_4d(sbase + Tr::OFF_Q + s * Tr::TILE + pn * BM * ROWB, &tmQ, qd_full(s), pn * PANEL, kvh * p.g,
                      qt * p.T, b);
          tma_load_4d(sbase + Tr::OFF_DO + s * Tr::TILE + pn * BM * ROWB, &tmDO, qd_full(s), pn * PANEL,
                      kvh * p.g, qt * p.T, b);
        }
      };
      int qd_issued = 0, lse_issued = 1, d_issued = 1;
      for (; qd_issued < QS && qd_issued < nq; ++qd_issued) load_qd(qd_issued);
      for (int i = 0; i + 1 < nq; ++i) {
        // Tile i's softmax statistics are read: fetch tile i + 1's into the same buffers.
        const size_t slot = slot0 + static_cast<size_t>(i + 1) * kBwdTile;
        if (!mbar_wait(p_ready(1), i & 1, abort_flag, kSiteProducer)) break;
        mbar_expect_tx(lse_full, 512);
        bulk_load(sbase + Tr::OFF_LSE, p.lse2 + slot, 512, lse_full);
        lse_issued = i + 2;
        if (!mbar_wait(ds_ready, i & 1, abort_flag, kSiteProducer)) break;
        mbar_expect_tx(d_full, 512);
        bulk_load(sbase + Tr::OFF_D, p.D + slot, 512, d_full);
        d_issued = i + 2;
        // Stage i % QS is free once the MMAs of tile i are done with it.
        if (i + QS < nq) {
          if (!mbar_wait(qd_empty(i % QS), (i / QS) & 1, abort_flag, kSiteProducer)) break;
          load_qd(i + QS);
          qd_issued = i + QS + 1;
        }
      }
      if (*abort_flag) {  // let in-flight copies land before the CTA exits
        mbar_wait_drain(kv_full, 0);
        mbar_wait_drain(lse_full, (lse_issued - 1) & 1);
        mbar_wait_drain(d_full, (d_issued - 1) & 1);
        for (int i = max(0, qd_issued - QS); i < qd_issued; ++i) mbar_wait_drain(qd_full(i % QS), (i / QS) & 1);
      }
    }
  } else if (warp == Tr::WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
    constexpr uint32_t idesc_kv = idesc_bf16_f32(128, DH, false, true);   // dV, dK (A in TMEM, B MN-major)
    const uint32_t k_addr = sbase + Tr::OFF_K, v_addr = sbase + Tr::OFF_V;
    // S^T = K Q^T (or dP^T = V dO^T): M = 128 keys, N = 128 stacked query rows, K = dh.
    auto issue_s = [&](uint32_t d_col, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
      for (int ks = 0; ks < DH / 16; ++ks) {
        const uint32_t pn = (ks * 16) / PANEL, off = ((ks * 16) % PANEL) * 2;
        mma_ss_w(tmem + d_col, smem_desc(a_addr + pn * NK * ROWB + off, 16, 8 * ROWB, Tr::LAYOUT),
                 smem_desc(b_addr + pn * BM * ROWB + off, 16, 8 * ROWB, Tr::LAYOUT), idesc_s, ks > 0);
      }
    };
    bool ok = mbar_wait_warp(kv_full, 0, abort_flag, kSiteMma);
    if (ok) ok = mbar_wait_warp(qd_full(0), 0, abort_flag, kSiteMma);
    if (ok) {
      tc_fence_after();
      issue_s(Tr::TM_ST, k_addr, sbase + Tr::OFF_Q);
      mma_commit_w(s_full);
      issue_s(Tr::TM_DPT, v_addr, sbase + Tr::OFF_DO);
      mma_commit_w(dp_full);
    }
    for (int i = 0; ok && i < nq; ++i) {
      const int s = i % QS, s1 = (i + 1) % QS;
      const uint32_t q_addr = sbase + Tr::OFF_Q + s * Tr::TILE, do_addr = sbase + Tr::OFF_DO + s * Tr::TILE;
      // dV += P^T dO: M = 128 keys, N = dh, K = the 64 query rows of one half in
      // steps of 16.  Warpgroup w packed the P^T of rows 64 hh + 32 w + [0, 32)
      // into columns 64 hh + 32 w + [0, 16), with LO the remainders into
      // 64 hh + 32 w + [16, 32): a second MMA on the same dO rows adds them.
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (!(ok = mbar_wait_warp(p_ready(hh), i & 1, abort_flag, kSiteMma))) break;
        tc_fence_after();
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const uint32_t acol = 64u * hh + 32u * (k4 >> 1) + 8u * (k4 & 1);
          const uint32_t row0 = 64u * hh + 16u * k4;
          const uint64_t bdesc = smem_desc(do_addr + row0 * ROWB, BM * ROWB, 8 * ROWB, Tr::LAYOUT);
          mma_ts_w(tmem + Tr::TM_DV, tmem + Tr::TM_ST + acol, bdesc, idesc_kv, (i > 0 || hh > 0 || k4 > 0) ? 1u : 0u);
          if constexpr (LO) mma_ts_w(tmem + Tr::TM_DV, tmem + Tr::TM_ST + acol + 16u, bdesc, idesc_kv, 1u);
        }
      }
      if (!ok) break;
      // S^T of the next tile, over the P^T columns the dV MMAs just issued read first.
      if (i + 1 < nq) {
        if (!(ok = mbar_wait_warp(qd_full(s1), ((i + 1) / QS) & 1, abort_flag, kSiteMma))) break;
        tc_fence_after();
        issue_s(Tr::TM_ST, k_addr, sbase + Tr::OFF_Q + s1 * Tr::TILE);
        mma_commit_w(s_full);
      }
      // dK += dS^T Q (dS^T packed like P^T, in dP^T's columns).
      if (!(ok = mbar_wait_warp(ds_ready, i & 1, abort_flag, kSiteMma))) break;
      tc_fence_after();
#pragma unroll
      for (int k8 = 0; k8 < 8; ++k8) {
        const uint32_t acol = 64u * (k8 >> 2) + 32u * ((k8 >> 1) & 1) + 8u * (k8 & 1);
        const uint64_t bdesc = smem_desc(q_addr + 16u * k8 * ROWB, BM * ROWB, 8 * ROWB, Tr::LAYOUT);
        mma_ts_w(tmem + Tr::TM_DK, tmem + Tr::TM_DPT + acol, bdesc, idesc_kv, (i > 0 || k8 > 0) ? 1u : 0u);
        if constexpr (LO) mma_ts_w(tmem + Tr::TM_DK, tmem + Tr::TM_DPT + acol + 16u, bdesc, idesc_kv, 1u);
      }
      mma_commit_w(qd_empty(s));  // the last MMAs reading Q / dO of this stage
      // dP^T of the next tile, over the dS^T columns the dK MMAs just issued read first.
      if (i + 1 < nq) {
        issue_s(Tr::TM_DPT, v_addr, sbase + Tr::OFF_DO + s1 * Tr::TILE);
        mma_commit_w(dp_full);
      }
    }
    if (ok) {
      mma_commit_w(dkv_final);
    } else {
      mma_commit_w(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= Tr::WARP_SOFTMAX0) {
    // ------------------------------------------------------------ P^T, dS^T, dK/dV epilogue
    const int w = (warp - Tr::WARP_SOFTMAX0) >> 2;  // warpgroup
    const int kk = (warp & 3) * 32 + lane;          // TMEM lane: key
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = k0 + kk;
    const bool key_ok = key < p.N;
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    const float* nl2 = reinterpret_cast<const float*>(smem + Tr::OFF_LSE);
    const float* nd = reinterpret_cast<const float*>(smem + Tr::OFF_D);
    bool ok = true;
    for (int i = 0; i < nq; ++i) {
      const int qt = qt_first + i;
      const bool masked = p.causal && (k0 + NK - 1 > qt * p.T);
      // P is zeroed where lim > rtok[row]: keys past N always, keys after the
      // row's token on the causal diagonal.
      const int lim = !key_ok ? 0x7fffffff : (masked ? key - qt * p.T : -0x7fffffff);
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, i & 1, abort_flag, kSiteSoftmax) &&
                                       mbar_wait(lse_full, i & 1, abort_flag, kSiteSoftmax));
      if (!ok) break;
      tc_fence_after();
      // P^T of both halves (their S^T columns loaded with one wait); kept in
      // registers (fp32) for dS.
      float pr[2][32];
      uint32_t sr2[64];  // [0, 32): half 0, [32, 64): half 1
      tmem_ld32x2(lane_addr + Tr::TM_ST + 32 * w, lane_addr + Tr::TM_ST + 64 + 32 * w, sr2);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int col0 = 64 * hh + 32 * w;
        const uint32_t* sr = sr2 + 32 * hh;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(nl2 + col0 + e);
          const int4 r4 = *reinterpret_cast<const int4*>(rtok + col0 + e);
          const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), sl2,
                                        make_float2(l4.x, l4.y));
          const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3])), sl2,
                                        make_float2(l4.z, l4.w));
          pr[hh][e] = lim > r4.x ? 0.f : ex2(x01.x);
          pr[hh][e + 1] = lim > r4.y ? 0.f : ex2(x01.y);
          pr[hh][e + 2] = lim > r4.z ? 0.f : ex2(x23.x);
          pr[hh][e + 3] = lim > r4.w ? 0.f : ex2(x23.y);
        }
        uint32_t pk[16];
        if constexpr (LO) {
          uint32_t pl[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) split_bf16x2(pr[hh][2 * e], pr[hh][2 * e + 1], pk[e], pl[e]);
          tmem_st16(lane_addr + Tr::TM_ST + col0 + 16, pl);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pr[hh][2 * e], pr[hh][2 * e + 1]);
        }
        tmem_st16(lane_addr + Tr::TM_ST + col0, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_ready(hh));
      }
      // dS^T = P^T (dP^T - D) into dP^T's columns (bf16 pairs).
      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, i & 1, abort_flag, kSiteSoftmax) &&
                                       mbar_wait(d_full, i & 1, abort_flag, kSiteSoftmax));
      if (!ok) break;
      tc_fence_after();
      uint32_t dr2[64];  // dP^T of both halves, one wait
      tmem_ld32x2(lane_addr + Tr::TM_DPT + 32 * w, lane_addr + Tr::TM_DPT + 64 + 32 * w, dr2);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int col0 = 64 * hh + 32 * w;
        const uint32_t* dr = dr2 + 32 * hh;
        uint32_t dk[16], dl[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(nd + col0 + e);
          const float2 t01 = __fadd2_rn(make_float2(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])),
                                        make_float2(d4.x, d4.y));
          const float2 t23 = __fadd2_rn(make_float2(__uint_as_float(dr[e + 2]), __uint_as_float(dr[e + 3])),
                                        make_float2(d4.z, d4.w));
          const float2 s01 = __fmul2_rn(make_float2(pr[hh][e], pr[hh][e + 1]), t01);
          const float2 s23 = __fmul2_rn(make_float2(pr[hh][e + 2], pr[hh][e + 3]), t23);
          if constexpr (LO) {
            split_bf16x2(s01.x, s01.y, dk[e >> 1], dl[e >> 1]);
            split_bf16x2(s23.x, s23.y, dk[(e >> 1) + 1], dl[(e >> 1) + 1]);
          } else {
            dk[e >> 1] = pack_bf16x2(s01.x, s01.y);
            dk[(e >> 1) + 1] = pack_bf16x2(s23.x, s23.y);
          }
        }
        tmem_st16(lane_addr + Tr::TM_DPT + col0, dk);
        if constexpr (LO) tmem_st16(lane_addr + Tr::TM_DPT + col0 + 16, dl);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_ready);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dkv_final, 0, abort_flag, kSiteEpilogue));
    if (ok) {
      tc_fence_after();
      const size_t off = ((static_cast<size_t>(b) * p.N + (key_ok ? key : 0)) * p.Hkv + kvh) * DH + w * (DH / 2);
      float v[DH / 2];
      tmem_ld_half<DH>(lane_addr + Tr::TM_DV + w * (DH / 2), v);
      if (key_ok) {
#pragma unroll
        for (int c = 0; c < DH / 2; c += 8) {
          uint4 o;
          o.x = pack_bf16x2(v[c], v[c + 1]);
          o.y = pack_bf16x2(v[c + 2], v[c + 3]);
          o.z = pack_bf16x2(v[c + 4], v[c + 5]);
          o.w = pack_bf16x2(v[c + 6], v[c + 7]);
          *reinterpret_cast<uint4*>(p.dv + off + c) = o;
        }
      }
      tmem_ld_half<DH>(lane_addr + Tr::TM_DK + w * (DH / 2), v);
      if (key_ok) {
        const float sc = p.scale;
#pragma unroll
        for (int c = 0; c < DH / 2; c += 8) {
          uint4 o;
          o.x = pack_bf16x2(v[c] * sc, v[c + 1] * sc);
          o.y = pack_bf16x2(v[c + 2] * sc, v[c + 3] * sc);
          o.z = pack_bf16x2(v[c + 4] * sc, v[c + 5] * sc);
          o.w = pack_bf16x2(v[c + 6] * sc, v[c + 7] * sc);
          *reinterpret_cast<uint4*>(p.dk + off + c) = o;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Tr::WARP_MMA) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// sqa_bwd_q_kernel<DH>: dQ, one CTA per stacked Q tile (128 rows: the g query
// heads of one KV head for T tokens) of one batch entry, heaviest (latest
// tokens under a causal mask) first.  The Q and dO tiles go into TMEM once,
// as the A operands of every S and dP product; K and V stream through a ring
// of 64-key stages.  Per key tile j (two TMEM buffers, j % 2):
//     S_j  = Q K_j^T, dP_j = dO V_j^T        (TMEM, query rows on lanes)
//     dS_j = 2^(S_j scale log2e - lse2) (dP_j - D), rewritten in place (bf16)
//     dQ  += dS_j K_j                         (A = dS_j from TMEM)
// Three issuers: one runs S_{j+1} ahead and one dP_{j+1} while the warps turn
// S_j and dP_j into dS_j, the third issues dQ of j as soon as dS_j is ready.
// (With one issuer for all three products its instruction stream, which shares
// its sub-partition with two busy softmax warps, took twice as long per key
// tile as the warps and set the pace: an N = 64 MMA takes longer to issue than
// to run.)  S_{j+2} and dP_{j+2} reuse buffer j % 2 once the dQ of j has read
// dS_j (dq_done).  dQ is scaled and written once, in bf16.
//
// TMEM (dh 128): Q [0, 64), dO [64, 128), S buffers 128 + 64 b, dP buffers
// 256 + 64 b, dQ [384, 512); at dh 64 the same with Q, dO of 32 columns.
// Roles (384 threads): warp 0 producer, warp 1 TMEM allocator and S issuer,
// warp 2 dQ issuer, warp 3 dP issuer, warps 4-11 two warpgroups (warpgroup w: keys 32 w .. 32 w + 31 of each
// stage, query row = TMEM lane), which also load Q and dO into TMEM and write
// dQ.

struct BwdQParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* dout;
  const float* lse2;  // stacked, negated (see BwdParams)
  const float* D;
  __nv_bfloat16* dq;
  int N, Hq, Hkv, g, T, rows, n_qt, n_bh, causal;
  float scale_log2, scale;
};

template <int DH>
struct BwdQTraits {
  static_assert(DH == 64 || DH == 128, "query-major backward handles dh 64 and 128");
  static constexpr int BM = 128, NK = 64;
  static constexpr int PANEL = 64, NPANEL = DH / PANEL, ROWB = 128;
  static constexpr uint32_t LAYOUT = 2u;
  static constexpr int KV_BYTES = NK * DH * 2;
  static constexpr int STAGES = DH == 128 ? 6 : 8;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
  // kv_full[S], kv_empty[S], qd_ready, sd_full[2], ds_ready[2], dq_final, drain[3], dq_done[2]
  static constexpr int N_BARS = 2 * STAGES + 11;
  static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
  static constexpr int SMEM_BYTES = (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) + 1024;
  static constexpr uint32_t TM_Q = 0, TM_DO = DH / 2;
  __host__ __device__ static constexpr uint32_t tm_s(int b) { return 128u + 64u * b; }
  __host__ __device__ static constexpr uint32_t tm_dp(int b) { return 256u + 64u * b; }
  static constexpr uint32_t TM_DQ = 384, TM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr int WARP_PRODUCER = 0, WARP_MMA = 1, WARP_MMA_Q = 2, WARP_MMA_DP = 3, WARP_SOFTMAX0 = 4;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(TM_DQ + DH <= TM_COLS, "TMEM budget");
};

template <int DH>
__global__ void __launch_bounds__(384, 1)
    sqa_bwd_q_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const BwdQParams p) {
  using Tr = BwdQTraits<DH>;
  using namespace dev;
  constexpr int NK = Tr::NK, ROWB = Tr::ROWB, PANEL = Tr::PANEL, ST = Tr::STAGES;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Latest Q tiles first: under a causal mask they see the most keys.
  const int qt = p.n_qt - 1 - static_cast<int>(blockIdx.x / p.n_bh);
  const int bh = blockIdx.x % p.n_bh;
  const int b = bh / p.Hkv, kvh = bh % p.Hkv;
  const int kend = p.causal ? min(p.N, (qt + 1) * p.T) : p.N;  // keys [0, kend) are visible to some row
  const int nkv = (kend + NK - 1) / NK;

  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  auto kv_full = [&](int s) { return bar0 + 8u * s; };
  auto kv_empty = [&](int s) { return bar0 + 8u * (ST + s); };
  const uint32_t qd_ready = bar0 + 8u * (2 * ST);
  auto sd_full = [&](int x) { return bar0 + 8u * (2 * ST + 1 + x); };
  auto ds_ready = [&](int x) { return bar0 + 8u * (2 * ST + 3 + x); };
  const uint32_t dq_final = bar0 + 8u * (2 * ST + 5);
  auto drain = [&](int i) { return bar0 + 8u * (2 * ST + 6 + i); };  // one per issuer
  auto dq_done = [&](int x) { return bar0 + 8u * (2 * ST + 9 + x); };  // dQ of a tile in buffer x has read its dS
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(qd_ready, 256);
    for (int x = 0; x < 2; ++x) {
      mbar_init(sd_full(x), 2);  // the S and the dP issuer
      mbar_init(ds_ready(x), 256);
      mbar_init(dq_done(x), 1);
    }
    mbar_init(dq_final, 1);
    for (int i = 0; i < 3; ++i) mbar_init(drain(i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Tr::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), Tr::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == Tr::WARP_PRODUCER) {
    // ------------------------------------------------------------ producer: K / V ring
    if (lane == 0) {
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      int j = 0;
      for (; j < nkv; ++j) {
        const int s = j % ST;
        if (j >= ST && !mbar_wait(kv_empty(s), ((j / ST) - 1) & 1, abort_flag, kSiteProducer)) break;
        mbar_expect_tx(kv_full(s), 2u * Tr::KV_BYTES);
        for (int pn = 0; pn < Tr::NPANEL; ++pn) {
          tma_load_4d(sbase + Tr::OFF_K + s * Tr::KV_BYTES + pn * NK * ROWB, &tmK, kv_full(s), pn * PANEL, kvh,
                      j * NK, b);
          tma_load_4d(sbase + Tr::OFF_V + s * Tr::KV_BYTES + pn * NK * ROWB, &tmV, kv_full(s), pn * PANEL, kvh,
                      j * NK, b);
        }
      }
      if (*abort_flag) {
        for (int i = max(0, j - ST); i < j; ++i) mbar_wait_drain(kv_full(i % ST), (i / ST) & 1);
      }
    }
  } else if (warp == Tr::WARP_MMA || warp == Tr::WARP_MMA_DP) {
    // ------------------------------------------------------------ S issuer (warp 1), dP issuer (warp 3)
    // S_j = Q K_j^T or dP_j = dO V_j^T: M = 128 rows, N = 64 keys, K = dh in
    // steps of 16 (8 TMEM columns of Q / dO); A from TMEM, B K-major in smem.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, NK, false, false);
    const bool is_s = warp == Tr::WARP_MMA;
    const uint64_t db0 = smem_desc(sbase + (is_s ? Tr::OFF_K : Tr::OFF_V), 16, 8 * ROWB, Tr::LAYOUT);
    const uint32_t ta = tmem + (is_s ? Tr::TM_Q : Tr::TM_DO);
    bool ok = mbar_wait_warp(qd_ready, 0, abort_flag, kSiteMma);
    for (int j = 0; ok && j < nkv; ++j) {
      const int x = j & 1;
      if (!(ok = mbar_wait_warp(kv_full(j % ST), (j / ST) & 1, abort_flag, kSiteMma))) break;
      // buffer j % 2 held dS_{j-2} (and dP_{j-2}): the dQ MMA has read it
      if (j >= 2 && !(ok = mbar_wait_warp(dq_done(x), ((j - 2) >> 1) & 1, abort_flag, kSiteMma))) break;
      tc_fence_after();
      const uint32_t td = tmem + (is_s ? Tr::tm_s(x) : Tr::tm_dp(x));
      const uint64_t so = static_cast<uint64_t>(((j % ST) * Tr::KV_BYTES) >> 4);
#pragma unroll
      for (int ks = 0; ks < DH / 16; ++ks) {
        const uint64_t ko = so + ((((ks * 16) / PANEL) * NK * ROWB + ((ks * 16) % PANEL) * 2) >> 4);
        mma_ts_w(td, ta + 8u * ks, db0 + ko, idesc_s, ks > 0);
      }
      mma_commit_w(sd_full(x));
    }
    if (!ok) {
      const int d = is_s ? 0 : 2;
      mma_commit_w(drain(d));
      mbar_wait_drain(drain(d), 0);
    }
  } else if (warp == Tr::WARP_MMA_Q) {
    // ------------------------------------------------------------ dQ issuer
    constexpr uint32_t idesc_q = idesc_bf16_f32(128, DH, false, true);  // dQ: A = dS in TMEM, B = K MN-major
    const uint64_t dkmn0 = smem_desc(sbase + Tr::OFF_K, NK * ROWB, 8 * ROWB, Tr::LAYOUT);
    // dQ += dS_j K_j: M = 128 rows, N = dh, K = 64 keys in steps of 16.  Warpgroup w
    // packed the dS of keys 32 w .. 32 w + 31 into columns 32 w .. 32 w + 15.
    bool ok = true;
    for (int j = 0; ok && j < nkv; ++j) {
      const int s = j % ST, x = j & 1;
      if (!(ok = mbar_wait_warp(ds_ready(x), (j >> 1) & 1, abort_flag, kSiteMma))) break;
      tc_fence_after();
      const uint64_t so = static_cast<uint64_t>((s * Tr::KV_BYTES) >> 4);
#pragma unroll
      for (int ks = 0; ks < NK / 16; ++ks)
        mma_ts_w(tmem + Tr::TM_DQ, tmem + Tr::tm_s(x) + 32u * (ks >> 1) + 8u * (ks & 1),
                 dkmn0 + so + ((ks * 16 * ROWB) >> 4), idesc_q, (j > 0 || ks > 0) ? 1u : 0u);
      mma_commit_w(dq_done(x));
      // K_j and V_j are read: S_j and dP_j completed before the warps made dS_j
      mma_commit_w(kv_empty(s));
    }
    if (ok) {
      mma_commit_w(dq_final);
    } else {
      mma_commit_w(drain(1));
      mbar_wait_drain(drain(1), 0);
    }
  } else if (warp >= Tr::WARP_SOFTMAX0) {
    // ------------------------------------------------------------ Q / dO into TMEM, dS, dQ epilogue
    const int w = (warp - Tr::WARP_SOFTMAX0) >> 2;
    const int r = (warp & 3) * 32 + lane;  // stacked query row = TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int tok = qt * p.T + r / p.g;
    const int head = kvh * p.g + r % p.g;
    const bool row_ok = r < p.rows && tok < p.N;
    const size_t row = (static_cast<size_t>(b) * p.N + (row_ok ? tok : 0)) * p.Hq + head;
    // Warpgroup w writes the A operand of Q (w = 0) or dO (w = 1): this row's dh
    // values as bf16 pairs (zeros for padding rows).
    {
      const __nv_bfloat16* src = (w == 0 ? p.q : p.dout) + row * DH;
      const uint32_t dst = lane_addr + (w == 0 ? Tr::TM_Q : Tr::TM_DO);
#pragma unroll
      for (int c = 0; c < DH; c += 32) {
        uint32_t v[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint4 x4 = row_ok ? *reinterpret_cast<const uint4*>(src + c + 8 * u) : make_uint4(0, 0, 0, 0);
          v[4 * u] = x4.x;
          v[4 * u + 1] = x4.y;
          v[4 * u + 2] = x4.z;
          v[4 * u + 3] = x4.w;
        }
        tmem_st16(dst + c / 2, v);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(qd_ready);
    }
    const size_t slot = (static_cast<size_t>(bh) * p.n_qt + qt) * kBwdTile + r;
    const float nl2 = p.lse2[slot], nd = p.D[slot];  // negated statistics of this row
    const float sl2 = p.scale_log2;
    // visible keys of this row: [0, last]
    const int last = row_ok ? (p.causal ? tok : p.N - 1) : -1;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int x = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(sd_full(x), (j >> 1) & 1, abort_flag, kSiteSoftmax));
      if (!ok) break;
      tc_fence_after();
      const int k0 = j * NK + 32 * w;  // this warpgroup's first key
      uint32_t sd[64];                 // [0, 32): S, [32, 64): dP (one wait for both loads)
      tmem_ld32x2(lane_addr + Tr::tm_s(x) + 32 * w, lane_addr + Tr::tm_dp(x) + 32 * w, sd);
      const bool edge = __any_sync(0xffffffffu, k0 + 31 > last);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float p0 = ex2(fmaf(__uint_as_float(sd[e]), sl2, nl2));
        float p1 = ex2(fmaf(__uint_as_float(sd[e + 1]), sl2, nl2));
        if (edge) {
          if (k0 + e > last) p0 = 0.f;
          if (k0 + e + 1 > last) p1 = 0.f;
        }
        const float2 ds = __fmul2_rn(make_float2(p0, p1),
                                     __fadd2_rn(make_float2(__uint_as_float(sd[32 + e]), __uint_as_float(sd[33 + e])),
                                                make_float2(nd, nd)));
        pk[e >> 1] = pack_bf16x2(ds.x, ds.y);
      }
      // dS of keys k0 .. k0 + 31 into columns 32 w .. 32 w + 15 of the S buffer
      // (scores this warpgroup has already read).
      tmem_st16(lane_addr + Tr::tm_s(x) + 32 * w, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_ready(x));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dq_final, 0, abort_flag, kSiteEpilogue));
    if (ok) {
      tc_fence_after();
      float v[DH / 2];
      tmem_ld_half<DH>(lane_addr + Tr::TM_DQ + w * (DH / 2), v);
      if (row_ok) {
        __nv_bfloat16* dst = p.dq + row * DH + w * (DH / 2);
        const float sc = p.scale;
#pragma unroll
        for (int c = 0; c < DH / 2; c += 8) {
          uint4 o;
          o.x = pack_bf16x2(v[c] * sc, v[c + 1] * sc);
          o.y = pack_bf16x2(v[c + 2] * sc, v[c + 3] * sc);
          o.z = pack_bf16x2(v[c + 4] * sc, v[c + 5] * sc);
          o.w = pack_bf16x2(v[c + 6] * sc, v[c + 7] * sc);
          *reinterpret_cast<uint4*>(dst + c) = o;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Tr::WARP_MMA) tmem_dealloc(tmem, Tr::TM_COLS);
}

}  // namespace sqa

// sqa_bwd_tf32.cuh -- Sparse Query Attention backward, main kernel for head
// dims 16 and 32 (the SQAT-m shapes).
//
// Same decomposition as sqa_bwd_kernel (one CTA per 128-key tile, batch and KV
// head; stacked Q tiles of the g query heads of the group, so dK and dV are
// reduced over the group inside the tensor-core accumulation), organised for
// small head dims, where the exponentials and the MMA issue rate, not the tensor
// core, set the pace:
//
//  * dV += P^T dO and dK += dS^T Q run as tf32 MMAs with K-major operands (tf32
//    operands stored MN-major produced zeros on this hardware).  P^T and dS^T
//    stay in fp32 in TMEM, in place; a converter warp writes transposed fp32
//    copies of the Q and dO tiles ([dh][128 rows], rows contiguous).  dS is
//    rounded to tf32 (to nearest), P is passed as is.  tf32 keeps bf16's
//    exponent range and three more mantissa bits, which matters when a large
//    query group sums many terms into one dK or dV row.  dQ = dS K sums only
//    over keys and runs in bf16 (dS as bf16 in shared memory, K as loaded).
//    S^T = K Q^T and dP^T = V dO^T run in bf16 (exact products).
//
//  * The 128-row Q tile is split into two 64-column halves with their own TMEM
//    buffers; warpgroup w always takes half w, so the two warpgroups work on
//    different halves at any moment instead of in lockstep.
//
//  * Two MMA-issuing threads: A issues S^T / dP^T and dQ, B issues dV / dK.  B
//    signals when a TMEM buffer has been read, before A overwrites it.
//
// Roles (384 threads):
//   warps 0-3   P^T / dS^T for half 0 of every Q tile (warpgroup 0), warps 4-7 for
//               half 1 (warpgroup 1); also the dQ epilogue (fp32 atomics) and the
//               dK / dV epilogue
//   warp 8      TMA producer (K, V once; Q, dO, lse2, D per Q tile)
//   warp 9      TMEM allocator and MMA issuer A; warp 10 MMA issuer B
//   warp 11     bf16 -> fp32 transposing converter for Q and dO
// TMEM: half buffer b: S^T at 128 b, dP^T at 128 b + 64 (64 columns each);
// dV at 256, dK at 320, dQ of Q tile i at 384 + 64 (i % 2).
#pragma once

#include "sqa_bwd.cuh"
#include "sqa_tmem_wide.cuh"

namespace sqa {

namespace dev {
// Instruction descriptor for kind::tf32 (A and B tf32, fp32 accumulation).
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void mma_ss_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// fp32 bits rounded to the nearest tf32 value (10 mantissa bits; halfway cases
// away from zero), with integer operations only.
__device__ __forceinline__ uint32_t round_tf32(float x) {
  return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u;
}
// Byte offset of 16-byte chunk `chunk` of row `r` in a tile with `rowb`-byte rows
// stored with the matching TMA / UMMA swizzle (32, 64 or 128 bytes).
__device__ __forceinline__ uint32_t swz_off(int r, int chunk, int rowb) {
  return static_cast<uint32_t>(r * rowb + ((chunk ^ ((r * rowb >> 7) & (rowb / 16 - 1))) << 4));
}
}  // namespace dev

template <int DH>
struct BwdTf32Traits {
  static_assert(DH == 16 || DH == 32, "tf32 backward handles dh 16 and 32");
  static constexpr int NK = kBwdTile, BM = kBwdTile;
  static constexpr int ROWB = DH * 2;  // bf16 row bytes (one swizzle panel)
  static constexpr uint32_t LAYOUT = ROWB == 32 ? 6u : 4u;  // bf16 tiles: SW32 / SW64
  // fp32 tiles are transposed, [dh][128] K-major with a 128-byte swizzle: four
  // panels of 32 values, each panel dh rows of 128 bytes.
  static constexpr int PANEL32 = DH * 128;
  static constexpr int TILE = 128 * DH * 2;
  static constexpr int TILE32 = 128 * DH * 4;
  static constexpr int QS = 2;
  static constexpr int DS_BYTES = 128 * 128 * 2;  // bf16 dS, MN-major (query rows contiguous)
  static constexpr int OFF_DS = 0;
  static constexpr int OFF_K = OFF_DS + DS_BYTES;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;
  static constexpr int OFF_DO = OFF_Q + QS * TILE;
  static constexpr int OFF_Q32 = OFF_DO + QS * TILE;
  static constexpr int OFF_DO32 = OFF_Q32 + QS * TILE32;
  static constexpr int OFF_STAT = OFF_DO32 + QS * TILE32;  // per stage: lse2[128], D[128]
  static constexpr int OFF_RTOK = OFF_STAT + QS * 1024;
  static constexpr int OFF_BAR = OFF_RTOK + 512;
  // kv_full, qd_full[2], qd_empty[2], cvt_full[2], s_full[2], ds_ready[2], kvmma_done[2], dq_full,
  // dq_empty[2], dkv_final, drain[2]
  static constexpr int N_BARS = 20;
  static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
  // Enough shared memory that only one CTA fits per SM (each holds all 512 TMEM columns).
  static constexpr int SMEM_BYTES = (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) + 1024;
  static constexpr uint32_t TM_DV = 256, TM_DK = 320;
  __host__ __device__ static constexpr uint32_t tm_st(int b) { return 128u * b; }
  __host__ __device__ static constexpr uint32_t tm_dpt(int b) { return 128u * b + 64u; }
  __host__ __device__ static constexpr uint32_t tm_dq(int i) { return 384u + 64u * (i & 1); }
  static constexpr int THREADS = 384;
  static constexpr int WARP_PRODUCER = 8, WARP_MMA_A = 9, WARP_MMA_B = 10, WARP_CVT = 11;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Convert a bf16 tile [128 rows][dh] (rows of 2*dh bytes, swizzled as loaded by
// TMA) into the transposed fp32 tile [dh][128] in K-major 128-byte-swizzled
// panels of 32 rows, with one warp.  The warp writes one 128-byte row segment
// per store instruction.
template <int DH>
__device__ __forceinline__ void convert_tile_t(const uint8_t* src, uint8_t* dst, int lane) {
  constexpr int ROWB = DH * 2;
#pragma unroll 1
  for (int r = lane; r < 128; r += 32) {
    float v[DH];
#pragma unroll
    for (int c = 0; c < ROWB / 16; ++c) {
      const uint4 u = *reinterpret_cast<const uint4*>(src + dev::swz_off(r, c, ROWB));
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        v[8 * c + 2 * e] = f.x;
        v[8 * c + 2 * e + 1] = f.y;
      }
    }
    uint8_t* base = dst + (r >> 5) * (DH * 128) + (r & 3) * 4;
    const int chunk = (r & 31) >> 2;
#pragma unroll
    for (int n = 0; n < DH; ++n) *reinterpret_cast<float*>(base + n * 128 + ((chunk ^ (n & 7)) << 4)) = v[n];
  }
}

template <int DH>
__global__ void __launch_bounds__(384, 1)
    sqa_bwd_tf32_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                        const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const BwdParams p) {
  using Tr = BwdTf32Traits<DH>;
  using namespace dev;
  constexpr int BM = Tr::BM, NK = Tr::NK, ROWB = Tr::ROWB, QS = Tr::QS;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Under a causal mask the first key tiles see the most query tiles: they go first.
  const int kt = static_cast<int>(blockIdx.x / p.n_bh);
  const int bh = blockIdx.x % p.n_bh;
  const int b = bh / p.Hkv, kvh = bh % p.Hkv;
  const int k0 = kt * NK;
  const int qt_first = p.causal ? k0 / p.T : 0;
  const int nq = p.n_qt - qt_first;

  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  const uint32_t kv_full = bar0;
  auto qd_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto qd_empty = [&](int s) { return bar0 + 8u * (3 + s); };
  auto cvt_full = [&](int s) { return bar0 + 8u * (5 + s); };
  auto s_full = [&](int bb) { return bar0 + 8u * (7 + bb); };
  auto ds_ready = [&](int bb) { return bar0 + 8u * (9 + bb); };
  auto kvmma_done = [&](int bb) { return bar0 + 8u * (11 + bb); };
  const uint32_t dq_full = bar0 + 8u * 13;
  auto dq_empty = [&](int x) { return bar0 + 8u * (14 + x); };
  const uint32_t dkv_final = bar0 + 8u * 16;
  auto drain = [&](int x) { return bar0 + 8u * (17 + x); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* rtok = reinterpret_cast<int*>(smem + Tr::OFF_RTOK);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(qd_full(s), 1);
      mbar_init(qd_empty(s), 2);  // released by both MMA issuers
      mbar_init(cvt_full(s), 32);
    }
    for (int bb = 0; bb < 2; ++bb) {
      mbar_init(s_full(bb), 1);
      mbar_init(ds_ready(bb), 128);
      mbar_init(kvmma_done(bb), 1);
      mbar_init(dq_empty(bb), 256);
      mbar_init(drain(bb), 1);
    }
    mbar_init(dq_full, 1);
    mbar_init(dkv_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 128) rtok[threadIdx.x] = threadIdx.x < p.rows ? threadIdx.x / p.g : (1 << 30);
  if (p.rows < BM) {  // stacked rows the TMA box does not cover stay zero (the fp32 copies follow)
    for (int s = 0; s < QS; ++s)
      for (int which = 0; which < 2; ++which) {
        uint8_t* base = smem + (which ? Tr::OFF_DO : Tr::OFF_Q) + s * Tr::TILE + p.rows * ROWB;
        for (int i = threadIdx.x * 16; i < (BM - p.rows) * ROWB; i += Tr::THREADS * 16)
          *reinterpret_cast<uint4*>(base + i) = make_uint4(0, 0, 0, 0);
      }
    fence_async_smem();
  }
  if (warp == Tr::WARP_MMA_A) {
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
      mbar_expect_tx(kv_full, 2u * Tr::TILE);
      tma_load_4d(sbase + Tr::OFF_K, &tmK, kv_full, 0, kvh, k0, b);
      tma_load_4d(sbase + Tr::OFF_V, &tmV, kv_full, 0, kvh, k0, b);
      const uint32_t qd_bytes = 2u * p.rows * ROWB + 2u * 512u;
      int issued = 0;
      for (int i = 0; i < nq; ++i) {
        const int s = i % QS, qt = qt_first + i;
        if (i >= QS && !mbar_wait(qd_empty(s), ((i / QS) - 1) & 1, abort_flag, kSiteProducer)) break;
        mbar_expect_tx(qd_full(s), qd_bytes);
        tma_load_4d(sbase + Tr::OFF_Q + s * Tr::TILE, &tmQ, qd_full(s), 0, kvh * p.g, qt * p.T, b);
        tma_load_4d(sbase + Tr::OFF_DO + s * Tr::TILE, &tmDO, qd_full(s), 0, kvh * p.g, qt * p.T, b);
        const size_t slot = (static_cast<size_t>(bh) * p.n_qt + qt) * kBwdTile;
        bulk_load(sbase + Tr::OFF_STAT + s * 1024, p.lse2 + slot, 512, qd_full(s));
        bulk_load(sbase + Tr::OFF_STAT + s * 1024 + 512, p.D + slot, 512, qd_full(s));
        issued = i + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(kv_full, 0);
        for (int i = max(0, issued - QS); i < issued; ++i) mbar_wait_drain(qd_full(i % QS), (i / QS) & 1);
      }
    }
  } else if (warp == Tr::WARP_CVT) {
    // ------------------------------------------------------------ bf16 -> fp32 converter
    for (int i = 0; i < nq; ++i) {
      const int s = i % QS;
      // The producer refills stage s only after both MMA issuers released the
      // tile that used it last, so its fp32 copies are free too.
      if (!__all_sync(0xffffffffu, mbar_wait(qd_full(s), (i / QS) & 1, abort_flag, kSiteEpilogue))) break;
      convert_tile_t<DH>(smem + Tr::OFF_Q + s * Tr::TILE, smem + Tr::OFF_Q32 + s * Tr::TILE32, lane);
      convert_tile_t<DH>(smem + Tr::OFF_DO + s * Tr::TILE, smem + Tr::OFF_DO32 + s * Tr::TILE32, lane);
      fence_async_smem();
      mbar_arrive(cvt_full(s));
    }
  } else if (warp == Tr::WARP_MMA_A) {
    // ------------------------------------------------------------ MMA issuer A: S^T, dP^T, dQ
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);  // S^T, dP^T halves
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, DH, true, true);    // dQ = dS K (both MN-major)
      // Descriptors of stage 0 / K-step 0; others add their byte offset / 16.
      const uint64_t dk = smem_desc(sbase + Tr::OFF_K, 16, 8 * ROWB, Tr::LAYOUT);
      const uint64_t dv = smem_desc(sbase + Tr::OFF_V, 16, 8 * ROWB, Tr::LAYOUT);
      const uint64_t dqt = smem_desc(sbase + Tr::OFF_Q, 16, 8 * ROWB, Tr::LAYOUT);
      const uint64_t ddo = smem_desc(sbase + Tr::OFF_DO, 16, 8 * ROWB, Tr::LAYOUT);
      const uint64_t dds = smem_desc(sbase + Tr::OFF_DS, 16384, 1024, 2u);
      const uint64_t dkmn = smem_desc(sbase + Tr::OFF_K, NK * ROWB, 8 * ROWB, Tr::LAYOUT);
      // S^T and dP^T of half h (query rows 64 (h % 2) ..) into TMEM buffer h % 2.
      auto issue_s = [&](int h) {
        const int s = (h >> 1) % QS, hh = h & 1;
        const uint64_t off = static_cast<uint64_t>((s * Tr::TILE + hh * 64 * ROWB) >> 4);
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          mma_ss(tmem + Tr::tm_st(hh), dk + 2 * ks, dqt + off + 2 * ks, idesc_s, ks > 0);
          mma_ss(tmem + Tr::tm_dpt(hh), dv + 2 * ks, ddo + off + 2 * ks, idesc_s, ks > 0);
        }
        mma_commit(s_full(hh));
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag, kSiteMma) && mbar_wait(qd_full(0), 0, abort_flag, kSiteMma);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_s(1);
      }
      for (int i = 0; ok && i < nq; ++i) {
        const int s = i % QS;
        const bool next = i + 1 < nq;
        if (next) {
          // Half 0 of the next Q tile, once B has read buffer 0 (half 2i).
          ok = mbar_wait(qd_full((i + 1) % QS), ((i + 1) / QS) & 1, abort_flag, kSiteMma) &&
               mbar_wait(kvmma_done(0), i & 1, abort_flag, kSiteMma);
          if (!ok) break;
          tc_fence_after();
          issue_s(2 * i + 2);
        }
        // dQ of tile i needs both halves of dS.  Half 2i is covered: B read it
        // before signalling kvmma_done(0) above (or, for the last tile, below).
        if (!next && !mbar_wait(kvmma_done(0), i & 1, abort_flag, kSiteMma)) { ok = false; break; }
        if (!mbar_wait(ds_ready(1), i & 1, abort_flag, kSiteMma)) { ok = false; break; }
        if (i >= 2 && !mbar_wait(dq_empty(i & 1), ((i >> 1) - 1) & 1, abort_flag, kSiteMma)) { ok = false; break; }
        tc_fence_after();
        // dQ = dS K: M = 128 query rows, N = dh, K = 128 keys in steps of 16 (2 KB of dS, 16 K rows).
#pragma unroll
        for (int ks = 0; ks < NK / 16; ++ks)
          mma_ss(tmem + Tr::tm_dq(i), dds + 128 * ks, dkmn + ((ks * 16 * ROWB) >> 4), idesc_q, ks > 0);
        mma_commit(dq_full);
        mma_commit(qd_empty(s));
        if (next) {
          // Half 1 of the next Q tile, once B has read buffer 1 (half 2i + 1).
          if (!mbar_wait(kvmma_done(1), i & 1, abort_flag, kSiteMma)) { ok = false; break; }
          tc_fence_after();
          issue_s(2 * i + 3);
        }
      }
      if (!ok) {
        mma_commit(drain(0));
        mbar_wait_drain(drain(0), 0);
      }
    }
  } else if (warp == Tr::WARP_MMA_B) {
    // ------------------------------------------------------------ MMA issuer B: dV, dK
    if (lane == 0) {
      constexpr uint32_t idesc_g = idesc_tf32_f32(128, DH, false, false);
      const uint64_t ddo32 = smem_desc(sbase + Tr::OFF_DO32, 16, 1024, 2u);
      const uint64_t dq32 = smem_desc(sbase + Tr::OFF_Q32, 16, 1024, 2u);
      bool ok = true;
      for (int h = 0; ok && h < 2 * nq; ++h) {
        const int i = h >> 1, hh = h & 1, s = i % QS;
        if (!mbar_wait(ds_ready(hh), i & 1, abort_flag, kSiteMma)) { ok = false; break; }
        if (hh == 0 && !mbar_wait(cvt_full(s), (i / QS) & 1, abort_flag, kSiteMma)) { ok = false; break; }
        tc_fence_after();
        // K = 8 query rows per tf32 MMA: rows q0..q0+7 are 32 bytes at offset
        // (q0 % 32) * 4 of panel q0 / 32 of the transposed fp32 tile.
        const uint64_t stage_off = static_cast<uint64_t>((s * Tr::TILE32) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t acc = (h > 0 || ks > 0) ? 1u : 0u;
          const int q0 = hh * 64 + ks * 8;
          const uint64_t boff = stage_off + (((q0 >> 5) * Tr::PANEL32 + (q0 & 31) * 4) >> 4);
          mma_ts_tf32(tmem + Tr::TM_DV, tmem + Tr::tm_st(hh) + 8 * ks, ddo32 + boff, idesc_g, acc);
          mma_ts_tf32(tmem + Tr::TM_DK, tmem + Tr::tm_dpt(hh) + 8 * ks, dq32 + boff, idesc_g, acc);
        }
        mma_commit(kvmma_done(hh));
        if (hh == 1) mma_commit(qd_empty(s));
      }
      if (ok) mma_commit(dkv_final);
      else {
        mma_commit(drain(1));
        mbar_wait_drain(drain(1), 0);
      }
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T, dQ and dK/dV epilogues
    const int w = warp >> 2;                  // this warpgroup's half of every Q tile and TMEM buffer
    const int kk = (warp & 3) * 32 + lane;    // TMEM lane: key (S^T, dP^T, dK, dV) or query row (dQ)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = k0 + kk;
    const bool key_ok = key < p.N;
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    const int qrow_tok = kk < p.rows ? kk / p.g : (1 << 30);
    const int qrow_head = kvh * p.g + kk % p.g;
    uint8_t* ds_smem = smem + Tr::OFF_DS;
    bool ok = true;

    // dQ of Q tile i: TMEM -> fp32 accumulator (this warpgroup: dh/2 columns).
    auto dq_epilogue = [&](int i) {
      float v[DH / 2];
      tmem_ld_half<DH>(lane_addr + Tr::tm_dq(i) + w * (DH / 2), v);
      tc_fence_before();
      mbar_arrive(dq_empty(i & 1));
      const int tok = (qt_first + i) * p.T + qrow_tok;
      if (tok < p.N) {
        float* dst = p.dq_acc + ((static_cast<size_t>(b) * p.N + tok) * p.Hq + qrow_head) * DH + w * (DH / 2);
#pragma unroll
        for (int c = 0; c < DH / 2; c += 4)
          atomicAdd(reinterpret_cast<float4*>(dst + c), make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]));
      }
    };

    for (int i = 0; i < nq; ++i) {
      const int s = i % QS, qt = qt_first + i;
      ok = __all_sync(0xffffffffu, mbar_wait(qd_full(s), (i / QS) & 1, abort_flag, kSiteSoftmax) &&
                                       mbar_wait(s_full(w), i & 1, abort_flag, kSiteSoftmax));
      if (!ok) break;
      tc_fence_after();
      const bool masked = p.causal && (k0 + NK - 1 > qt * p.T);
      const int key_rel = key - qt * p.T;  // visible iff key_rel <= rtok[r]
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int col0 = 64 * w + 32 * c;  // first query row (of the 128-row tile) of this chunk
        const float* lse2 = reinterpret_cast<const float*>(smem + Tr::OFF_STAT + s * 1024) + col0;
        const float* Dv = lse2 + 128;
        uint32_t sr[64];  // [0,32): S^T, [32,64): dP^T
        tmem_ld32x2(lane_addr + Tr::tm_st(w) + 32 * c, lane_addr + Tr::tm_dpt(w) + 32 * c, sr);
        uint32_t pt[32], dst[32], dsb[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2 + e);
          const float4 d4 = *reinterpret_cast<const float4*>(Dv + e);
#pragma unroll
          for (int u = 0; u < 4; u += 2) {
            const float2 nl = u == 0 ? make_float2(-l4.x, -l4.y) : make_float2(-l4.z, -l4.w);
            const float2 nd = u == 0 ? make_float2(-d4.x, -d4.y) : make_float2(-d4.z, -d4.w);
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[e + u]), __uint_as_float(sr[e + u + 1])),
                                        sl2, nl);
            float p0 = ex2(x.x), p1 = ex2(x.y);
            if (!key_ok) p0 = p1 = 0.f;
            if (masked) {
              if (key_rel > rtok[col0 + e + u]) p0 = 0.f;
              if (key_rel > rtok[col0 + e + u + 1]) p1 = 0.f;
            }
            const float2 t = __fadd2_rn(
                make_float2(__uint_as_float(sr[32 + e + u]), __uint_as_float(sr[32 + e + u + 1])), nd);
            const float2 ds = __fmul2_rn(make_float2(p0, p1), t);
            pt[e + u] = __float_as_uint(p0);
            pt[e + u + 1] = __float_as_uint(p1);
            dst[e + u] = round_tf32(ds.x);
            dst[e + u + 1] = round_tf32(ds.y);
            dsb[(e + u) >> 1] = pack_bf16x2(ds.x, ds.y);
          }
        }
        tmem_st32(lane_addr + Tr::tm_st(w) + 32 * c, pt);
        tmem_st32(lane_addr + Tr::tm_dpt(w) + 32 * c, dst);
        // dS (bf16) for the dQ MMA: the dQ of the previous Q tile read this
        // buffer, so wait for it before the first write of a tile.
        if (c == 0 && i > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(dq_full, (i - 1) & 1, abort_flag, kSiteSoftmax));
          if (!ok) break;
        }
        // dS[q][key] for q = col0..col0+31 into the MN-major 128B-swizzled tile:
        // panel q / 64, key row kk (128 bytes), 16-byte chunk (q % 64) / 8.
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int q = col0 + 8 * ch;
          const int panel = q >> 6, chunk = (q & 63) >> 3;
          *reinterpret_cast<uint4*>(ds_smem + panel * 16384 + kk * 128 + ((chunk ^ (kk & 7)) << 4)) =
              make_uint4(dsb[4 * ch], dsb[4 * ch + 1], dsb[4 * ch + 2], dsb[4 * ch + 3]);
        }
      }
      if (!ok) break;
      tmem_wait_st();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ds_ready(w));
      if (i > 0) {
        tc_fence_after();
        dq_epilogue(i - 1);
      }
    }
    if (ok && nq > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full, (nq - 1) & 1, abort_flag, kSiteEpilogue));
      if (ok) {
        tc_fence_after();
        dq_epilogue(nq - 1);
      }
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
  if (warp == Tr::WARP_MMA_A) tmem_dealloc(tmem, 512);
}

}  // namespace sqa

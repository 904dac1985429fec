// sqa_bwd_tf32.cuh -- Sparse Query Attention backward, main kernel for head
// dims 16 and 32 (the SQAT-m shapes).
//
// Same decomposition as sqa_bwd_kernel (one CTA per 128-key tile, batch and KV
// head; stacked Q tiles of the g query heads of the group, so dK and dV are
// reduced over the group inside the tensor-core accumulation), organised for
// small head dims.  There every tensor-core instruction is tiny (N = dh) and
// costs the tensor pipe a fixed number of cycles whatever its size, so the
// schedule is built around keeping MMAs in flight while the softmax warps work:
//
//  * dV += P^T dO and dK += dS^T Q run as tf32 MMAs with K-major operands (tf32
//    operands stored MN-major produced zeros on this hardware).  P^T and dS^T
//    stay in fp32 in TMEM, in place; the transposed fp32 copies of the Q and dO
//    tiles come ready-made from the prep kernel and are bulk-copied.  dS is
//    rounded to tf32 (to nearest), P is passed as is.  tf32 keeps bf16's
//    exponent range and three more mantissa bits, which matters when a large
//    query group sums many terms into one dK or dV row.  dQ = dS K sums only
//    over keys and runs in bf16 (dS as bf16 in shared memory, K as loaded).
//    S^T = K Q^T and dP^T = V dO^T run in bf16 (exact products).
//
//  * The 128-row Q tile is split into two 64-column halves, processed one after
//    the other by both warpgroups (32 columns each).  Halves rotate through
//    three TMEM buffers: while the warpgroups work on one, the dV / dK MMAs of
//    the previous one run and S^T / dP^T of the next one are ready.
//
//  * Three MMA-issuing threads, each in its own warp: A issues S^T / dP^T and
//    dQ, DV issues the dV MMAs, DK the dK MMAs.  dS has two shared-memory
//    buffers, so the softmax warps never wait for the dQ of the previous tile.
//
// Roles (384 threads):
//   warps 0-7   P^T / dS^T (warpgroup w: columns 32 w .. 32 w + 31 of each half),
//               the dQ epilogue (fp32 atomics) and the dK / dV epilogue
//   warp 8      TMA producer (K, V once; Q, dO, their fp32 images, lse2, D per Q tile)
//   warp 9      TMEM allocator and MMA issuer A; warp 10 issuer DV; warp 11 issuer DK
// TMEM: buffer x (0..2): S^T at 128 x, dP^T at 128 x + 64 (64 columns each);
// dV at 384, dK at 416, dQ of Q tile i at 448 + 32 (i % 2).
// The softmax statistics arrive negated (-lse * log2 e and -D), so they are added.
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
}  // namespace dev

template <int DH>
struct BwdTf32Traits {
  static_assert(DH == 16 || DH == 32, "tf32 backward handles dh 16 and 32");
  static constexpr int NK = kBwdTile, BM = kBwdTile;
  static constexpr int ROWB = DH * 2;  // bf16 row bytes (one swizzle panel)
  static constexpr uint32_t LAYOUT = ROWB == 32 ? 6u : 4u;  // bf16 tiles: SW32 / SW64
  // fp32 images: [dh][128] K-major with a 128-byte swizzle, four panels of 32
  // rows, each panel dh lines of 128 bytes (tf32_image_index).
  static constexpr int PANEL32 = DH * 128;
  static constexpr int TILE = 128 * DH * 2;
  static constexpr int TILE32 = 128 * DH * 4;
  static constexpr int QS = DH == 16 ? 3 : 2;  // Q / dO stages (shared memory bounds dh 32 to two)
  static constexpr int NBUF = 3;  // S^T / dP^T buffers in TMEM
  static constexpr int DS_BYTES = 128 * 128 * 2;  // bf16 dS, MN-major (query rows contiguous)
  static constexpr int OFF_DS = 0;                 // two buffers: Q tile i uses buffer i % 2
  static constexpr int OFF_K = OFF_DS + 2 * DS_BYTES;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;
  static constexpr int OFF_DO = OFF_Q + QS * TILE;
  static constexpr int OFF_Q32 = OFF_DO + QS * TILE;
  static constexpr int OFF_DO32 = OFF_Q32 + QS * TILE32;
  static constexpr int OFF_STAT = OFF_DO32 + QS * TILE32;  // per stage: lse2[128], D[128]
  static constexpr int OFF_RTOK = OFF_STAT + QS * 1024;
  static constexpr int OFF_BAR = OFF_RTOK + 512;
  // kv_full, qd_full[3], qd_empty[3], s_full[3], ds_ready[3], kvmma_done[3], dsq_ready[2],
  // dq_full[2], dq_empty[2], dkv_final, drain[3]
  static constexpr int N_BARS = 26;
  static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
  // Enough shared memory that only one CTA fits per SM (each holds all 512 TMEM columns).
  static constexpr int SMEM_BYTES = (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) + 1024;
  static constexpr uint32_t TM_DV = 384, TM_DK = 416;
  __host__ __device__ static constexpr uint32_t tm_st(int x) { return 128u * x; }
  __host__ __device__ static constexpr uint32_t tm_dpt(int x) { return 128u * x + 64u; }
  __host__ __device__ static constexpr uint32_t tm_dq(int i) { return 448u + 32u * (i & 1); }
  static constexpr int THREADS = 384;
  static constexpr int WARP_PRODUCER = 8, WARP_MMA_A = 9, WARP_MMA_DV = 10, WARP_MMA_DK = 11;
  static_assert(OFF_Q32 % 1024 == 0 && TILE32 % 1024 == 0, "fp32 images need 1024-byte alignment");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// P^T, tf32-rounded dS^T and bf16 dS for 32 query columns of one key row (the
// calling thread's TMEM lane).  sr: S^T in [0, 32), dP^T in [32, 64); nl2, nd:
// the columns' negated statistics (-lse * log2 e, -D); with MASK, P is zeroed
// where lim > rtok[column].
template <bool MASK>
__device__ __forceinline__ void bwd_p_ds(const uint32_t (&sr)[64], const float* nl2, const float* nd,
                                         const int* rtok, int lim, float2 sl2, uint32_t (&pt)[32],
                                         uint32_t (&dst)[32], uint32_t (&dsb)[16]) {
  using namespace dev;
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 l4 = *reinterpret_cast<const float4*>(nl2 + e);
    const float4 d4 = *reinterpret_cast<const float4*>(nd + e);
    int4 r4 = make_int4(0, 0, 0, 0);
    if (MASK) r4 = *reinterpret_cast<const int4*>(rtok + e);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float2 l = u == 0 ? make_float2(l4.x, l4.y) : make_float2(l4.z, l4.w);
      const float2 d = u == 0 ? make_float2(d4.x, d4.y) : make_float2(d4.z, d4.w);
      const float2 xx = __ffma2_rn(make_float2(__uint_as_float(sr[e + u]), __uint_as_float(sr[e + u + 1])), sl2, l);
      float p0 = ex2(xx.x), p1 = ex2(xx.y);
      if (MASK) {
        if (lim > (u == 0 ? r4.x : r4.z)) p0 = 0.f;
        if (lim > (u == 0 ? r4.y : r4.w)) p1 = 0.f;
      }
      const float2 t = __fadd2_rn(make_float2(__uint_as_float(sr[32 + e + u]), __uint_as_float(sr[32 + e + u + 1])), d);
      const float2 ds = __fmul2_rn(make_float2(p0, p1), t);
      pt[e + u] = __float_as_uint(p0);
      pt[e + u + 1] = __float_as_uint(p1);
      dst[e + u] = round_tf32(ds.x);
      dst[e + u + 1] = round_tf32(ds.y);
      dsb[(e + u) >> 1] = pack_bf16x2(ds.x, ds.y);
    }
  }
}

template <int DH>
__global__ void __launch_bounds__(384, 1)
    sqa_bwd_tf32_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                        const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const BwdParams p) {
  using Tr = BwdTf32Traits<DH>;
  using namespace dev;
  constexpr int BM = Tr::BM, NK = Tr::NK, ROWB = Tr::ROWB, QS = Tr::QS, NBUF = Tr::NBUF;

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
  const int nh = 2 * nq;  // halves

  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  const uint32_t kv_full = bar0;
  auto qd_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto qd_empty = [&](int s) { return bar0 + 8u * (4 + s); };
  auto s_full = [&](int x) { return bar0 + 8u * (7 + x); };
  auto ds_ready = [&](int x) { return bar0 + 8u * (10 + x); };
  auto kvmma_done = [&](int x) { return bar0 + 8u * (13 + x); };
  auto dsq_ready = [&](int w) { return bar0 + 8u * (16 + w); };  // warpgroup w wrote its half of dS
  auto dq_full = [&](int x) { return bar0 + 8u * (18 + x); };    // dQ of tile i in buffer x = i % 2 done
  auto dq_empty = [&](int x) { return bar0 + 8u * (20 + x); };
  const uint32_t dkv_final = bar0 + 8u * 22;
  auto drain = [&](int x) { return bar0 + 8u * (23 + x); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* rtok = reinterpret_cast<int*>(smem + Tr::OFF_RTOK);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(qd_full(s), 1);
      mbar_init(qd_empty(s), 3);  // released by the three MMA issuers
    }
    for (int x = 0; x < NBUF; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(ds_ready(x), 256);  // both warpgroups
      mbar_init(kvmma_done(x), 2);  // DV and DK
      mbar_init(drain(x), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(dsq_ready(x), 128);
      mbar_init(dq_full(x), 1);
      mbar_init(dq_empty(x), 256);
    }
    mbar_init(dkv_final, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 128) rtok[threadIdx.x] = threadIdx.x < p.rows ? threadIdx.x / p.g : (1 << 30);
  if (p.rows < BM) {  // stacked rows the TMA box does not cover stay zero
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
      const uint32_t qd_bytes = 2u * p.rows * ROWB + 2u * 512u + 2u * Tr::TILE32;
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
        bulk_load(sbase + Tr::OFF_Q32 + s * Tr::TILE32, p.q32 + slot * DH, Tr::TILE32, qd_full(s));
        bulk_load(sbase + Tr::OFF_DO32 + s * Tr::TILE32, p.do32 + slot * DH, Tr::TILE32, qd_full(s));
        issued = i + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(kv_full, 0);
        for (int i = max(0, issued - QS); i < issued; ++i) mbar_wait_drain(qd_full(i % QS), (i / QS) & 1);
      }
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
      // S^T and dP^T of half h (query rows 64 (h % 2) .. of Q tile h / 2) into
      // TMEM buffer h % 3, once its Q / dO tile has landed and DV and DK have
      // finished reading the half that used the buffer before (h - 3).
      auto issue_half = [&](int h) -> bool {
        const int i = h >> 1, s = i % QS, x = h % NBUF;
        if ((h & 1) == 0 && !mbar_wait(qd_full(s), (i / QS) & 1, abort_flag, kSiteMma)) return false;
        if (h >= NBUF && !mbar_wait(kvmma_done(x), ((h / NBUF) - 1) & 1, abort_flag, kSiteMma)) return false;
        tc_fence_after();
        const uint64_t off = static_cast<uint64_t>((s * Tr::TILE + (h & 1) * 64 * ROWB) >> 4);
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          mma_ss(tmem + Tr::tm_st(x), dk + 2 * ks, dqt + off + 2 * ks, idesc_s, ks > 0);
          mma_ss(tmem + Tr::tm_dpt(x), dv + 2 * ks, ddo + off + 2 * ks, idesc_s, ks > 0);
        }
        mma_commit(s_full(x));
        return true;
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag, kSiteMma);
      for (int h = 0; ok && h < NBUF && h < nh; ++h) ok = issue_half(h);
      for (int i = 0; ok && i < nq; ++i) {
        // dQ of tile i once both warpgroups wrote their half of dS, into the
        // dQ buffer the epilogue of tile i - 2 has emptied.
        if (!mbar_wait(dsq_ready(0), i & 1, abort_flag, kSiteMma) ||
            !mbar_wait(dsq_ready(1), i & 1, abort_flag, kSiteMma)) { ok = false; break; }
        if (i >= 2 && !mbar_wait(dq_empty(i & 1), ((i >> 1) - 1) & 1, abort_flag, kSiteMma)) { ok = false; break; }
        tc_fence_after();
        // dQ = dS K: M = 128 query rows, N = dh, K = 128 keys in steps of 16 (2 KB of dS, 16 K rows).
        const uint64_t dsb = dds + static_cast<uint64_t>(((i & 1) * Tr::DS_BYTES) >> 4);
#pragma unroll
        for (int ks = 0; ks < NK / 16; ++ks)
          mma_ss(tmem + Tr::tm_dq(i), dsb + 128 * ks, dkmn + ((ks * 16 * ROWB) >> 4), idesc_q, ks > 0);
        mma_commit(dq_full(i & 1));
        mma_commit(qd_empty(i % QS));
        if (2 * i + 3 < nh && !(ok = issue_half(2 * i + 3))) break;
        if (2 * i + 4 < nh && !(ok = issue_half(2 * i + 4))) break;
      }
      if (!ok) {
        mma_commit(drain(0));
        mbar_wait_drain(drain(0), 0);
      }
    }
  } else if (warp == Tr::WARP_MMA_DV || warp == Tr::WARP_MMA_DK) {
    // ------------------------------------------------------------ MMA issuers DV (dV += P^T dO) and DK (dK += dS^T Q)
    if (lane == 0) {
      const bool is_dv = warp == Tr::WARP_MMA_DV;
      constexpr uint32_t idesc_g = idesc_tf32_f32(128, DH, false, false);
      const uint64_t dimg = smem_desc(sbase + (is_dv ? Tr::OFF_DO32 : Tr::OFF_Q32), 16, 1024, 2u);
      const uint32_t d_acc = tmem + (is_dv ? Tr::TM_DV : Tr::TM_DK);
      const uint32_t a_col = is_dv ? 0u : 64u;  // P^T or dS^T inside a buffer
      bool ok = true;
      for (int h = 0; h < nh; ++h) {
        const int i = h >> 1, hh = h & 1, s = i % QS, x = h % NBUF;
        if (!mbar_wait(ds_ready(x), (h / NBUF) & 1, abort_flag, kSiteMma)) { ok = false; break; }
        // The image arrived with the Q tile (already complete: the warpgroup waited for it).
        if (hh == 0 && !mbar_wait(qd_full(s), (i / QS) & 1, abort_flag, kSiteMma)) { ok = false; break; }
        tc_fence_after();
        // K = 8 query rows per tf32 MMA: rows q0..q0+7 are 32 bytes at offset
        // (q0 % 32) * 4 of panel q0 / 32 of the image.
        const uint64_t stage_off = static_cast<uint64_t>((s * Tr::TILE32) >> 4);
        const uint32_t a0 = tmem + Tr::tm_st(x) + a_col;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int q0 = hh * 64 + ks * 8;
          const uint64_t boff = stage_off + (((q0 >> 5) * Tr::PANEL32 + (q0 & 31) * 4) >> 4);
          mma_ts_tf32(d_acc, a0 + 8 * ks, dimg + boff, idesc_g, (h > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(kvmma_done(x));
        if (hh == 1) mma_commit(qd_empty(s));
      }
      if (ok) mma_commit(dkv_final);
      else {
        const int x = is_dv ? 1 : 2;
        mma_commit(drain(x));
        mbar_wait_drain(drain(x), 0);
      }
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T, dQ and dK/dV epilogues
    const int w = warp >> 2;                  // warpgroup: 32-column slice of each half, dh/2 columns of dQ, dK, dV
    const int kk = (warp & 3) * 32 + lane;    // TMEM lane: key (S^T, dP^T, dK, dV) or query row (dQ)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = k0 + kk;
    const bool key_ok = key < p.N;
    const bool ragged = k0 + NK > p.N;  // the last key tile: rows past N hold zeros
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    const int qrow_tok = kk < p.rows ? kk / p.g : (1 << 30);
    const int qrow_head = kvh * p.g + kk % p.g;
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
      ok = __all_sync(0xffffffffu, mbar_wait(qd_full(s), (i / QS) & 1, abort_flag, kSiteSoftmax));
      if (!ok) break;
      const bool masked = p.causal && (k0 + NK - 1 > qt * p.T);
      // P is zeroed where lim > rtok[row]: keys past N always, keys after the
      // row's token on the causal diagonal.
      const int lim = !key_ok ? 0x7fffffff : (masked ? key - qt * p.T : -0x7fffffff);
      uint8_t* ds_smem = smem + Tr::OFF_DS + (i & 1) * Tr::DS_BYTES;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        // Both warpgroups work on half hh of the tile: this one on its 32
        // query columns col0 .. col0 + 31.
        const int h = 2 * i + hh, x = h % NBUF;
        const int col0 = 64 * hh + 32 * w;
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(x), (h / NBUF) & 1, abort_flag, kSiteSoftmax));
        if (!ok) break;
        tc_fence_after();
        const float* nl2 = reinterpret_cast<const float*>(smem + Tr::OFF_STAT + s * 1024) + col0;
        uint32_t sr[64];  // [0,32): S^T, [32,64): dP^T
        tmem_ld32x2(lane_addr + Tr::tm_st(x) + 32 * w, lane_addr + Tr::tm_dpt(x) + 32 * w, sr);
        uint32_t pt[32], dst[32], dsb[16];
        if (masked || ragged)
          bwd_p_ds<true>(sr, nl2, nl2 + 128, rtok + col0, lim, sl2, pt, dst, dsb);
        else
          bwd_p_ds<false>(sr, nl2, nl2 + 128, rtok + col0, lim, sl2, pt, dst, dsb);
        tmem_st32(lane_addr + Tr::tm_st(x) + 32 * w, pt);
        tmem_st32(lane_addr + Tr::tm_dpt(x) + 32 * w, dst);
        // dS (bf16) for the dQ MMA: the dQ of Q tile i - 2 read this buffer, so
        // wait for it before the first write of a tile.
        if (hh == 0 && i >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(dq_full(i & 1), ((i >> 1) - 1) & 1, abort_flag, kSiteSoftmax));
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
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(ds_ready(x));
      }
      if (!ok) break;
      // dsq_ready(w) is signalled only after the dQ of tile i - 1 completed,
      // which keeps it at most one phase ahead of issuer A's wait.
      if (i > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(dq_full((i - 1) & 1), ((i - 1) >> 1) & 1, abort_flag, kSiteSoftmax));
        if (!ok) break;
      }
      mbar_arrive(dsq_ready(w));
      if (i > 0) {
        tc_fence_after();
        dq_epilogue(i - 1);
      }
    }
    if (ok && nq > 0) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(dq_full((nq - 1) & 1), ((nq - 1) >> 1) & 1, abort_flag, kSiteEpilogue));
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

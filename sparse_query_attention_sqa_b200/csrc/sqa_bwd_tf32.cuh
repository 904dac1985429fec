// sqa_bwd_tf32.cuh -- Sparse Query Attention backward, main kernel for head
// dims 16 and 32 (the SQAT-m shapes).
//
// Same decomposition as sqa_bwd_kernel (work item = 128-key tile, batch and KV
// head; stacked Q tiles of the g query heads of the group, so dK and dV are
// reduced over the group inside the tensor-core accumulation), organised for
// small head dims.  The grid is persistent: each CTA walks a snake-ordered,
// heaviest-first list of items, with K / V double-buffered so the next item's
// tiles load while the current one finishes.  There every tensor-core instruction is tiny (N = dh) and
// costs the tensor pipe a fixed number of cycles whatever its size, so the
// schedule is built around keeping MMAs in flight while the softmax warps work:
//
//  * dV += P^T dO and dK += dS^T Q run as tf32 MMAs with K-major operands (tf32
//    operands stored MN-major produced zeros on this hardware).  P^T and dS^T
//    stay in fp32 in TMEM, in place; the transposed fp32 copies of the dO and Q
//    tiles are built in shared memory from the bf16 tiles by the DV and DK
//    issuing warps themselves, while the softmax warps work on the tile's
//    first half (the issuers are otherwise waiting for them).  dS is
//    rounded to tf32 (to nearest), P is passed as is.  tf32 keeps bf16's
//    exponent range and three more mantissa bits, which matters when a large
//    query group sums many terms into one dK or dV row.  dQ = dS K sums only
//    over keys and runs in bf16 (dS as bf16 in shared memory, K as loaded).
//    S^T = K Q^T and dP^T = V dO^T run in bf16 (exact products).
//
//  * The 128-row Q tile is split into two 64-column halves; warpgroup w takes
//    half w of every tile, all 64 columns, in four 16-column chunks whose
//    TMEM loads run one chunk ahead of the arithmetic.  (Splitting each half's
//    columns between the warpgroups instead pays every hand-off twice per half
//    and keeps both warpgroups in the same phase.)  Halves rotate through
//    three TMEM buffers: while the warpgroups work on two of them, the dV / dK
//    MMAs of the previous half run and S^T / dP^T of the next are ready.
//
//  * Three MMA-issuing threads, each in its own warp: A issues S^T / dP^T and
//    dQ, DV issues the dV MMAs, DK the dK MMAs.  dS has two shared-memory
//    buffers, so the softmax warps never wait for the dQ of the previous tile.
//
// Roles (384 threads):
//   warps 0-7   P^T / dS^T (warpgroup w: half w of each Q tile), the dQ
//               epilogue (fp32 atomics) and the dK / dV epilogue
//   warp 8      TMA producer (K, V once; Q, dO, lse2, D per Q tile)
//   warp 9      TMEM allocator and MMA issuer A; warp 10 issuer DV (and the dO
//               images); warp 11 issuer DK (and the Q images)
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
// Warp-collective form: every lane calls it, one elected lane issues.
__device__ __forceinline__ void mma_ts_tf32_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
}  // namespace dev

// Offset (in floats) of element (row r, column n) inside the fp32 image of one
// stacked 128-row tile: the tile transposed to [dh][128] and cut into four
// panels of 32 rows, each panel dh lines of 128 bytes with the 128-byte swizzle
// (16-byte chunk c of line n stored at chunk c ^ (n % 8)).  This is the K-major
// operand layout of a tf32 MMA whose contraction runs over the tile's rows.
__host__ __device__ __forceinline__ int tf32_image_index(int r, int n, int dh) {
  return (r >> 5) * dh * 32 + n * 32 + ((((r & 31) >> 2) ^ (n & 7)) << 2) + (r & 3);
}

// The fp32 image of a bf16 tile as the tensor map wrote it into shared memory
// (row r at r * 2 dh bytes, its 16-byte chunks permuted by the 32-byte swizzle
// at dh 16 and the 64-byte one at dh 32: byte offset o is stored at
// o ^ (((o >> 7) & m) << 4), m = 1 or 3), by the 32 lanes of one warp: lane l
// takes rows l, l + 32, l + 64, l + 96.  For a fixed column the 32 lanes write
// the 32 words of one 128-byte line, so the stores are free of bank conflicts.
template <int DH>
__device__ __forceinline__ void to_tf32_image(const uint8_t* src, float* dst, int lane) {
  constexpr uint32_t ROWB = DH * 2, M = DH == 16 ? 1u : 3u;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = 32 * k + lane;
#pragma unroll
    for (int c = 0; c < DH / 8; ++c) {
      const uint32_t o = r * ROWB + 16u * c;
      const uint4 v = *reinterpret_cast<const uint4*>(src + (o ^ (((o >> 7) & M) << 4)));
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {  // a bf16 is the upper half of its fp32 value
        dst[tf32_image_index(r, 8 * c + 2 * e, DH)] = __uint_as_float(wv[e] << 16);
        dst[tf32_image_index(r, 8 * c + 2 * e + 1, DH)] = __uint_as_float(wv[e] & 0xffff0000u);
      }
    }
  }
}

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
  static constexpr int QS = DH == 16 ? 4 : 2;  // Q / dO stages (shared memory bounds dh 32 to two)
  static constexpr int NBUF = 3;  // S^T / dP^T buffers in TMEM
  static constexpr int DS_BYTES = 128 * 128 * 2;  // bf16 dS, MN-major (query rows contiguous)
  static constexpr int OFF_DS = 0;                 // two buffers: Q tile i uses buffer i % 2
  static constexpr int OFF_K = OFF_DS + 2 * DS_BYTES;  // two buffers each (item r uses r % 2)
  static constexpr int OFF_V = OFF_K + 2 * TILE;
  static constexpr int OFF_Q = OFF_V + 2 * TILE;
  static constexpr int OFF_DO = OFF_Q + QS * TILE;
  static constexpr int OFF_Q32 = OFF_DO + QS * TILE;
  static constexpr int OFF_DO32 = OFF_Q32 + QS * TILE32;
  static constexpr int OFF_STAT = OFF_DO32 + QS * TILE32;  // per stage: lse2[128], D[128]
  static constexpr int OFF_RTOK = OFF_STAT + QS * 1024;
  static constexpr int OFF_BAR = OFF_RTOK + 512;
  // Barrier slots: kv_full[2], kv_empty[2], qd_full[QS], qd_empty[QS], s_full[3], ds_ready[3],
  // kvmma_done[3], dsq_ready[2], dq_full[2], dq_empty[2], dkv_final, dkv_free, drain[3].
  static constexpr int B_QF = 4, B_QE = B_QF + QS, B_SF = B_QE + QS, B_DR = B_SF + NBUF, B_KD = B_DR + NBUF;
  static constexpr int B_DSQ = B_KD + NBUF, B_DQF = B_DSQ + 2, B_DQE = B_DQF + 2, B_DKV = B_DQE + 2;
  static constexpr int B_DRAIN = B_DKV + 2;
  static constexpr int N_BARS = B_DRAIN + 3;
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

// P^T, tf32-rounded dS^T and bf16 dS for 16 query columns of one key row (the
// calling thread's TMEM lane).  sr: S^T in [0, 16), dP^T in [16, 32); nl2, nd:
// the columns' negated statistics (-lse * log2 e, -D); P is zeroed where
// lim > rtok[column].  dS is rounded to the nearest tf32 value by
// Veltkamp splitting (with C = 2^13 + 1, C x - (C x - x) keeps the 11 leading
// significant bits, rounded to nearest), in packed fp32 pairs.
__device__ __forceinline__ void bwd_p_ds16(const uint32_t (&sr)[32], const float* nl2, const float* nd,
                                           const int* rtok, int lim, float2 sl2, uint32_t (&pt)[16],
                                           uint32_t (&dst)[16], uint32_t (&dsb)[8]) {
  using namespace dev;
  const float2 split = make_float2(8193.f, 8193.f), minus1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int e = 0; e < 16; e += 4) {
    const float4 l4 = *reinterpret_cast<const float4*>(nl2 + e);
    const float4 d4 = *reinterpret_cast<const float4*>(nd + e);
    const int4 r4 = *reinterpret_cast<const int4*>(rtok + e);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float2 l = u == 0 ? make_float2(l4.x, l4.y) : make_float2(l4.z, l4.w);
      const float2 d = u == 0 ? make_float2(d4.x, d4.y) : make_float2(d4.z, d4.w);
      const float2 xx = __ffma2_rn(make_float2(__uint_as_float(sr[e + u]), __uint_as_float(sr[e + u + 1])), sl2, l);
      float p0 = ex2(xx.x), p1 = ex2(xx.y);
      if (lim > (u == 0 ? r4.x : r4.z)) p0 = 0.f;
      if (lim > (u == 0 ? r4.y : r4.w)) p1 = 0.f;
      const float2 t = __fadd2_rn(make_float2(__uint_as_float(sr[16 + e + u]), __uint_as_float(sr[16 + e + u + 1])), d);
      const float2 ds = __fmul2_rn(make_float2(p0, p1), t);
      const float2 cx = __fmul2_rn(ds, split);
      const float2 hi = __ffma2_rn(__ffma2_rn(ds, minus1, cx), minus1, cx);
      pt[e + u] = __float_as_uint(p0);
      pt[e + u + 1] = __float_as_uint(p1);
      dst[e + u] = __float_as_uint(hi.x);
      dst[e + u + 1] = __float_as_uint(hi.y);
      dsb[(e + u) >> 1] = pack_bf16x2(ds.x, ds.y);
    }
  }
}

// One work item of the persistent backward: a 128-key tile of one (batch, KV
// head).  Items are numbered key tile major, so under a causal mask the first
// key tiles, which see the most Q tiles, come first.
struct BwdItem {
  int b, kvh, bh, k0, qt_first, nq;
};
__device__ __forceinline__ BwdItem bwd_decode(const BwdParams& p, int item) {
  BwdItem it;
  const int kt = item / p.n_bh;
  it.bh = item % p.n_bh;
  it.b = it.bh / p.Hkv;
  it.kvh = it.bh % p.Hkv;
  it.k0 = kt * kBwdTile;
  it.qt_first = p.causal ? it.k0 / p.T : 0;
  it.nq = p.n_qt - it.qt_first;
  return it;
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

  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  auto kv_full = [&](int kb) { return bar0 + 8u * (0 + kb); };
  auto kv_empty = [&](int kb) { return bar0 + 8u * (2 + kb); };
  auto qd_full = [&](int s) { return bar0 + 8u * (Tr::B_QF + s); };
  auto qd_empty = [&](int s) { return bar0 + 8u * (Tr::B_QE + s); };
  auto s_full = [&](int x) { return bar0 + 8u * (Tr::B_SF + x); };
  auto ds_ready = [&](int x) { return bar0 + 8u * (Tr::B_DR + x); };
  auto kvmma_done = [&](int x) { return bar0 + 8u * (Tr::B_KD + x); };
  auto dsq_ready = [&](int w) { return bar0 + 8u * (Tr::B_DSQ + w); };  // warpgroup w wrote its columns of dS
  auto dq_full = [&](int x) { return bar0 + 8u * (Tr::B_DQF + x); };    // dQ of tile G in buffer x = G % 2 done
  auto dq_empty = [&](int x) { return bar0 + 8u * (Tr::B_DQE + x); };
  const uint32_t dkv_final = bar0 + 8u * Tr::B_DKV;       // dV / dK of the item complete
  const uint32_t dkv_free = bar0 + 8u * (Tr::B_DKV + 1);  // the epilogue has read them
  auto drain = [&](int x) { return bar0 + 8u * (Tr::B_DRAIN + x); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* rtok = reinterpret_cast<int*>(smem + Tr::OFF_RTOK);

  if (threadIdx.x == 0) {
    for (int kb = 0; kb < 2; ++kb) {
      mbar_init(kv_full(kb), 1);
      mbar_init(kv_empty(kb), 1);  // issuer A
    }
    for (int s = 0; s < QS; ++s) {
      mbar_init(qd_full(s), 1);
      mbar_init(qd_empty(s), 3);  // released by the three MMA issuers
    }
    for (int x = 0; x < NBUF; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(ds_ready(x), 128);  // the warpgroup that owns the half
      mbar_init(kvmma_done(x), 2);  // DV and DK
      mbar_init(drain(x), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(dsq_ready(x), 128);
      mbar_init(dq_full(x), 1);
      mbar_init(dq_empty(x), 256);
    }
    mbar_init(dkv_final, 2);
    mbar_init(dkv_free, 256);
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

  // Counters shared by every role: r = this CTA's item round, gt = Q tiles of
  // earlier items.  Global tile G = gt + i, global half H = 2 G + hh.
  if (warp == Tr::WARP_PRODUCER) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmDO);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      const uint32_t qd_bytes = 2u * p.rows * ROWB + 2u * 512u;
      int gt = 0, items_issued = 0, tiles_issued = 0;
      bool ok = true;
      for (int r = 0, item; ok && (item = snake_item(r, p.n_items)) >= 0; ++r) {
        const BwdItem it = bwd_decode(p, item);
        const int kb = r & 1;
        if (r >= 2 && !mbar_wait(kv_empty(kb), ((r >> 1) - 1) & 1, abort_flag, kSiteProducer)) break;
        mbar_expect_tx(kv_full(kb), 2u * Tr::TILE);
        tma_load_4d(sbase + Tr::OFF_K + kb * Tr::TILE, &tmK, kv_full(kb), 0, it.kvh, it.k0, it.b);
        tma_load_4d(sbase + Tr::OFF_V + kb * Tr::TILE, &tmV, kv_full(kb), 0, it.kvh, it.k0, it.b);
        items_issued = r + 1;
        for (int i = 0; i < it.nq; ++i) {
          const int G = gt + i, s = G % QS, qt = it.qt_first + i;
          if (G >= QS && !mbar_wait(qd_empty(s), ((G / QS) - 1) & 1, abort_flag, kSiteProducer)) {
            ok = false;
            break;
          }
          mbar_expect_tx(qd_full(s), qd_bytes);
          tma_load_4d(sbase + Tr::OFF_Q + s * Tr::TILE, &tmQ, qd_full(s), 0, it.kvh * p.g, qt * p.T, it.b);
          tma_load_4d(sbase + Tr::OFF_DO + s * Tr::TILE, &tmDO, qd_full(s), 0, it.kvh * p.g, qt * p.T, it.b);
          const size_t slot = (static_cast<size_t>(it.bh) * p.n_qt + qt) * kBwdTile;
          bulk_load(sbase + Tr::OFF_STAT + s * 1024, p.lse2 + slot, 512, qd_full(s));
          bulk_load(sbase + Tr::OFF_STAT + s * 1024 + 512, p.D + slot, 512, qd_full(s));
          tiles_issued = G + 1;
        }
        gt += it.nq;
      }
      if (*abort_flag) {  // let in-flight copies land before the CTA exits
        for (int j = max(0, items_issued - 2); j < items_issued; ++j) mbar_wait_drain(kv_full(j & 1), (j >> 1) & 1);
        for (int G = max(0, tiles_issued - QS); G < tiles_issued; ++G) mbar_wait_drain(qd_full(G % QS), (G / QS) & 1);
      }
    }
  } else if (warp == Tr::WARP_MMA_A) {
    // ------------------------------------------------------------ MMA issuer A: S^T, dP^T, dQ
    // The whole warp runs the loop; one elected lane issues each MMA.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);  // S^T, dP^T halves
    constexpr uint32_t idesc_q = idesc_bf16_f32(128, DH, true, true);    // dQ = dS K (both MN-major)
    // Descriptors of buffer / stage 0 and K-step 0; others add their byte offset / 16.
    const uint64_t dk0 = smem_desc(sbase + Tr::OFF_K, 16, 8 * ROWB, Tr::LAYOUT);
    const uint64_t dv0 = smem_desc(sbase + Tr::OFF_V, 16, 8 * ROWB, Tr::LAYOUT);
    const uint64_t dqt = smem_desc(sbase + Tr::OFF_Q, 16, 8 * ROWB, Tr::LAYOUT);
    const uint64_t ddo = smem_desc(sbase + Tr::OFF_DO, 16, 8 * ROWB, Tr::LAYOUT);
    const uint64_t dds = smem_desc(sbase + Tr::OFF_DS, 16384, 1024, 2u);
    const uint64_t dkmn0 = smem_desc(sbase + Tr::OFF_K, NK * ROWB, 8 * ROWB, Tr::LAYOUT);
    int gt = 0;
    bool ok = true;
    for (int r = 0, item; ok && (item = snake_item(r, p.n_items)) >= 0; ++r) {
      const BwdItem it = bwd_decode(p, item);
      const int kb = r & 1, nh = 2 * it.nq;
      const uint64_t koff = static_cast<uint64_t>((kb * Tr::TILE) >> 4);
      if (!(ok = mbar_wait_warp(kv_full(kb), (r >> 1) & 1, abort_flag, kSiteMma))) break;
      // S^T and dP^T of the item's half hl (query rows 64 (hl % 2) .. of its tile
      // hl / 2) into TMEM buffer H % 3, once the Q / dO tile has landed and DV and
      // DK have finished reading the half that used the buffer before (H - 3).
      auto issue_half = [&](int hl) -> bool {
        const int G = gt + (hl >> 1), H = 2 * gt + hl, s = G % QS, x = H % NBUF;
        if ((hl & 1) == 0 && !mbar_wait_warp(qd_full(s), (G / QS) & 1, abort_flag, kSiteMma)) return false;
        if (H >= NBUF && !mbar_wait_warp(kvmma_done(x), ((H / NBUF) - 1) & 1, abort_flag, kSiteMma)) return false;
        tc_fence_after();
        const uint64_t off = static_cast<uint64_t>((s * Tr::TILE + (hl & 1) * 64 * ROWB) >> 4);
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          mma_ss_w(tmem + Tr::tm_st(x), dk0 + koff + 2 * ks, dqt + off + 2 * ks, idesc_s, ks > 0);
          mma_ss_w(tmem + Tr::tm_dpt(x), dv0 + koff + 2 * ks, ddo + off + 2 * ks, idesc_s, ks > 0);
        }
        mma_commit_w(s_full(x));
        return true;
      };
      for (int hl = 0; ok && hl < NBUF && hl < nh; ++hl) ok = issue_half(hl);
      for (int i = 0; ok && i < it.nq; ++i) {
        const int G = gt + i;
        // S^T / dP^T of the next tile's second half go ahead of this tile's dQ,
        // so that the softmax warps find them computed when they get there.
        // (The next-but-one tile's first half stays behind dQ: with two Q / dO
        // stages its load waits for the stage this dQ releases.)
        if (2 * i + 3 < nh && !(ok = issue_half(2 * i + 3))) break;
        // dQ of tile G once both warpgroups wrote their columns of dS, into the
        // dQ buffer the epilogue of tile G - 2 has emptied.
        if (!mbar_wait_warp(dsq_ready(0), G & 1, abort_flag, kSiteMma) ||
            !mbar_wait_warp(dsq_ready(1), G & 1, abort_flag, kSiteMma)) { ok = false; break; }
        if (G >= 2 && !mbar_wait_warp(dq_empty(G & 1), ((G >> 1) - 1) & 1, abort_flag, kSiteMma)) { ok = false; break; }
        tc_fence_after();
        // dQ = dS K: M = 128 query rows, N = dh, K = 128 keys in steps of 16 (2 KB of dS, 16 K rows).
        const uint64_t dsb = dds + static_cast<uint64_t>(((G & 1) * Tr::DS_BYTES) >> 4);
#pragma unroll
        for (int ks = 0; ks < NK / 16; ++ks)
          mma_ss_w(tmem + Tr::tm_dq(G), dsb + 128 * ks, dkmn0 + koff + ((ks * 16 * ROWB) >> 4), idesc_q, ks > 0);
        mma_commit_w(dq_full(G & 1));
        mma_commit_w(qd_empty(G % QS));
        if (2 * i + 4 < nh && !(ok = issue_half(2 * i + 4))) break;
      }
      if (!ok) break;
      mma_commit_w(kv_empty(kb));  // every MMA reading this item's K and V has been issued
      gt += it.nq;
    }
    if (!ok) {
      mma_commit_w(drain(0));
      mbar_wait_drain(drain(0), 0);
    }
  } else if (warp == Tr::WARP_MMA_DV || warp == Tr::WARP_MMA_DK) {
    // ------------------------------------------------------------ MMA issuers DV (dV += P^T dO) and DK (dK += dS^T Q)
    // The whole warp runs the loop; one elected lane issues each MMA.
    const bool is_dv = warp == Tr::WARP_MMA_DV;
    constexpr uint32_t idesc_g = idesc_tf32_f32(128, DH, false, false);
    const uint64_t dimg = smem_desc(sbase + (is_dv ? Tr::OFF_DO32 : Tr::OFF_Q32), 16, 1024, 2u);
    const uint32_t d_acc = tmem + (is_dv ? Tr::TM_DV : Tr::TM_DK);
    const uint32_t a_col = is_dv ? 0u : 64u;  // P^T or dS^T inside a buffer
    int gt = 0;
    bool ok = true;
    for (int r = 0, item; ok && (item = snake_item(r, p.n_items)) >= 0; ++r) {
      const BwdItem it = bwd_decode(p, item);
      for (int hl = 0; hl < 2 * it.nq; ++hl) {
        const int G = gt + (hl >> 1), H = 2 * gt + hl, s = G % QS, x = H % NBUF;
        if ((hl & 1) == 0) {
          // This warp's fp32 image of tile G (dO for DV, Q for DK), built while
          // the softmax warps work on the tile.  The stage's previous image was
          // last read by this warp's MMAs of tile G - QS, which completed before
          // the producer could refill the stage (qd_empty), so before qd_full.
          if (!(ok = mbar_wait_warp(qd_full(s), (G / QS) & 1, abort_flag, kSiteMma))) break;
          to_tf32_image<DH>(smem + (is_dv ? Tr::OFF_DO : Tr::OFF_Q) + s * Tr::TILE,
                            reinterpret_cast<float*>(smem + (is_dv ? Tr::OFF_DO32 : Tr::OFF_Q32) + s * Tr::TILE32),
                            lane);
          fence_async_smem();  // the image, to the tensor core's reads
          __syncwarp();
        }
        if (!(ok = mbar_wait_warp(ds_ready(x), (H / NBUF) & 1, abort_flag, kSiteMma))) break;
        // The accumulators still hold the previous item until its epilogue has read them.
        if (hl == 0 && r > 0 && !(ok = mbar_wait_warp(dkv_free, (r - 1) & 1, abort_flag, kSiteMma))) break;
        tc_fence_after();
        // K = 8 query rows per tf32 MMA: rows q0..q0+7 are 32 bytes at offset
        // (q0 % 32) * 4 of panel q0 / 32 of the image.
        const uint64_t stage_off = static_cast<uint64_t>((s * Tr::TILE32) >> 4);
        const uint32_t a0 = tmem + Tr::tm_st(x) + a_col;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int q0 = (hl & 1) * 64 + ks * 8;
          const uint64_t boff = stage_off + (((q0 >> 5) * Tr::PANEL32 + (q0 & 31) * 4) >> 4);
          mma_ts_tf32_w(d_acc, a0 + 8 * ks, dimg + boff, idesc_g, (hl > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit_w(kvmma_done(x));
        if (hl & 1) mma_commit_w(qd_empty(s));
      }
      if (!ok) break;
      mma_commit_w(dkv_final);
      gt += it.nq;
    }
    if (!ok) {
      const int x = is_dv ? 1 : 2;
      mma_commit_w(drain(x));
      mbar_wait_drain(drain(x), 0);
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T, dQ and dK/dV epilogues
    const int w = warp >> 2;                  // warpgroup: 32-column slice of each half, dh/2 columns of dQ, dK, dV
    const int kk = (warp & 3) * 32 + lane;    // TMEM lane: key (S^T, dP^T, dK, dV) or query row (dQ)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    const int qrow_tok = kk < p.rows ? kk / p.g : (1 << 30);
    int gt = 0;
    bool ok = true;
    for (int r = 0, item; ok && (item = snake_item(r, p.n_items)) >= 0; ++r) {
      const BwdItem it = bwd_decode(p, item);
      const int key = it.k0 + kk;
      const bool key_ok = key < p.N;
      const int qrow_head = it.kvh * p.g + kk % p.g;

      // dQ of the item's tile i (global G): TMEM -> fp32 accumulator (this warpgroup: dh/2 columns).
      auto dq_epilogue = [&](int i) {
        const int G = gt + i;
        float v[DH / 2];
        tmem_ld_half<DH>(lane_addr + Tr::tm_dq(G) + w * (DH / 2), v);
        tc_fence_before();
        mbar_arrive(dq_empty(G & 1));
        const int tok = (it.qt_first + i) * p.T + qrow_tok;
        if (tok < p.N) {
          float* dst =
              p.dq_acc + ((static_cast<size_t>(it.b) * p.N + tok) * p.Hq + qrow_head) * DH + w * (DH / 2);
#pragma unroll
          for (int c = 0; c < DH / 2; c += 4)
            atomicAdd(reinterpret_cast<float4*>(dst + c), make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]));
        }
      };

      for (int i = 0; i < it.nq; ++i) {
        const int G = gt + i, s = G % QS, qt = it.qt_first + i;
        ok = __all_sync(0xffffffffu, mbar_wait(qd_full(s), (G / QS) & 1, abort_flag, kSiteSoftmax));
        if (!ok) break;
        const bool masked = p.causal && (it.k0 + NK - 1 > qt * p.T);
        // P is zeroed where lim > rtok[row]: keys past N always, keys after the
        // row's token on the causal diagonal.
        const int lim = !key_ok ? 0x7fffffff : (masked ? key - qt * p.T : -0x7fffffff);
        uint8_t* ds_smem = smem + Tr::OFF_DS + (G & 1) * Tr::DS_BYTES;
        // dS (bf16) for the dQ MMA goes to this buffer, which the dQ of tile G - 2 read.
        if (G >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(dq_full(G & 1), ((G >> 1) - 1) & 1, abort_flag, kSiteSoftmax));
          if (!ok) break;
        }
        {
          // This warpgroup's half of the tile: query columns col0 .. col0 + 63.
          const int H = 2 * G + w, x = H % NBUF;
          const int col0 = 64 * w;
          ok = __all_sync(0xffffffffu, mbar_wait(s_full(x), (H / NBUF) & 1, abort_flag, kSiteSoftmax));
          if (!ok) break;
          tc_fence_after();
          const float* nl2 = reinterpret_cast<const float*>(smem + Tr::OFF_STAT + s * 1024) + col0;
          const uint32_t tS = lane_addr + Tr::tm_st(x), tP = lane_addr + Tr::tm_dpt(x);
          // Four chunks of 16 columns; the next chunk's TMEM load is in flight
          // while one chunk is computed.
          uint32_t ca[32], cb[32];  // [0,16): S^T, [16,32): dP^T
          tmem_ld16x2(tS, tP, ca);
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            uint32_t(&cur)[32] = (c16 & 1) ? cb : ca;
            uint32_t(&nxt)[32] = (c16 & 1) ? ca : cb;
            if (c16 + 1 < 4) tmem_ld16x2_nowait(tS + 16 * (c16 + 1), tP + 16 * (c16 + 1), nxt);
            // The mask test runs on every tile (lim makes it a no-op off the
            // diagonal): cheaper than branching between two versions.
            uint32_t pt[16], dst[16], dsb[8];
            bwd_p_ds16(cur, nl2 + 16 * c16, nl2 + 128 + 16 * c16, rtok + col0 + 16 * c16, lim, sl2, pt, dst, dsb);
            tmem_st16x2(tS + 16 * c16, tP + 16 * c16, pt, dst);
            // dS[q][key] for q = col0 + 16 c16 .. + 15 into the MN-major 128B-swizzled
            // tile: panel q / 64, key row kk (128 bytes), 16-byte chunk (q % 64) / 8.
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              const int q = col0 + 16 * c16 + 8 * ch;
              const int panel = q >> 6, chunk = (q & 63) >> 3;
              *reinterpret_cast<uint4*>(ds_smem + panel * 16384 + kk * 128 + ((chunk ^ (kk & 7)) << 4)) =
                  make_uint4(dsb[4 * ch], dsb[4 * ch + 1], dsb[4 * ch + 2], dsb[4 * ch + 3]);
            }
            if (c16 + 1 < 4) tmem_wait_ld32(nxt);
          }
          tmem_wait_st();
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(ds_ready(x));
        }
        if (!ok) break;
        // dsq_ready(w) is signalled only after the dQ of tile G - 1 completed,
        // which keeps it at most one phase ahead of issuer A's wait.
        if (G > 0) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(dq_full((G - 1) & 1), ((G - 1) >> 1) & 1, abort_flag, kSiteSoftmax));
          if (!ok) break;
        }
        mbar_arrive(dsq_ready(w));
        if (i > 0) {
          tc_fence_after();
          dq_epilogue(i - 1);
        }
      }
      if (!ok) break;
      {
        const int G = gt + it.nq - 1;
        ok = __all_sync(0xffffffffu, mbar_wait(dq_full(G & 1), (G >> 1) & 1, abort_flag, kSiteEpilogue));
        if (!ok) break;
        tc_fence_after();
        dq_epilogue(it.nq - 1);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(dkv_final, r & 1, abort_flag, kSiteEpilogue));
      if (!ok) break;
      tc_fence_after();
      float dv[DH / 2], dk[DH / 2];
      tmem_ld_half<DH>(lane_addr + Tr::TM_DV + w * (DH / 2), dv);
      tmem_ld_half<DH>(lane_addr + Tr::TM_DK + w * (DH / 2), dk);
      tc_fence_before();
      mbar_arrive(dkv_free);
      if (key_ok) {
        const size_t off = ((static_cast<size_t>(it.b) * p.N + key) * p.Hkv + it.kvh) * DH + w * (DH / 2);
        const float sc = p.scale;
#pragma unroll
        for (int c = 0; c < DH / 2; c += 8) {
          uint4 o;
          o.x = pack_bf16x2(dv[c], dv[c + 1]);
          o.y = pack_bf16x2(dv[c + 2], dv[c + 3]);
          o.z = pack_bf16x2(dv[c + 4], dv[c + 5]);
          o.w = pack_bf16x2(dv[c + 6], dv[c + 7]);
          *reinterpret_cast<uint4*>(p.dv + off + c) = o;
          o.x = pack_bf16x2(dk[c] * sc, dk[c + 1] * sc);
          o.y = pack_bf16x2(dk[c + 2] * sc, dk[c + 3] * sc);
          o.z = pack_bf16x2(dk[c + 4] * sc, dk[c + 5] * sc);
          o.w = pack_bf16x2(dk[c + 6] * sc, dk[c + 7] * sc);
          *reinterpret_cast<uint4*>(p.dk + off + c) = o;
        }
      }
      gt += it.nq;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Tr::WARP_MMA_A) tmem_dealloc(tmem, 512);
}

}  // namespace sqa

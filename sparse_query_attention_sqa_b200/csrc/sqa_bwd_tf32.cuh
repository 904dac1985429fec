// sqa_bwd_tf32.cuh -- Sparse Query Attention backward, main kernel for head
// dims 16 and 32 (the SQAT-m shapes).
//
// Same decomposition as sqa_bwd_kernel (one CTA per 128-key tile, batch and KV
// head; stacked Q tiles of the g query heads of the group, so dK and dV are
// reduced over the group inside the tensor-core accumulation), with two
// differences:
//
//  * The three gradient contractions dV += P^T dO, dK += dS^T Q and dQ = dS K
//    run as tf32 MMAs with every operand K-major (tf32 operands stored
//    MN-major produced zeros on this hardware).  P^T and dS^T stay in fp32 in
//    TMEM (in place); two converter warps write transposed fp32 copies of the
//    Q, dO and K tiles ([dh][128 rows], rows contiguous); dS goes to shared
//    memory as [query][key].  dS is rounded to tf32 (round to nearest); P is
//    passed as is.  This
//    keeps bf16's exponent range and three more mantissa bits than bf16
//    operands, which matters when large query groups sum many terms into one
//    dK or dV row.  S^T = K Q^T and dP^T = V dO^T stay bf16 (exact products).
//
//  * The 128-row Q tile is processed as two 64-column halves in two TMEM
//    buffers, so the tensor core computes S^T and dP^T of the next half while
//    the softmax warps turn the current half into P^T and dS^T.
//
// Roles (384 threads):
//   warps 0-7   P^T / dS^T: warpgroup w takes 32 of the 64 columns of a half;
//               also the dQ epilogue (fp32 atomics) and the dK / dV epilogue
//   warp 8      TMA producer (K, V once; Q, dO, lse2, D per Q tile)
//   warp 9      TMEM allocator and MMA issuer (one thread)
//   warps 10-11 bf16 -> fp32 conversion of K (once) and Q, dO (per Q tile)
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
__device__ __forceinline__ void fsub2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fmul2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
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
  static constexpr int ROWB = DH * 2;     // bf16 row bytes (one swizzle panel)
  static constexpr int ROWB32 = DH * 4;   // fp32 row bytes
  static constexpr uint32_t LAYOUT = ROWB == 32 ? 6u : 4u;     // bf16 tiles: SW32 / SW64
  // fp32 tiles are transposed, [dh][128] K-major with a 128-byte swizzle: four
  // panels of 32 values, each panel dh rows of 128 bytes.
  static constexpr int PANEL32 = DH * 128;
  static constexpr int TILE = 128 * DH * 2;
  static constexpr int TILE32 = 128 * DH * 4;
  static constexpr int QS = 2;
  static constexpr int DS_BYTES = 128 * 128 * 4;  // fp32 dS [query][key], K-major, four 32-key panels
  static constexpr int OFF_DS = 0;
  static constexpr int OFF_K = OFF_DS + DS_BYTES;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_K32 = OFF_V + TILE;
  static constexpr int OFF_Q = OFF_K32 + TILE32;
  static constexpr int OFF_DO = OFF_Q + QS * TILE;
  static constexpr int OFF_Q32 = OFF_DO + QS * TILE;
  static constexpr int OFF_DO32 = OFF_Q32 + QS * TILE32;
  static constexpr int OFF_STAT = OFF_DO32 + QS * TILE32;  // per stage: lse2[128], D[128]
  static constexpr int OFF_RTOK = OFF_STAT + QS * 1024;
  static constexpr int OFF_BAR = OFF_RTOK + 512;
  // kv_full, cvt_k, qd_full[2], qd_empty[2], cvt_full[2], s_full[2], ds_ready[2], dq_full, dq_empty[2],
  // dkv_final, drain
  static constexpr int N_BARS = 18;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16 + 1024;
  static constexpr uint32_t TM_DV = 256, TM_DK = 320;
  __host__ __device__ static constexpr uint32_t tm_st(int b) { return 128u * b; }
  __host__ __device__ static constexpr uint32_t tm_dpt(int b) { return 128u * b + 64u; }
  __host__ __device__ static constexpr uint32_t tm_dq(int i) { return 384u + 64u * (i & 1); }
  static constexpr int THREADS = 384;
  static constexpr int WARP_PRODUCER = 8, WARP_MMA = 9, WARP_CVT0 = 10;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Convert a bf16 tile [128 rows][dh] (rows of 2*dh bytes, swizzled as loaded by
// TMA) into the transposed fp32 tile [dh][128] in K-major 128-byte-swizzled
// panels of 32 rows, with 64 threads.  A warp writes one 128-byte row segment
// per store instruction.
template <int DH>
__device__ __forceinline__ void convert_tile_t(const uint8_t* src, uint8_t* dst, int tid64) {
  constexpr int ROWB = DH * 2;
  for (int r = tid64; r < 128; r += 64) {
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
  const int nh = 2 * nq;  // 64-column halves

  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  const uint32_t kv_full = bar0, cvt_k = bar0 + 8;
  auto qd_full = [&](int s) { return bar0 + 8u * (2 + s); };
  auto qd_empty = [&](int s) { return bar0 + 8u * (4 + s); };
  auto cvt_full = [&](int s) { return bar0 + 8u * (6 + s); };
  auto s_full = [&](int bb) { return bar0 + 8u * (8 + bb); };
  auto ds_ready = [&](int bb) { return bar0 + 8u * (10 + bb); };
  const uint32_t dq_full = bar0 + 8u * 12;
  auto dq_empty = [&](int x) { return bar0 + 8u * (13 + x); };
  const uint32_t dkv_final = bar0 + 8u * 15, drain = bar0 + 8u * 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* rtok = reinterpret_cast<int*>(smem + Tr::OFF_RTOK);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(cvt_k, 64);
    for (int s = 0; s < QS; ++s) {
      mbar_init(qd_full(s), 1);
      mbar_init(qd_empty(s), 1);
      mbar_init(cvt_full(s), 64);
    }
    for (int bb = 0; bb < 2; ++bb) {
      mbar_init(s_full(bb), 1);
      mbar_init(ds_ready(bb), 256);
      mbar_init(dq_empty(bb), 256);
    }
    mbar_init(dq_full, 1);
    mbar_init(dkv_final, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 128) rtok[threadIdx.x] = threadIdx.x < p.rows ? threadIdx.x / p.g : (1 << 30);
  if (p.rows < BM) {  // stacked rows the TMA box does not cover stay zero (the fp32 copies follow)
    for (int s = 0; s < QS; ++s) {
      for (int which = 0; which < 2; ++which) {
        uint8_t* base = smem + (which ? Tr::OFF_DO : Tr::OFF_Q) + s * Tr::TILE + p.rows * ROWB;
        for (int i = threadIdx.x * 16; i < (BM - p.rows) * ROWB; i += Tr::THREADS * 16)
          *reinterpret_cast<uint4*>(base + i) = make_uint4(0, 0, 0, 0);
      }
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
  } else if (warp >= Tr::WARP_CVT0) {
    // ------------------------------------------------------------ bf16 -> fp32 converters
    const int tid64 = threadIdx.x - 32 * Tr::WARP_CVT0;
    bool ok = mbar_wait(kv_full, 0, abort_flag, kSiteEpilogue);
    if (ok) {
      convert_tile_t<DH>(smem + Tr::OFF_K, smem + Tr::OFF_K32, tid64);
      fence_async_smem();
      mbar_arrive(cvt_k);
    }
    for (int i = 0; ok && i < nq; ++i) {
      const int s = i % QS;
      // The producer refills stage s only after the MMAs of the tile that used
      // it last have completed, so the fp32 copies of that tile are free too.
      if (!mbar_wait(qd_full(s), (i / QS) & 1, abort_flag, kSiteEpilogue)) break;
      convert_tile_t<DH>(smem + Tr::OFF_Q + s * Tr::TILE, smem + Tr::OFF_Q32 + s * Tr::TILE32, tid64);
      convert_tile_t<DH>(smem + Tr::OFF_DO + s * Tr::TILE, smem + Tr::OFF_DO32 + s * Tr::TILE32, tid64);
      fence_async_smem();
      mbar_arrive(cvt_full(s));
    }
  } else if (warp == Tr::WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);  // S^T, dP^T halves
      constexpr uint32_t idesc_g = idesc_tf32_f32(128, DH, false, false);  // dV, dK (A in TMEM)
      constexpr uint32_t idesc_q = idesc_tf32_f32(128, DH, false, false);  // dQ (A = dS from smem)
      const uint32_t k_addr = sbase + Tr::OFF_K, v_addr = sbase + Tr::OFF_V, k32 = sbase + Tr::OFF_K32;
      const uint32_t ds_addr = sbase + Tr::OFF_DS;
      // S^T and dP^T for half h into TMEM buffer h % 2.
      auto issue_s = [&](int h) {
        const int s = (h >> 1) % QS, hh = h & 1;
        const uint32_t rows = hh * 64;
        const uint32_t q_addr = sbase + Tr::OFF_Q + s * Tr::TILE + rows * ROWB;
        const uint32_t do_addr = sbase + Tr::OFF_DO + s * Tr::TILE + rows * ROWB;
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          const uint32_t off = ks * 32;
          mma_ss(tmem + Tr::tm_st(h & 1), smem_desc(k_addr + off, 16, 8 * ROWB, Tr::LAYOUT),
                 smem_desc(q_addr + off, 16, 8 * ROWB, Tr::LAYOUT), idesc_s, ks > 0);
          mma_ss(tmem + Tr::tm_dpt(h & 1), smem_desc(v_addr + off, 16, 8 * ROWB, Tr::LAYOUT),
                 smem_desc(do_addr + off, 16, 8 * ROWB, Tr::LAYOUT), idesc_s, ks > 0);
        }
        mma_commit(s_full(h & 1));
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag, kSiteMma) && mbar_wait(qd_full(0), 0, abort_flag, kSiteMma) &&
                mbar_wait(cvt_k, 0, abort_flag, kSiteMma);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_s(1);
      }
      for (int h = 0; ok && h < nh; ++h) {
        const int i = h >> 1, hh = h & 1, s = i % QS;
        if (!mbar_wait(ds_ready(h & 1), (h >> 1) & 1, abort_flag, kSiteMma)) { ok = false; break; }
        if (hh == 0 && !mbar_wait(cvt_full(s), (i / QS) & 1, abort_flag, kSiteMma)) { ok = false; break; }
        tc_fence_after();
        // dV += P^T dO and dK += dS^T Q over the 64 query rows of this half (K = 8 per
        // tf32 MMA).  B = the transposed fp32 tile: query rows q0..q0+7 are 32 bytes
        // at offset (q0 % 32) * 4 of panel q0 / 32.
        const uint32_t do32 = sbase + Tr::OFF_DO32 + s * Tr::TILE32;
        const uint32_t q32 = sbase + Tr::OFF_Q32 + s * Tr::TILE32;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t acc = (h > 0 || ks > 0) ? 1u : 0u;
          const int q0 = hh * 64 + ks * 8;
          const uint32_t boff = (q0 >> 5) * Tr::PANEL32 + (q0 & 31) * 4;
          mma_ts_tf32(tmem + Tr::TM_DV, tmem + Tr::tm_st(h & 1) + 8 * ks, smem_desc(do32 + boff, 16, 1024, 2u),
                      idesc_g, acc);
          mma_ts_tf32(tmem + Tr::TM_DK, tmem + Tr::tm_dpt(h & 1) + 8 * ks, smem_desc(q32 + boff, 16, 1024, 2u),
                      idesc_g, acc);
        }
        if (hh == 1) {
          // dQ of Q tile i = dS K (M = 128 query rows, K = 128 keys, 8 per MMA).
          if (i >= 2 && !mbar_wait(dq_empty(i & 1), ((i >> 1) - 1) & 1, abort_flag, kSiteMma)) { ok = false; break; }
          tc_fence_after();
          // A = dS [query][key] (panels of 32 keys, 16 KB apart), B = K^T [dh][key].
#pragma unroll
          for (int ks = 0; ks < NK / 8; ++ks)
            mma_ss_tf32(tmem + Tr::tm_dq(i), smem_desc(ds_addr + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2u),
                        smem_desc(k32 + (ks >> 2) * Tr::PANEL32 + (ks & 3) * 32, 16, 1024, 2u), idesc_q, ks > 0);
          mma_commit(dq_full);
          mma_commit(qd_empty(s));
        }
        if (h + 2 < nh) {
          // The next half that uses this TMEM buffer; the MMAs above read it first.
          if (hh == 0) {
            const int i2 = i + 1;
            if (!mbar_wait(qd_full(i2 % QS), (i2 / QS) & 1, abort_flag, kSiteMma)) { ok = false; break; }
            tc_fence_after();
          }
          issue_s(h + 2);
        }
      }
      if (ok) mma_commit(dkv_final);
      else {
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T, dQ and dK/dV epilogues
    const int w = warp >> 2;                  // which 32 of the 64 columns of a half
    const int kk = (warp & 3) * 32 + lane;    // TMEM lane: key (S^T, dP^T, dK, dV) or query row (dQ)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = k0 + kk;
    const bool key_ok = key < p.N;
    const float sl2 = p.scale_log2;
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

    for (int h = 0; h < nh; ++h) {
      const int i = h >> 1, hh = h & 1, s = i % QS, qt = qt_first + i;
      ok = __all_sync(0xffffffffu, mbar_wait(qd_full(s), (i / QS) & 1, abort_flag, kSiteSoftmax) &&
                                       mbar_wait(s_full(h & 1), (h >> 1) & 1, abort_flag, kSiteSoftmax));
      if (!ok) break;
      tc_fence_after();
      const int col0 = hh * 64 + w * 32;  // first query row (of the 128-row tile) of this thread's columns
      const float* lse2 = reinterpret_cast<const float*>(smem + Tr::OFF_STAT + s * 1024) + col0;
      const float* Dv = lse2 + 128;
      const bool masked = p.causal && (k0 + NK - 1 > qt * p.T);
      const int key_rel = key - qt * p.T;  // visible iff key_rel <= rtok[r]
      uint32_t sr[64];  // [0,32): S^T, [32,64): dP^T
      tmem_ld32x2(lane_addr + Tr::tm_st(h & 1) + w * 32, lane_addr + Tr::tm_dpt(h & 1) + w * 32, sr);
      uint32_t pt[32], dst[32];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse2 + e);
        const float4 d4 = *reinterpret_cast<const float4*>(Dv + e);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int u = 0; u < 4; u += 2) {
          float x0, x1;
          ffma2(x0, x1, __uint_as_float(sr[e + u]), __uint_as_float(sr[e + u + 1]), sl2, sl2, -lv[u], -lv[u + 1]);
          float p0 = ex2(x0), p1 = ex2(x1);
          if (!key_ok) p0 = p1 = 0.f;
          if (masked) {
            if (key_rel > rtok[col0 + e + u]) p0 = 0.f;
            if (key_rel > rtok[col0 + e + u + 1]) p1 = 0.f;
          }
          float t0, t1, d0, d1;
          fsub2(t0, t1, __uint_as_float(sr[32 + e + u]), __uint_as_float(sr[32 + e + u + 1]), dv[u], dv[u + 1]);
          fmul2(d0, d1, p0, p1, t0, t1);
          pt[e + u] = __float_as_uint(p0);
          pt[e + u + 1] = __float_as_uint(p1);
          dst[e + u] = round_tf32(d0);
          dst[e + u + 1] = round_tf32(d1);
        }
      }
      tmem_st32(lane_addr + Tr::tm_st(h & 1) + w * 32, pt);
      tmem_st32(lane_addr + Tr::tm_dpt(h & 1) + w * 32, dst);
      // dS (fp32) for the dQ MMA: the dQ of the previous Q tile read this buffer,
      // so wait for it at the first half of a tile (at most one phase behind).
      if (hh == 0 && i > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(dq_full, (i - 1) & 1, abort_flag, kSiteSoftmax));
        if (!ok) break;
      }
      // dS[q][key]: key kk is word kk % 4 of chunk (kk % 32) / 4 of row q in panel kk / 32;
      // the 32 lanes of a warp fill one 128-byte row segment per store.
      {
        uint8_t* base = ds_smem + (kk >> 5) * 16384 + (kk & 3) * 4;
        const int chunk = (kk & 31) >> 2;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int q = col0 + e;
          *reinterpret_cast<uint32_t*>(base + q * 128 + ((chunk ^ (q & 7)) << 4)) = dst[e];
        }
      }
      tmem_wait_st();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ds_ready(h & 1));
      if (hh == 0 && i > 0) {
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
  if (warp == Tr::WARP_MMA) tmem_dealloc(tmem, 512);
}

}  // namespace sqa

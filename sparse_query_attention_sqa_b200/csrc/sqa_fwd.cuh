// sqa_fwd.cuh -- Sparse Query Attention forward on sm_100a.
//
// One CTA owns one key/value head of one batch entry and two Q tiles.  A Q tile
// stacks the g = H_q / H_kv query heads that share the key/value head: its 128
// MMA rows are (token, head) pairs, row r = t * g + head, which is exactly how
// [B][N][H_q][dh] stores the group's heads side by side, so one TMA box
// {dh, g, T} fills it.  Every K/V tile is therefore loaded once per KV head and
// used by all heads of its group (GQA summary, "The idea": a group shares one key
// head and one value head; arXiv 2510.01817 abstract: score FLOPs scale with H_q).
//
// Roles (384 threads):
//   warp 0      TMA producer: Q tiles once, then K/V tiles through a ring of stages
//   warp 1      TMEM allocator and MMA issuer (one thread):
//                 S_t = Q_t K_j^T  (tcgen05, both operands K-major in smem)
//                 O_t += P_t V_j   (tcgen05, P from TMEM, V MN-major in smem)
//   warps 4-7   softmax for Q tile 0; warps 8-11 softmax for Q tile 1
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+dh), O_1 [384,384+dh).
// P_t (bf16) overwrites the first half of S_t's columns in place.
//
// Online softmax (exact): each row keeps a reference maximum m (log2 units) and
// l = sum 2^(s*scale*log2e - m).  m is raised only when a tile's maximum exceeds
// it by more than 8, so P <= 256 and O is rescaled rarely; the final O / l and
// lse = ln2 * (m + log2 l) do not depend on which reference was used.
#pragma once

#include "sqa_device.cuh"

namespace sqa {

struct FwdParams {
  __nv_bfloat16* out;
  float* lse;
  int N, Hq, Hkv, g;
  int T;         // tokens per Q tile
  int rows;      // T * g stacked rows per Q tile (<= 128)
  int n_qtiles;  // ceil(N / T) per (batch, kv head)
  int n_pairs;   // ceil(n_qtiles / 2)
  int n_bh;      // B * Hkv
  int causal;
  float scale_log2;  // scale * log2(e)
};

template <int DH>
struct FwdTraits {
  static constexpr int BM = 128;  // stacked rows per Q tile
  static constexpr int NK = 128;  // keys per K/V tile
  static constexpr int PANEL = DH < 64 ? DH : 64;  // elements per swizzled row segment
  static constexpr int NPANEL = DH / PANEL;
  static constexpr int ROWB = PANEL * 2;  // bytes per row segment
  static constexpr uint32_t LAYOUT = ROWB == 32 ? 6u : (ROWB == 64 ? 4u : 2u);
  static constexpr int Q_BYTES = BM * DH * 2;
  static constexpr int KV_BYTES = NK * DH * 2;
  static constexpr int STAGES = DH <= 32 ? 4 : (DH == 64 ? 3 : 2);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
  static constexpr int N_BARS = 1 + 2 * STAGES + 6 + 1;
  static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
  // Ask for enough shared memory that only one CTA fits per SM (each CTA holds
  // all 512 TMEM columns), plus slack to align the base to 1024 bytes.
  static constexpr int SMEM_BYTES = (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) + 1024;
  // TMEM column of S_t and O_t
  __host__ __device__ static constexpr uint32_t tm_s(int t) { return t ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t tm_o(int t) { return t ? 384u : 256u; }
  static constexpr int THREADS = 384;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(DH % 16 == 0 && DH <= 128, "head dim");
};

template <int DH>
__global__ void __launch_bounds__(384, 1)
    sqa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using Tr = FwdTraits<DH>;
  using namespace dev;
  constexpr int BM = Tr::BM, NK = Tr::NK, ROWB = Tr::ROWB, PANEL = Tr::PANEL;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Heaviest Q-tile pairs (the latest tokens, under a causal mask) go first.
  const int pair = p.n_pairs - 1 - static_cast<int>(blockIdx.x / p.n_bh);
  const int bh = blockIdx.x % p.n_bh;
  const int b = bh / p.Hkv, kvh = bh % p.Hkv;
  const int qt0 = 2 * pair;
  const bool has1 = qt0 + 1 < p.n_qtiles;
  auto kv_tiles = [&](int qt) {
    const int end = p.causal ? min(p.N, (qt + 1) * p.T) : p.N;
    return (end + NK - 1) / NK;
  };
  const int nkv0 = kv_tiles(qt0);
  const int nkv1 = has1 ? kv_tiles(qt0 + 1) : 0;
  const int nkv = max(nkv0, nkv1);

  // Barriers: q_full | kv_full[S] | kv_empty[S] | s_full[2] | p_full[2] | o_final[2] | drain
  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  const uint32_t q_full = bar0;
  auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + Tr::STAGES + s); };
  auto s_full = [&](int t) { return bar0 + 8u * (1 + 2 * Tr::STAGES + t); };
  auto p_full = [&](int t) { return bar0 + 8u * (3 + 2 * Tr::STAGES + t); };
  auto o_final = [&](int t) { return bar0 + 8u * (5 + 2 * Tr::STAGES + t); };
  const uint32_t drain = bar0 + 8u * (7 + 2 * Tr::STAGES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < Tr::STAGES; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 128);
      mbar_init(o_final(t), 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Rows of a Q tile that the TMA box does not cover (when g does not divide
  // 128) stay zero, so their scores are finite; they are never stored.
  if (p.rows < BM) {
    const int pad_bytes = (BM - p.rows) * ROWB;
    for (int t = 0; t < 2; ++t)
      for (int pn = 0; pn < Tr::NPANEL; ++pn) {
        uint8_t* base = smem + Tr::OFF_Q + t * Tr::Q_BYTES + pn * BM * ROWB + p.rows * ROWB;
        for (int i = threadIdx.x * 16; i < pad_bytes; i += Tr::THREADS * 16)
          *reinterpret_cast<uint4*>(base + i) = make_uint4(0, 0, 0, 0);
      }
    fence_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      const uint32_t q_bytes = static_cast<uint32_t>(p.rows * ROWB * Tr::NPANEL);
      mbar_expect_tx(q_full, q_bytes * (has1 ? 2u : 1u));
      for (int t = 0; t < (has1 ? 2 : 1); ++t)
        for (int pn = 0; pn < Tr::NPANEL; ++pn)
          tma_load_4d(sbase + Tr::OFF_Q + t * Tr::Q_BYTES + pn * BM * ROWB, &tmQ, q_full, pn * PANEL,
                      kvh * p.g, (qt0 + t) * p.T, b);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % Tr::STAGES;
        if (j >= Tr::STAGES &&
            !mbar_wait(kv_empty(s), ((j / Tr::STAGES) - 1) & 1, abort_flag, kSiteProducer))
          break;
        mbar_expect_tx(kv_full(s), 2u * Tr::KV_BYTES);
        for (int pn = 0; pn < Tr::NPANEL; ++pn) {
          tma_load_4d(sbase + Tr::OFF_K + s * Tr::KV_BYTES + pn * NK * ROWB, &tmK, kv_full(s),
                      pn * PANEL, kvh, j * NK, b);
          tma_load_4d(sbase + Tr::OFF_V + s * Tr::KV_BYTES + pn * NK * ROWB, &tmV, kv_full(s),
                      pn * PANEL, kvh, j * NK, b);
        }
        issued = j + 1;
      }
      if (*abort_flag) {  // let in-flight copies land before the CTA exits
        mbar_wait_drain(q_full, 0);
        for (int j = max(0, issued - Tr::STAGES); j < issued; ++j)
          mbar_wait_drain(kv_full(j % Tr::STAGES), (j / Tr::STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, NK, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, DH, false, true);
      const uint32_t q_addr = sbase + Tr::OFF_Q, k_addr = sbase + Tr::OFF_K, v_addr = sbase + Tr::OFF_V;
      auto issue_qk = [&](int t, int s) {
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          const uint32_t pn = (ks * 16) / PANEL, off = ((ks * 16) % PANEL) * 2;
          const uint64_t a = smem_desc(q_addr + t * Tr::Q_BYTES + pn * BM * ROWB + off, 16, 8 * ROWB,
                                       Tr::LAYOUT);
          const uint64_t bd = smem_desc(k_addr + s * Tr::KV_BYTES + pn * NK * ROWB + off, 16, 8 * ROWB,
                                        Tr::LAYOUT);
          mma_ss(tmem + Tr::tm_s(t), a, bd, idesc_qk, ks > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int s, bool acc) {
#pragma unroll
        for (int ks = 0; ks < NK / 16; ++ks) {
          const uint64_t bd = smem_desc(v_addr + s * Tr::KV_BYTES + ks * 16 * ROWB, NK * ROWB, 8 * ROWB,
                                        Tr::LAYOUT);
          mma_ts(tmem + Tr::tm_o(t), tmem + Tr::tm_s(t) + ks * 8, bd, idesc_pv,
                 (acc || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, kSiteMma) &&
                mbar_wait(kv_full(0), 0, abort_flag, kSiteMma);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit(s_full(0));
        if (has1) {
          issue_qk(1, 0);
          mma_commit(s_full(1));
        }
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j % Tr::STAGES, sn = (j + 1) % Tr::STAGES;
        bool next_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {
          const int nkv_t = t ? nkv1 : nkv0;
          if (j >= nkv_t) continue;
          if (!mbar_wait(p_full(t), j & 1, abort_flag, kSiteMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(t, s, j > 0);
          if (j + 1 < nkv_t) {
            if (!next_ready) {
              if (!mbar_wait(kv_full(sn), ((j + 1) / Tr::STAGES) & 1, abort_flag, kSiteMma)) {
                ok = false;
                break;
              }
              tc_fence_after();
              next_ready = true;
            }
            issue_qk(t, sn);
            mma_commit(s_full(t));
          } else {
            mma_commit(o_final(t));
          }
        }
        mma_commit(kv_empty(s));
      }
      if (!ok) {  // wait for issued MMAs before TMEM is released
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int nkv_t = t ? nkv1 : nkv0;
    const int qt = qt0 + t;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t tS = lane_addr + Tr::tm_s(t), tO = lane_addr + Tr::tm_o(t);
    const int tok = qt * p.T + row / p.g;
    const int head = kvh * p.g + row % p.g;
    const bool row_valid = row < p.rows && tok < p.N;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = nkv_t > 0;
    for (int j = 0; ok && j < nkv_t; ++j) {
      // Every lane waits; the verdict is made warp-uniform so that the
      // warp-wide TMEM instructions below are never reached divergently.
      ok = __all_sync(0xffffffffu, mbar_wait(s_full(t), j & 1, abort_flag, kSiteSoftmax));
      if (!ok) break;
      tc_fence_after();
      const int k0 = j * NK;
      const bool masked = (k0 + NK > p.N) || (p.causal && k0 + NK - 1 > qt * p.T);
      // last visible key of this tile, relative to k0 (may be negative)
      const int last = masked ? min(p.N - 1, p.causal ? tok : p.N - 1) - k0 : NK - 1;
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < NK / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + c * 32, r);
        if (masked) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i <= last) mx = fmaxf(mx, __uint_as_float(r[i]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(r[i]));
        }
      }
      const float mnew = fmaxf(m, mx * sl2);
      const bool raise = mnew > m + 8.f;
      const float alpha = (raise && m != -INFINITY) ? ex2(m - mnew) : 1.f;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        // O holds P*V of the earlier tiles: the MMA that wrote it completed
        // before s_full fired for this tile.  Lanes that keep their reference
        // multiply by 1.
#pragma unroll 1
        for (int c = 0; c < DH; c += 16) {
          uint32_t r[16];
          tmem_ld16(tO + c, r);
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st16(tO + c, r);
        }
      }
      l *= alpha;
      if (raise) m = mnew;
      const float mref = m == -INFINITY ? 0.f : m;
#pragma unroll 1
      for (int c = 0; c < NK / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + c * 32, r);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float p0 = ex2(fmaf(__uint_as_float(r[i]), sl2, -mref));
          float p1 = ex2(fmaf(__uint_as_float(r[i + 1]), sl2, -mref));
          if (masked) {
            if (c * 32 + i > last) p0 = 0.f;
            if (c * 32 + i + 1 > last) p1 = 0.f;
          }
          l += p0 + p1;
          pk[i >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + c * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(t));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_final(t), 0, abort_flag, kSiteEpilogue));
    if (ok) {
      tc_fence_after();
      const float inv_l = row_valid ? 1.f / l : 0.f;
      __nv_bfloat16* dst = p.out + ((static_cast<size_t>(b) * p.N + (row_valid ? tok : 0)) * p.Hq + head) * DH;
#pragma unroll 1
      for (int c = 0; c < DH; c += 16) {
        uint32_t r[16];
        tmem_ld16(tO + c, r);  // warp-wide: every lane loads, only valid rows store
        uint4 lo, hi;
        lo.x = pack_bf16x2(__uint_as_float(r[0]) * inv_l, __uint_as_float(r[1]) * inv_l);
        lo.y = pack_bf16x2(__uint_as_float(r[2]) * inv_l, __uint_as_float(r[3]) * inv_l);
        lo.z = pack_bf16x2(__uint_as_float(r[4]) * inv_l, __uint_as_float(r[5]) * inv_l);
        lo.w = pack_bf16x2(__uint_as_float(r[6]) * inv_l, __uint_as_float(r[7]) * inv_l);
        hi.x = pack_bf16x2(__uint_as_float(r[8]) * inv_l, __uint_as_float(r[9]) * inv_l);
        hi.y = pack_bf16x2(__uint_as_float(r[10]) * inv_l, __uint_as_float(r[11]) * inv_l);
        hi.z = pack_bf16x2(__uint_as_float(r[12]) * inv_l, __uint_as_float(r[13]) * inv_l);
        hi.w = pack_bf16x2(__uint_as_float(r[14]) * inv_l, __uint_as_float(r[15]) * inv_l);
        if (row_valid) {
          *reinterpret_cast<uint4*>(dst + c) = lo;
          *reinterpret_cast<uint4*>(dst + c + 8) = hi;
        }
      }
      if (row_valid)
        p.lse[(static_cast<size_t>(b) * p.Hq + head) * p.N + tok] = (m + __log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace sqa

// sqa_bwd.cuh -- Sparse Query Attention backward on sm_100a.
//
// Three launches on the caller's stream:
//   1. prep:  -D_i = -<dO_i, O_i> and -lse_i * log2(e) for every query row,
//             written in the stacked-tile order the main kernel reads (slots of
//             padding rows get lse = +inf and D = 0, which makes their P exactly
//             0), the fp32 dQ accumulator zeroed, and for dh <= 32 transposed
//             fp32 images of the Q and dO tiles (tf32 MMA operands).
//   2. main:  one CTA per (128-key tile, batch, KV head).  It keeps K and V in
//             shared memory and walks the Q tiles that see its keys.  A Q tile
//             stacks the g query heads of the group (row r = t * g + head), so
//             the dK and dV MMAs contract over tokens and heads at once: the
//             reduction over the query-head group happens inside the tensor core
//             accumulation in TMEM.  Per Q tile:
//               S^T  = K Q^T,  dP^T = V dO^T            (TMEM, keys on lanes)
//               P^T  = 2^(S^T scale log2e - lse2),  dS^T = P^T (dP^T - D)
//               dV  += P^T dO,  dK += dS^T Q            (A operands from TMEM)
//               dQ   = dS K                             (A = dS from shared memory)
//             and dQ is added to the fp32 accumulator with vector atomics.
//   3. dq:    dQ = scale * accumulator, rounded to bf16.
// The formulas are those of the gradient of L = sum dO * O through
// softmax(scale Q K^T) V with query head h reading KV head floor(h / g).
#pragma once

#include <string>

#include "sqa.h"
#include "sqa_device.cuh"

namespace sqa {

constexpr int kBwdTile = 128;  // keys per CTA and stacked query rows per Q tile

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdLayout {
  int g, T, rows, n_qt, n_kt;
  size_t n_slots;     // B * H_kv * n_qt * 128
  size_t off_D;       // byte offsets inside the workspace
  size_t off_dq;
  size_t off_q32;     // dh <= 32 only: fp32 transposed images of the stacked Q and dO tiles
  size_t off_do32;
  size_t bytes;
};

inline BwdLayout bwd_layout(int B, int N, int Hq, int Hkv, int dh) {
  BwdLayout L{};
  L.g = Hq / Hkv;
  L.T = kBwdTile / L.g;
  L.rows = L.T * L.g;
  L.n_qt = (N + L.T - 1) / L.T;
  L.n_kt = (N + kBwdTile - 1) / kBwdTile;
  L.n_slots = static_cast<size_t>(B) * Hkv * L.n_qt * kBwdTile;
  L.off_D = align256(L.n_slots * sizeof(float));
  L.off_dq = L.off_D + align256(L.n_slots * sizeof(float));
  L.bytes = L.off_dq + align256(static_cast<size_t>(B) * N * Hq * dh * sizeof(float));
  if (dh <= 32) {
    const size_t img = align256(L.n_slots * dh * sizeof(float));
    L.off_q32 = L.bytes;
    L.off_do32 = L.bytes + img;
    L.bytes += 2 * img;
  }
  return L;
}

inline size_t bwd_workspace_bytes(int B, int N, int Hq, int Hkv, int dh) {
  return bwd_layout(B, N, Hq, Hkv, dh).bytes;
}

// ---------------------------------------------------------------------------
// 1. prep
struct BwdPrepParams {
  const __nv_bfloat16* dout;
  const __nv_bfloat16* out;
  const __nv_bfloat16* q;
  const float* lse;
  float* lse2;
  float* D;
  float* dq_acc;
  float* q32;   // null, or the fp32 tile images (see below)
  float* do32;
  int N, Hq, Hkv, g, T, rows, n_qt;
  long long n_slots;
  long long dq_vec4;  // dq accumulator length / 4
};

// Offset (in floats) of element (row r, column n) inside the fp32 image of one
// stacked 128-row tile: the tile transposed to [dh][128] and cut into four
// panels of 32 rows, each panel dh lines of 128 bytes with the 128-byte swizzle
// (16-byte chunk c of line n stored at chunk c ^ (n % 8)).  This is the K-major
// operand layout of a tf32 MMA whose contraction runs over the tile's rows, so
// the image is copied to shared memory as is.
__host__ __device__ __forceinline__ int tf32_image_index(int r, int n, int dh) {
  return (r >> 5) * dh * 32 + n * 32 + ((((r & 31) >> 2) ^ (n & 7)) << 2) + (r & 3);
}

template <int DH>
__global__ void __launch_bounds__(256) sqa_bwd_prep_kernel(const BwdPrepParams p) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (long long s = tid; s < p.n_slots; s += stride) {
    const int r = static_cast<int>(s % kBwdTile);
    const long long rest = s / kBwdTile;
    const int qt = static_cast<int>(rest % p.n_qt);
    const long long bkv = rest / p.n_qt;
    const int b = static_cast<int>(bkv / p.Hkv), kvh = static_cast<int>(bkv % p.Hkv);
    const int tok = qt * p.T + r / p.g;
    float l2 = INFINITY, d = 0.f;
    const bool live = r < p.rows && tok < p.N;
    float* qi = p.q32 ? p.q32 + (s - r) * DH : nullptr;
    float* di = p.q32 ? p.do32 + (s - r) * DH : nullptr;
    if (live) {
      const int head = kvh * p.g + r % p.g;
      const size_t row = (static_cast<size_t>(b) * p.N + tok) * p.Hq + head;
      const uint4* o = reinterpret_cast<const uint4*>(p.out + row * DH);
      const uint4* go = reinterpret_cast<const uint4*>(p.dout + row * DH);
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) {
        const uint4 a = o[c], bb = go[c];
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fa = __bfloat1622float2(a2[e]), fb = __bfloat1622float2(b2[e]);
          d = fmaf(fa.x, fb.x, d);
          d = fmaf(fa.y, fb.y, d);
          if (DH <= 32 && di) {
            di[tf32_image_index(r, 8 * c + 2 * e, DH)] = fb.x;
            di[tf32_image_index(r, 8 * c + 2 * e + 1, DH)] = fb.y;
          }
        }
      }
      if (DH <= 32 && qi) {
        const uint4* qr = reinterpret_cast<const uint4*>(p.q + row * DH);
#pragma unroll
        for (int c = 0; c < DH / 8; ++c) {
          const uint4 a = qr[c];
          const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fa = __bfloat1622float2(a2[e]);
            qi[tf32_image_index(r, 8 * c + 2 * e, DH)] = fa.x;
            qi[tf32_image_index(r, 8 * c + 2 * e + 1, DH)] = fa.y;
          }
        }
      }
      l2 = p.lse[(static_cast<size_t>(b) * p.Hq + head) * p.N + tok] * 1.4426950408889634f;
    } else if (DH <= 32 && qi) {
#pragma unroll
      for (int n = 0; n < DH; ++n) qi[tf32_image_index(r, n, DH)] = di[tf32_image_index(r, n, DH)] = 0.f;
    }
    // Stored negated: the main kernels add them (x = S * scale * log2(e) - lse2, dP - D).
    p.lse2[s] = -l2;
    p.D[s] = -d;
  }
  float4* acc = reinterpret_cast<float4*>(p.dq_acc);
  for (long long i = tid; i < p.dq_vec4; i += stride) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------
// 3. dq
__global__ void __launch_bounds__(256)
    sqa_bwd_dq_kernel(const float* acc, __nv_bfloat16* dq, long long n_vec8, float scale) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec8; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 c = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 o;
    o.x = dev::pack_bf16x2(a.x * scale, a.y * scale);
    o.y = dev::pack_bf16x2(a.z * scale, a.w * scale);
    o.z = dev::pack_bf16x2(c.x * scale, c.y * scale);
    o.w = dev::pack_bf16x2(c.z * scale, c.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = o;
  }
}

// ---------------------------------------------------------------------------
// 2. main
struct BwdParams {
  const float* lse2;  // stacked [B*H_kv][n_qt][128], negated: -lse * log2(e) (-inf on padding rows)
  const float* D;     // negated: -<dO, O> (0 on padding rows)
  float* dq_acc;      // [B][N][H_q][dh] fp32
  const float* q32;   // dh <= 32: fp32 images of the stacked Q and dO tiles
  const float* do32;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int N, Hq, Hkv, g, T, rows, n_qt, n_bh, causal;
  int n_items;  // persistent kernels: 128-key tiles x (batch, KV head)
  float scale_log2, scale;
};

template <int DH>
struct BwdTraits {
  static constexpr int BM = kBwdTile, NK = kBwdTile;
  static constexpr int PANEL = DH < 64 ? DH : 64;
  static constexpr int NPANEL = DH / PANEL;
  static constexpr int ROWB = PANEL * 2;
  static constexpr uint32_t LAYOUT = ROWB == 32 ? 6u : (ROWB == 64 ? 4u : 2u);
  static constexpr int TILE = 128 * DH * 2;  // one Q, dO, K or V tile
  static constexpr int QS = DH == 128 ? 1 : 2;  // Q/dO stages
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;
  static constexpr int OFF_DO = OFF_Q + QS * TILE;
  static constexpr int OFF_DS = OFF_DO + QS * TILE;
  static constexpr int OFF_STAT = OFF_DS + DS_BYTES;    // per stage: lse2[128], D[128]
  static constexpr int OFF_RTOK = OFF_STAT + QS * 1024;  // 128 ints: row -> token offset
  static constexpr int OFF_BAR = OFF_RTOK + 512;
  static constexpr int N_BARS = 1 + 2 * QS + 6;
  static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
  static constexpr int SMEM_BYTES = (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) + 1024;
  // TMEM columns.  At dh = 128 the dQ accumulator shares S^T's columns.
  static constexpr uint32_t TM_ST = 0, TM_DPT = 128;
  static constexpr uint32_t TM_DQ = DH == 128 ? 0u : 256u;
  static constexpr uint32_t TM_DV = DH == 128 ? 256u : 384u;
  static constexpr uint32_t TM_DK = DH == 128 ? 384u : 448u;
  static constexpr int THREADS = 384;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// dh/2 fp32 columns of this thread's TMEM lane.
template <int DH>
__device__ __forceinline__ void tmem_ld_half(uint32_t taddr, float (&v)[DH / 2]) {
  if constexpr (DH / 2 == 8) {
    uint32_t r[8];
    dev::tmem_ld8(taddr, r);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
  } else {
#pragma unroll
    for (int c = 0; c < DH / 2; c += 16) {
      uint32_t r[16];
      dev::tmem_ld16(taddr + c, r);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[c + i] = __uint_as_float(r[i]);
    }
  }
}

template <int DH>
__global__ void __launch_bounds__(384, 1)
    sqa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const BwdParams p) {
  using Tr = BwdTraits<DH>;
  using namespace dev;
  constexpr int BM = Tr::BM, NK = Tr::NK, ROWB = Tr::ROWB, PANEL = Tr::PANEL, QS = Tr::QS;

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
  auto qd_empty = [&](int s) { return bar0 + 8u * (1 + QS + s); };
  const uint32_t s_full = bar0 + 8u * (1 + 2 * QS);
  const uint32_t ds_ready = s_full + 8, dq_full = s_full + 16, dq_empty = s_full + 24;
  const uint32_t dkv_final = s_full + 32, drain = s_full + 40;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* rtok = reinterpret_cast<int*>(smem + Tr::OFF_RTOK);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(qd_full(s), 1);
      mbar_init(qd_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(ds_ready, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 256);
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
      tma_prefetch_map(&tmDO);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      mbar_expect_tx(kv_full, 2u * Tr::TILE);
      for (int pn = 0; pn < Tr::NPANEL; ++pn) {
        tma_load_4d(sbase + Tr::OFF_K + pn * NK * ROWB, &tmK, kv_full, pn * PANEL, kvh, k0, b);
        tma_load_4d(sbase + Tr::OFF_V + pn * NK * ROWB, &tmV, kv_full, pn * PANEL, kvh, k0, b);
      }
      const uint32_t qd_bytes = 2u * p.rows * ROWB * Tr::NPANEL + 2u * 512u;
      int issued = 0;
      for (int i = 0; i < nq; ++i) {
        const int s = i % QS, qt = qt_first + i;
        if (i >= QS && !mbar_wait(qd_empty(s), ((i / QS) - 1) & 1, abort_flag, kSiteProducer)) break;
        mbar_expect_tx(qd_full(s), qd_bytes);
        for (int pn = 0; pn < Tr::NPANEL; ++pn) {
          tma_load_4d(sbase + Tr::OFF_Q + s * Tr::TILE + pn * BM * ROWB, &tmQ, qd_full(s), pn * PANEL, kvh * p.g,
                      qt * p.T, b);
          tma_load_4d(sbase + Tr::OFF_DO + s * Tr::TILE + pn * BM * ROWB, &tmDO, qd_full(s), pn * PANEL,
                      kvh * p.g, qt * p.T, b);
        }
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (the whole warp; one elected lane issues)
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);   // S^T, dP^T
    constexpr uint32_t idesc_kv = idesc_bf16_f32(128, DH, false, true);    // dV, dK (A in TMEM)
    constexpr uint32_t idesc_q = idesc_bf16_f32(128, DH, true, true);      // dQ (A = dS MN-major)
    const uint32_t k_addr = sbase + Tr::OFF_K, v_addr = sbase + Tr::OFF_V;
    const uint32_t ds_addr = sbase + Tr::OFF_DS;
    bool ok = mbar_wait_warp(kv_full, 0, abort_flag, kSiteMma);
    for (int i = 0; ok && i < nq; ++i) {
      const int s = i % QS;
      const uint32_t q_addr = sbase + Tr::OFF_Q + s * Tr::TILE, do_addr = sbase + Tr::OFF_DO + s * Tr::TILE;
      if (!mbar_wait_warp(qd_full(s), (i / QS) & 1, abort_flag, kSiteMma)) { ok = false; break; }
      if (Tr::TM_DQ == Tr::TM_ST && i > 0 && !mbar_wait_warp(dq_empty, (i - 1) & 1, abort_flag, kSiteMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // S^T = K Q^T and dP^T = V dO^T: M = 128 keys, N = 128 stacked query rows, K = dh.
#pragma unroll
      for (int ks = 0; ks < DH / 16; ++ks) {
        const uint32_t pn = (ks * 16) / PANEL, off = ((ks * 16) % PANEL) * 2;
        mma_ss_w(tmem + Tr::TM_ST, smem_desc(k_addr + pn * NK * ROWB + off, 16, 8 * ROWB, Tr::LAYOUT),
                 smem_desc(q_addr + pn * BM * ROWB + off, 16, 8 * ROWB, Tr::LAYOUT), idesc_s, ks > 0);
        mma_ss_w(tmem + Tr::TM_DPT, smem_desc(v_addr + pn * NK * ROWB + off, 16, 8 * ROWB, Tr::LAYOUT),
                 smem_desc(do_addr + pn * BM * ROWB + off, 16, 8 * ROWB, Tr::LAYOUT), idesc_s, ks > 0);
      }
      mma_commit_w(s_full);
      if (!mbar_wait_warp(ds_ready, i & 1, abort_flag, kSiteMma)) { ok = false; break; }
      tc_fence_after();
      // dV += P^T dO and dK += dS^T Q: K = 128 stacked query rows.  P^T / dS^T sit
      // in two 32-column halves of packed bf16 pairs at column offsets 0 and 64.
#pragma unroll
      for (int ks = 0; ks < BM / 16; ++ks) {
        const uint32_t acol = ks < 4 ? 8u * ks : 64u + 8u * (ks - 4);
        const uint32_t brow = ks * 16 * ROWB;
        mma_ts_w(tmem + Tr::TM_DV, tmem + Tr::TM_ST + acol,
                 smem_desc(do_addr + brow, BM * ROWB, 8 * ROWB, Tr::LAYOUT), idesc_kv, (i > 0 || ks > 0));
        mma_ts_w(tmem + Tr::TM_DK, tmem + Tr::TM_DPT + acol,
                 smem_desc(q_addr + brow, BM * ROWB, 8 * ROWB, Tr::LAYOUT), idesc_kv, (i > 0 || ks > 0));
      }
      if (Tr::TM_DQ != Tr::TM_ST && i > 0 && !mbar_wait_warp(dq_empty, (i - 1) & 1, abort_flag, kSiteMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // dQ = dS K: M = 128 stacked query rows, N = dh, K = 128 keys.  dS is
      // MN-major (query rows contiguous) with a 128-byte swizzle: two 64-row
      // panels 16 KB apart, 8-key groups 1 KB apart.
#pragma unroll
      for (int ks = 0; ks < NK / 16; ++ks)
        mma_ss_w(tmem + Tr::TM_DQ, smem_desc(ds_addr + ks * 2048, 16384, 1024, 2u),
                 smem_desc(k_addr + ks * 16 * ROWB, NK * ROWB, 8 * ROWB, Tr::LAYOUT), idesc_q, ks > 0);
      mma_commit_w(dq_full);
      mma_commit_w(qd_empty(s));
    }
    if (ok) mma_commit_w(dkv_final);
    else {
      mma_commit_w(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P, dS, dQ epilogue, dK/dV epilogue
    const int w = (warp - 4) >> 2;            // column half of the Q tile this warpgroup handles
    const int kk = (warp & 3) * 32 + lane;    // TMEM lane: key (S^T, dP^T, dK, dV) or query row (dQ)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = k0 + kk;
    const bool key_ok = key < p.N;
    const float sl2 = p.scale_log2;
    // dQ rows of this lane
    const int qrow_tok = kk < p.rows ? kk / p.g : (1 << 30);
    const int qrow_head = kvh * p.g + kk % p.g;
    uint8_t* ds_smem = smem + Tr::OFF_DS;
    bool ok = true;
    for (int i = 0; i < nq; ++i) {
      const int s = i % QS, qt = qt_first + i;
      // The statistics were bulk-copied into this stage; wait on that copy
      // directly (the stage is not refilled before this tile's ds_ready).
      ok = __all_sync(0xffffffffu, mbar_wait(qd_full(s), (i / QS) & 1, abort_flag, kSiteSoftmax) &&
                                       mbar_wait(s_full, i & 1, abort_flag, kSiteSoftmax));
      if (!ok) break;
      tc_fence_after();
      const float* lse2 = reinterpret_cast<const float*>(smem + Tr::OFF_STAT + s * 1024);  // negated
      const float* Dv = lse2 + 128;                                                          // negated
      const bool masked = p.causal && (k0 + NK - 1 > qt * p.T);
      const int key_rel = key - qt * p.T;  // visible iff key_rel <= rtok[r]
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int col0 = 64 * w + 32 * c;
        uint32_t sr[32], dr[32];
        tmem_ld32(lane_addr + Tr::TM_ST + col0, sr);
        tmem_ld32(lane_addr + Tr::TM_DPT + col0, dr);
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pv[2], dv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int r = col0 + e + u;
            float pr = ex2(fmaf(__uint_as_float(sr[e + u]), sl2, lse2[r]));
            if (!key_ok || (masked && key_rel > rtok[r])) pr = 0.f;
            pv[u] = pr;
            dv[u] = pr * (__uint_as_float(dr[e + u]) + Dv[r]);
          }
          pp[e >> 1] = pack_bf16x2(pv[0], pv[1]);
          dd[e >> 1] = pack_bf16x2(dv[0], dv[1]);
        }
        tmem_st16(lane_addr + Tr::TM_ST + 64 * w + 16 * c, pp);
        tmem_st16(lane_addr + Tr::TM_DPT + 64 * w + 16 * c, dd);
        // dS[q][key] for q = col0..col0+31 into the MN-major 128B-swizzled tile.
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int q = col0 + 8 * ch;
          const int panel = q >> 6, chunk = (q & 63) >> 3;
          uint4 v4 = make_uint4(dd[4 * ch], dd[4 * ch + 1], dd[4 * ch + 2], dd[4 * ch + 3]);
          *reinterpret_cast<uint4*>(ds_smem + panel * 16384 + kk * 128 + ((chunk ^ (kk & 7)) << 4)) = v4;
        }
      }
      tmem_wait_st();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ds_ready);
      // dQ epilogue: this warpgroup adds dh/2 columns of every stacked query row.
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full, i & 1, abort_flag, kSiteEpilogue));
      if (!ok) break;
      tc_fence_after();
      float v[DH / 2];
      tmem_ld_half<DH>(lane_addr + Tr::TM_DQ + w * (DH / 2), v);
      tc_fence_before();
      mbar_arrive(dq_empty);
      const int tok = qt * p.T + qrow_tok;
      if (tok < p.N) {
        float* dst = p.dq_acc + ((static_cast<size_t>(b) * p.N + tok) * p.Hq + qrow_head) * DH + w * (DH / 2);
#pragma unroll
        for (int c = 0; c < DH / 2; c += 4)
          atomicAdd(reinterpret_cast<float4*>(dst + c), make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]));
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
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace sqa

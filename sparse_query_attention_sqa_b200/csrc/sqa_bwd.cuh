// sqa_bwd.cuh -- Sparse Query Attention backward on sm_100a: workspace
// layout, the preprocess and dQ-conversion kernels, and what the main kernels
// (sqa_bwd_tf32.cuh for dh 16 / 32, sqa_bwd_bf16.cuh for dh 64 / 128) share.
//
// Three launches on the caller's stream:
//   1. prep:  -D_i = -<dO_i, O_i> and -lse_i * log2(e) for every query row,
//             written in the stacked-tile order the main kernel reads (slots of
//             padding rows get lse = +inf and D = 0, which makes their P exactly
//             0), and for dh <= 32 the fp32 dQ accumulator zeroed.
//   2. main:  work item = (128-key tile, batch, KV head).  K and V stay in
//             shared memory while the Q tiles that see those keys stream by.  A
//             Q tile stacks the g query heads of the group (row r = t * g +
//             head), so the dK and dV MMAs contract over tokens and heads at
//             once: the reduction over the query-head group happens inside the
//             tensor core accumulation in TMEM.  Per Q tile:
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
  size_t off_dq;       // dh <= 32 only: the fp32 dQ accumulator
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
  L.bytes = L.off_dq;
  if (dh <= 32)  // dh 64 / 128: dQ comes from its own kernel, with no accumulator
    L.bytes += align256(static_cast<size_t>(B) * N * Hq * dh * sizeof(float));
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
  const float* lse;
  float* lse2;
  float* D;
  float* dq_acc;
  int N, Hq, Hkv, g, T, rows, n_qt;
  long long n_slots;
  long long dq_vec4;  // dq accumulator length / 4
};

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
        }
      }
      l2 = p.lse[(static_cast<size_t>(b) * p.Hq + head) * p.N + tok] * 1.4426950408889634f;
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
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int N, Hq, Hkv, g, T, rows, n_qt, n_bh, causal;
  int n_items;  // persistent kernels: 128-key tiles x (batch, KV head)
  float scale_log2, scale;
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

}  // namespace sqa

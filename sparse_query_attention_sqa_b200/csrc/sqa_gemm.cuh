// sqa_gemm.cuh -- the projections around the attention core on sm_100a:
// D[M x N] = sum over K segments of A_s[M x K_s] B_s[K_s x N], bf16 operands
// staged by TMA (128-byte swizzle), tcgen05 MMAs with fp32 accumulators in
// TMEM, and one of three epilogues:
//   kStoreBf16  D rounded to bf16, row-major with a leading dimension
//   kQkvRope    the fused Q/K/V projection: columns [0, nq) are Q, [nq, nq + nk)
//               K, the rest V; Q and K columns are turned by the rotary
//               embedding of their token (pair (2j, 2j+1) of a head by the
//               angle pos * base^(-2j/dh), from a cos/sin table) and each part
//               is written bf16 to its own [M][width] tensor
//   kAtomicF32  D added to an fp32 row-major output with vector reductions
//               (split-K: each work item covers a range of K blocks)
//   kSwiGLU     the SwiGLU feed-forward's first product: each 256-column tile
//               is 128 columns of U W1 (the gate, from the first B map) beside
//               the same 128 columns of U W3 (from the second); the epilogue
//               writes a = U W1, b = U W3 and silu(a) * b, bf16
//   kSwiGLUBwd  its backward: D = dM (the gradient of silu(a) * b); with the
//               saved a and b the epilogue writes da = dM * b * silu'(a) and
//               db = dM * silu(a), bf16
// kStoreBf16 can add a bf16 residual (same layout as the output) before rounding.
// SQAT-m model card, "Model size difference": the query and output
// projections shrink with the query-head count (W_q is d x H_q dh, W_o is
// H_q dh x d); "Architecture details": rotary position embedding.
//
// Operands are K-major (K contiguous: row-major [M][K] for A, [N][K] for B)
// or MN-major (M or N contiguous: [K][M] for A, [K][N] for B), chosen by the
// template arguments, so X W, X^T G and G W^T all map onto the same kernel.
//
// Persistent: one CTA per SM walks the work items (128-row x BN-column output
// tiles, times the K splits).  Roles (256 threads): warp 0 TMA producer
// through a ring of STAGES stages of 64 K elements; warp 1 TMEM allocator and
// MMA issuer; warps 4-7 the epilogue (warp 4 + i reads TMEM lanes 32 i ..
// 32 i + 31, one output row per thread).  Two TMEM accumulators of BN columns
// let the epilogue of one item overlap the main loop of the next.
#pragma once

#include "sqa_device.cuh"
#include "sqa_tmem_wide.cuh"

namespace sqa {

enum GemmEpilogue : int { kStoreBf16 = 0, kQkvRope = 1, kAtomicF32 = 2, kSwiGLU = 3, kSwiGLUBwd = 4 };

struct GemmParams {
  int M, N;
  int n_seg;
  int kseg[3];    // K of each segment
  int kblk0[4];   // first K block (of 64) of each segment; kblk0[n_seg] = total blocks
  int tiles_m, tiles_n, split_k, n_items;
  int mode;
  // kStoreBf16 (and the outputs of the SwiGLU epilogues)
  __nv_bfloat16* out;
  long long ld_out;
  const __nv_bfloat16* resid;  // kStoreBf16: added before rounding, or null
  // kSwiGLU: a, b written beside out; kSwiGLUBwd: a, b read, da -> out, db -> out2
  __nv_bfloat16* sw_a;
  __nv_bfloat16* sw_b;
  __nv_bfloat16* out2;
  // kAtomicF32
  float* out32;
  long long ld_out32;
  // kQkvRope
  __nv_bfloat16* q;
  __nv_bfloat16* k;
  __nv_bfloat16* v;
  int nq, nk, nv;          // column counts of the three parts (multiples of 8)
  int dh, n_tokens;        // head dim; tokens per sequence (position = row % n_tokens)
  const float2* rope_cs;   // [n_tokens][dh / 2] (cos, sin), or null for no rotation
};

template <int BN>
struct GemmTraits {
  static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;  // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int OFF_BAR = STAGES * STAGE;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int N_BARS = 2 * STAGES + 5;
  static constexpr int SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
  static constexpr int SMEM_BYTES = (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) + 1024;
  static constexpr int THREADS = 256;
  static constexpr int WARP_PRODUCER = 0, WARP_MMA = 1, WARP_EPI0 = 4;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Work item -> (tile row, tile column, K-block range).
struct GemmItem {
  int m0, n0, kb0, kb1;
};
__device__ __forceinline__ GemmItem gemm_item(const GemmParams& p, int item, int bn) {
  GemmItem it;
  const int split = item % p.split_k;
  const int tile = item / p.split_k;
  it.m0 = (tile % p.tiles_m) * 128;
  it.n0 = (tile / p.tiles_m) * bn;
  const int nblk = p.kblk0[p.n_seg];
  it.kb0 = static_cast<int>(static_cast<long long>(nblk) * split / p.split_k);
  it.kb1 = static_cast<int>(static_cast<long long>(nblk) * (split + 1) / p.split_k);
  return it;
}

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(256, 1)
    sqa_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                    const GemmParams p) {
  using Tr = GemmTraits<BN>;
  using namespace dev;
  constexpr int BM = Tr::BM, BK = Tr::BK, ST = Tr::STAGES;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (ST + s); };
  auto acc_full = [&](int b) { return bar0 + 8u * (2 * ST + b); };
  auto acc_empty = [&](int b) { return bar0 + 8u * (2 * ST + 2 + b); };
  const uint32_t drain = bar0 + 8u * (2 * ST + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
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
      const CUtensorMap* mA[3] = {&tmA0, &tmA1, &tmA2};
      const CUtensorMap* mB[3] = {&tmB0, &tmB1, &tmB2};
      for (int sgi = 0; sgi < p.n_seg; ++sgi) {
        tma_prefetch_map(mA[sgi]);
        tma_prefetch_map(mB[sgi]);
      }
      int g = 0;  // K blocks issued so far (across items)
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const GemmItem it = gemm_item(p, item, p.mode == kSwiGLU ? BN / 2 : BN);
        const int n0 = it.n0;
        int sgi = 0;
        for (int kb = it.kb0; kb < it.kb1; ++kb, ++g) {
          while (kb >= p.kblk0[sgi + 1]) ++sgi;
          const int k0 = (kb - p.kblk0[sgi]) * BK;
          const int s = g % ST;
          if (g >= ST && !mbar_wait(empty(s), ((g / ST) - 1) & 1, abort_flag, kSiteProducer)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = sbase + s * Tr::STAGE, b_dst = a_dst + Tr::A_BYTES;
          mbar_expect_tx(full(s), Tr::STAGE);
          if (A_MN) {  // [K][M]: two 64-row panels of M, each 64 K rows x 128 bytes
            tma_load_2d(a_dst, mA[sgi], full(s), it.m0, k0);
            tma_load_2d(a_dst + 8192, mA[sgi], full(s), it.m0 + 64, k0);
          } else {  // [M][K]: 128 rows x 128 bytes
            tma_load_2d(a_dst, mA[sgi], full(s), k0, it.m0);
          }
          if (BN >= 128 && B_MN && p.mode == kSwiGLU) {  // BN / 2 columns of W1, then the same of W3
            constexpr int HALF = BN >= 128 ? BN / 128 : 1;  // 64-column panels per half
#pragma unroll
            for (int pn = 0; pn < BN / 64; ++pn)
              tma_load_2d(b_dst + pn * 8192, pn < HALF ? mB[0] : mB[1], full(s), n0 + 64 * (pn % HALF), k0);
          } else if (B_MN) {  // [K][N]: BN / 64 panels of N, each 64 K rows x 128 bytes
#pragma unroll
            for (int pn = 0; pn < BN / 64; ++pn) tma_load_2d(b_dst + pn * 8192, mB[sgi], full(s), n0 + 64 * pn, k0);
          } else {  // [N][K]: BN rows x 128 bytes
            tma_load_2d(b_dst, mB[sgi], full(s), k0, n0);
          }
        }
      }
      if (*abort_flag) {
        for (int j = max(0, g - ST); j < g; ++j) mbar_wait_drain(full(j % ST), (j / ST) & 1);
      }
    }
  } else if (warp == Tr::WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one elected lane)
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
    int g = 0, r = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++r) {
      const GemmItem it = gemm_item(p, item, p.mode == kSwiGLU ? BN / 2 : BN);
      const int ab = r & 1;
      if (r >= 2 && !(ok = mbar_wait_warp(acc_empty(ab), ((r >> 1) - 1) & 1, abort_flag, kSiteMma))) break;
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(ab * BN);
      for (int kb = it.kb0; kb < it.kb1; ++kb, ++g) {
        const int s = g % ST;
        if (!(ok = mbar_wait_warp(full(s), (g / ST) & 1, abort_flag, kSiteMma))) break;
        tc_fence_after();
        const uint32_t a_addr = sbase + s * Tr::STAGE, b_addr = a_addr + Tr::A_BYTES;
#pragma unroll
        for (int ks = 0; ks < BK / 16; ++ks) {
          // K-major: 16 K elements are 32 bytes along the swizzled row; MN-major:
          // 16 K rows of 128 bytes, panels 8 KB apart.
          const uint64_t da = A_MN ? smem_desc(a_addr + ks * 2048, 8192, 1024, 2u)
                                   : smem_desc(a_addr + ks * 32, 16, 1024, 2u);
          const uint64_t db = B_MN ? smem_desc(b_addr + ks * 2048, 8192, 1024, 2u)
                                   : smem_desc(b_addr + ks * 32, 16, 1024, 2u);
          mma_ss_w(d_tmem, da, db, idesc, (kb > it.kb0 || ks > 0) ? 1u : 0u);
        }
        mma_commit_w(empty(s));
      }
      if (!ok) break;
      mma_commit_w(acc_full(ab));
    }
    if (!ok) {
      mma_commit_w(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= Tr::WARP_EPI0) {
    // ------------------------------------------------------------ epilogue: one output row per thread
    const int lw = warp - Tr::WARP_EPI0;
    const int row = lw * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(lw * 32) << 16);
    int r = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++r) {
      const GemmItem it = gemm_item(p, item, p.mode == kSwiGLU ? BN / 2 : BN);
      const int ab = r & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(acc_full(ab), (r >> 1) & 1, abort_flag, kSiteEpilogue));
      if (!ok) break;
      tc_fence_after();
      const int m = it.m0 + row;
      const bool row_ok = m < p.M;
      const int n_base = it.n0;
      if (p.mode == kSwiGLU) {
        // columns [0, BN/2): a = U W1, [BN/2, BN): b = U W3, for hidden columns n_base ..
#pragma unroll 1
        for (int c0 = 0; c0 < BN / 2; c0 += 32) {
          uint32_t ra[32], rb[32];
          tmem_ld32(lane_addr + static_cast<uint32_t>(ab * BN + c0), ra);
          tmem_ld32(lane_addr + static_cast<uint32_t>(ab * BN + BN / 2 + c0), rb);
          if (c0 + 32 == BN / 2) {
            tc_fence_before();
            mbar_arrive(acc_empty(ab));
          }
          if (!row_ok) continue;
          const long long o = static_cast<long long>(m) * p.ld_out + n_base + c0;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            if (n_base + c0 + e >= p.N) continue;
            uint4 oa, ob, om;
            uint32_t* pa = &oa.x;
            uint32_t* pb = &ob.x;
            uint32_t* pm = &om.x;
#pragma unroll
            for (int u = 0; u < 8; u += 2) {
              const float a0 = __uint_as_float(ra[e + u]), a1 = __uint_as_float(ra[e + u + 1]);
              const float b0 = __uint_as_float(rb[e + u]), b1 = __uint_as_float(rb[e + u + 1]);
              // silu(a) = a / (1 + 2^(-a log2 e))
              const float s0 = a0 / (1.f + ex2(-1.4426950408889634f * a0));
              const float s1 = a1 / (1.f + ex2(-1.4426950408889634f * a1));
              pa[u >> 1] = pack_bf16x2(a0, a1);
              pb[u >> 1] = pack_bf16x2(b0, b1);
              pm[u >> 1] = pack_bf16x2(s0 * b0, s1 * b1);
            }
            *reinterpret_cast<uint4*>(p.sw_a + o + e) = oa;
            *reinterpret_cast<uint4*>(p.sw_b + o + e) = ob;
            *reinterpret_cast<uint4*>(p.out + o + e) = om;
          }
        }
        continue;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t rr[32];
        tmem_ld32(lane_addr + static_cast<uint32_t>(ab * BN + c0), rr);
        if (c0 + 32 == BN) {  // every column of this accumulator is in registers
          tc_fence_before();
          mbar_arrive(acc_empty(ab));
        }
        if (!row_ok) continue;
        if (p.mode == kAtomicF32) {
          float* dst = p.out32 + static_cast<long long>(m) * p.ld_out32 + n_base + c0;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            if (n_base + c0 + e < p.N)
              atomicAdd(reinterpret_cast<float4*>(dst + e),
                        make_float4(__uint_as_float(rr[e]), __uint_as_float(rr[e + 1]), __uint_as_float(rr[e + 2]),
                                    __uint_as_float(rr[e + 3])));
        } else if (p.mode == kStoreBf16) {
          const long long o0 = static_cast<long long>(m) * p.ld_out + n_base + c0;
          __nv_bfloat16* dst = p.out + o0;
#pragma unroll
          for (int e = 0; e < 32; e += 8)
            if (n_base + c0 + e < p.N) {
              float y[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) y[u] = __uint_as_float(rr[e + u]);
              if (p.resid) {
                const uint4 rv = *reinterpret_cast<const uint4*>(p.resid + o0 + e);
                const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rv);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const float2 f = __bfloat1622float2(r2[u]);
                  y[2 * u] += f.x;
                  y[2 * u + 1] += f.y;
                }
              }
              uint4 o;
              o.x = pack_bf16x2(y[0], y[1]);
              o.y = pack_bf16x2(y[2], y[3]);
              o.z = pack_bf16x2(y[4], y[5]);
              o.w = pack_bf16x2(y[6], y[7]);
              *reinterpret_cast<uint4*>(dst + e) = o;
            }
        } else if (p.mode == kSwiGLUBwd) {
          // D = dM; with the saved a, b: da = dM b silu'(a), db = dM silu(a),
          // silu'(a) = s + a s (1 - s), s = 1 / (1 + e^-a)
          const long long o0 = static_cast<long long>(m) * p.ld_out + n_base + c0;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            if (n_base + c0 + e >= p.N) continue;
            const uint4 av = *reinterpret_cast<const uint4*>(p.sw_a + o0 + e);
            const uint4 bv = *reinterpret_cast<const uint4*>(p.sw_b + o0 + e);
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&av);
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bv);
            uint4 oa, ob;
            uint32_t* pa = &oa.x;
            uint32_t* pb = &ob.x;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 a = __bfloat1622float2(a2[u]), b = __bfloat1622float2(b2[u]);
              const float dm0 = __uint_as_float(rr[e + 2 * u]), dm1 = __uint_as_float(rr[e + 2 * u + 1]);
              const float s0 = 1.f / (1.f + ex2(-1.4426950408889634f * a.x));
              const float s1 = 1.f / (1.f + ex2(-1.4426950408889634f * a.y));
              pa[u] = pack_bf16x2(dm0 * b.x * (s0 + a.x * s0 * (1.f - s0)), dm1 * b.y * (s1 + a.y * s1 * (1.f - s1)));
              pb[u] = pack_bf16x2(dm0 * a.x * s0, dm1 * a.y * s1);
            }
            *reinterpret_cast<uint4*>(p.out + o0 + e) = oa;
            *reinterpret_cast<uint4*>(p.out2 + o0 + e) = ob;
          }
        } else {  // kQkvRope
          const int pos = m % p.n_tokens;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            const int n = n_base + c0 + e;  // 8 columns of one part and one head (parts are multiples of 8)
            if (n >= p.N) continue;
            __nv_bfloat16* base;
            int c, width;
            bool rot;
            if (n < p.nq) {
              base = p.q; c = n; width = p.nq; rot = true;
            } else if (n < p.nq + p.nk) {
              base = p.k; c = n - p.nq; width = p.nk; rot = true;
            } else {
              base = p.v; c = n - p.nq - p.nk; width = p.nv; rot = false;
            }
            float y[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) y[u] = __uint_as_float(rr[e + u]);
            if (rot && p.rope_cs) {
              const float2* cs = p.rope_cs + static_cast<long long>(pos) * (p.dh >> 1) + ((c % p.dh) >> 1);
#pragma unroll
              for (int u = 0; u < 8; u += 2) {
                const float2 t = cs[u >> 1];
                const float a = y[u], b = y[u + 1];
                y[u] = a * t.x - b * t.y;
                y[u + 1] = a * t.y + b * t.x;
              }
            }
            uint4 o;
            o.x = pack_bf16x2(y[0], y[1]);
            o.y = pack_bf16x2(y[2], y[3]);
            o.z = pack_bf16x2(y[4], y[5]);
            o.w = pack_bf16x2(y[6], y[7]);
            *reinterpret_cast<uint4*>(base + static_cast<long long>(m) * width + c) = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Tr::WARP_MMA) tmem_dealloc(tmem, 512);
}

// Rotary table: cs[pos][j] = (cos, sin)(pos * base^(-2j/dh)), angles formed and
// reduced in double precision, then rounded to fp32.
__global__ void __launch_bounds__(256) sqa_rope_table_kernel(float2* cs, int n_tokens, int dh, double base) {
  const int half = dh >> 1;
  const long long n = static_cast<long long>(n_tokens) * half;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int pos = static_cast<int>(i / half), j = static_cast<int>(i % half);
    const double theta = pow(base, -2.0 * j / dh);
    double s, c;
    sincos(static_cast<double>(pos) * theta, &s, &c);
    cs[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

// Inverse rotation in place on x [rows][width] bf16 (width a multiple of dh):
// pair (2j, 2j+1) of every head of row r turned by -pos * theta_j, pos = r % n_tokens.
__global__ void __launch_bounds__(256)
    sqa_rope_inverse_kernel(__nv_bfloat16* x, long long rows, int width, int dh, int n_tokens, const float2* cs) {
  const long long n8 = rows * (width / 8);
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / (width / 8);
    const int c = static_cast<int>(i % (width / 8)) * 8;
    const int pos = static_cast<int>(r % n_tokens);
    uint4* ptr = reinterpret_cast<uint4*>(x + r * width + c);
    uint4 v = *ptr;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
    const float2* t = cs + static_cast<long long>(pos) * (dh >> 1) + ((c % dh) >> 1);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(h[u]);
      const float2 cs2 = t[u];
      const float a = f.x * cs2.x + f.y * cs2.y;   // turn by -angle
      const float b = -f.x * cs2.y + f.y * cs2.x;
      h[u] = __floats2bfloat162_rn(a, b);
    }
    *ptr = v;
  }
}

}  // namespace sqa

// sqa_decode.cuh -- Sparse Query Attention decoding step on sm_100a: one new
// query token per sequence attends to the first lens[b] entries of its
// key/value cache.
//
// The cost of this step is reading the cache (H_kv heads of K and V per
// position), not the scores: reducing the query heads saves nothing here
// (arXiv 2510.01817 abstract: the gains are in compute-bound settings; the
// GQA summary, "The idea": the K/V head count sets the cache size).  So the
// kernels are built to stream the cache from HBM once at full width.  With g
// query heads per K/V head there are 4 g dh flops per cached position (scores
// and P V): for small groups the CUDA cores keep up with HBM; from about five
// heads up they do not, and warp-level tensor-core MMAs take the products.
//
// Two launches, split-K over the cache:
//   1. split:   one CTA per (range of positions, batch entry[, K/V head]),
//               writing per query head the range's unnormalised output o with
//               its running maximum m and sum l (log2 units) to the workspace.
//               Three paths:
//               - register-resident (groups of at most 4 query heads, a
//                 power-of-two K/V head count): the range's cache rows of all
//                 K/V heads are one contiguous run; dh / 8 lanes share a row,
//                 each thread slot keeps its own running softmax state in
//                 registers with several rows' loads in flight, and the slots
//                 of each K/V head merge once at the end.  The number of
//                 ranges makes about four waves of resident CTAs.
//               - tensor cores (groups of 5 to 16 heads): one CTA of four
//                 warps per (range, K/V head, batch entry), mma.sync on a
//                 16-head by 16-key tile per warp step (see the kernel).
//               - general (any group up to 128 heads): one CTA per (4 chunks
//                 of positions, K/V head, batch entry); chunks (256 positions
//                 at dh <= 32, 128 at dh = 64, 64 at dh = 128) are copied into
//                 shared memory with cp.async, double-buffered, and scored for
//                 all g heads of the group with block-wide online softmax.
//   2. combine: one CTA per (batch entry, query head) merges the ranges, its
//               threads spread over (column, range) pairs:
//               M = max m, L = sum l 2^(m - M), out = sum o 2^(m - M) / L (bf16),
//               lse = ln 2 * (M + log2 L).
#pragma once

#include "sqa_device.cuh"

namespace sqa {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeChunksPerCta = 4;
// Cache positions per chunk: sized so that two chunk buffers, a group of up to
// 128 heads' scores, queries and running outputs fit in shared memory.
__host__ __device__ constexpr int decode_chunk(int dh) { return dh <= 32 ? 256 : (dh == 64 ? 128 : 64); }
// Positions per split-kernel CTA (one partial result each).
__host__ __device__ constexpr int decode_span(int dh) { return decode_chunk(dh) * kDecodeChunksPerCta; }

struct DecodeParams {
  const __nv_bfloat16* q;  // [B][H_q][dh]
  const __nv_bfloat16* k;  // [B][N][H_kv][dh]
  const __nv_bfloat16* v;
  const int* lens;         // [B] positions in use, or null for all N
  float* part;             // [B * H_kv][n_split][g][dh + 2]: o, then m and l (log2 units)
  __nv_bfloat16* out;      // [B][H_q][dh]
  float* lse;              // [B][H_q]
  int N, Hq, Hkv, g, n_split;
  int span;                // positions per range (one partial each)
  float scale_log2;        // scale * log2(e)
};

// Register-resident split path, for groups of at most four query heads whose
// K/V head count is a power of two no larger than the rows a CTA takes per
// step.  L = dh / 8 lanes share one cache row (16 bytes of K and 16 of V
// each); a CTA of kDecodeThreads takes rows_step(dh) consecutive rows per step.
constexpr int kRowsMaxGroup = 4;
constexpr int kRowsMinSteps = 16;  // the shortest range is this many steps
__host__ __device__ constexpr int rows_step(int dh) { return kDecodeThreads * 8 / dh; }
__host__ __device__ constexpr bool rows_path(int g, int hkv, int dh) {
  return g >= 1 && g <= kRowsMaxGroup && hkv >= 1 && (hkv & (hkv - 1)) == 0 && hkv <= rows_step(dh);
}
// Shortest range of positions (kRowsMinSteps steps of the CTA).
__host__ __device__ constexpr int rows_min_span(int dh, int hkv) { return kRowsMinSteps * rows_step(dh) / hkv; }
// Rows in flight per thread of the register-resident path, and its ring of
// shared-memory slots (one more than that, so a refill never targets the slot
// being read).  Three rows ahead keep the ring at 32 KB, so that registers,
// not shared memory, bound the resident CTAs (three per SM for a group of
// two); more CTAs hide the arithmetic's latencies better than deeper rings.
constexpr int kRowsDepth = 3, kRowsSlots = kRowsDepth + 1;
// Shared memory of the register-resident path: the per-thread ring of K and V
// row pieces (16 bytes each) during the run, then one (o, m, l) record per
// thread slot for the end-of-range merge.
__host__ __device__ constexpr size_t rows_smem_bytes(int g, int dh) {
  const size_t ring = static_cast<size_t>(kRowsSlots) * kDecodeThreads * 32;
  const size_t recs = static_cast<size_t>(rows_step(dh)) * g * (dh + 2) * 4;
  return ring > recs ? ring : recs;
}

// Shared memory of the split kernel, in bytes: queries and running outputs
// [g][dh] fp32, scores [g][chunk] fp32, two K and two V chunk buffers (bf16),
// per-head m, l and rescale factor, and (for groups with fewer than one output
// per thread) two partial sums per thread.
__host__ __device__ constexpr size_t decode_smem_bytes(int g, int dh) {
  return 2 * static_cast<size_t>(g) * dh * 4 + static_cast<size_t>(g) * decode_chunk(dh) * 4 +
         4 * static_cast<size_t>(decode_chunk(dh)) * dh * 2 + static_cast<size_t>(g) * 12 +
         (g * dh < kDecodeThreads ? 2 * kDecodeThreads * 4 : 0);
}

__device__ __forceinline__ int decode_len(const DecodeParams& p, int b) {
  const int len = p.lens ? p.lens[b] : p.N;
  return len < 0 ? 0 : (len > p.N ? p.N : len);
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dev::smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// General split path: any group size, the range's chunks staged in shared memory.
template <int DH>
__device__ __forceinline__ void decode_split_general(const DecodeParams& p) {
  constexpr int CH = decode_chunk(DH), VEC = DH / 8;  // 16-byte vectors per row
  const int split = blockIdx.x / p.Hkv, kvh = blockIdx.x % p.Hkv, b = blockIdx.y;
  const int bk = b * p.Hkv + kvh, g = p.g, go = g * DH;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int len = decode_len(p, b);
  const int c_first = split * kDecodeChunksPerCta;
  const int n_chunks = max(0, min(kDecodeChunksPerCta, (len + CH - 1) / CH - c_first));
  float* part = p.part + (static_cast<size_t>(bk) * p.n_split + split) * g * (DH + 2);

  if (n_chunks == 0) {  // range past this sequence's length: an empty partial
    for (int i = tid; i < g * (DH + 2); i += kDecodeThreads) {
      const int c = i % (DH + 2);
      part[i] = c == DH ? -INFINITY : 0.f;
    }
    return;
  }

  extern __shared__ __align__(16) uint8_t dsm[];
  float* qs = reinterpret_cast<float*>(dsm);                         // [g][DH]
  float* os = qs + go;                                                // [g][DH] running output
  float* ss = os + go;                                                // [g][CH] scores, then weights
  __nv_bfloat16* kvs = reinterpret_cast<__nv_bfloat16*>(ss + g * CH);  // [2][K, V][CH][DH]
  float* mrun = reinterpret_cast<float*>(kvs + 4 * CH * DH);           // [g]
  float* lrun = mrun + g;                                              // [g]
  float* alpha = lrun + g;                                             // [g]
  float* red = alpha + g;  // [2 * kDecodeThreads] partial sums, only when g * DH < kDecodeThreads

  auto chunk_rows = [&](int c) { return min(CH, len - (c_first + c) * CH); };
  auto load_chunk = [&](int c) {  // cp.async of chunk c into buffer c % 2
    const int j0 = (c_first + c) * CH, cnt = chunk_rows(c);
    __nv_bfloat16* kb = kvs + (c & 1) * 2 * CH * DH;
    __nv_bfloat16* vb = kb + CH * DH;
    for (int i = tid; i < cnt * VEC; i += kDecodeThreads) {
      const int j = i / VEC, cc = i % VEC;
      const size_t row = (static_cast<size_t>(b) * p.N + j0 + j) * p.Hkv + kvh;
      cp_async16(kb + j * DH + cc * 8, p.k + row * DH + cc * 8);
      cp_async16(vb + j * DH + cc * 8, p.v + row * DH + cc * 8);
    }
    cp_async_commit();
  };

  load_chunk(0);
  // Queries of the group (heads kvh*g .. kvh*g+g-1 are adjacent); running state.
  const __nv_bfloat16* qg = p.q + (static_cast<size_t>(b) * p.Hq + kvh * g) * DH;
  for (int i = tid; i < go; i += kDecodeThreads) {
    qs[i] = __bfloat162float(qg[i]);
    os[i] = 0.f;
  }
  for (int h = tid; h < g; h += kDecodeThreads) {
    mrun[h] = -INFINITY;
    lrun[h] = 0.f;
  }

  for (int c = 0; c < n_chunks; ++c) {
    if (c + 1 < n_chunks) {
      load_chunk(c + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // chunk c (and, at c = 0, the queries) visible to every thread
    const int cnt = chunk_rows(c);
    const __nv_bfloat16* kb = kvs + (c & 1) * 2 * CH * DH;
    const __nv_bfloat16* vb = kb + CH * DH;

    // Scores in log2 units; positions past the chunk's end get -inf.
    if constexpr (CH == kDecodeThreads) {
      // One position per thread: its key row is read once into registers and
      // dotted with every query of the group in packed fp32 pairs (the queries
      // are the same address for the whole warp).
      const int j = tid;
      float2 kr[DH / 2];
      if (j < cnt) {
#pragma unroll
        for (int cc = 0; cc < VEC; ++cc) {
          const uint4 u = reinterpret_cast<const uint4*>(kb + j * DH)[cc];
          const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) kr[4 * cc + e] = __bfloat1622float2(k2[e]);
        }
      }
      for (int h = 0; h < g; ++h) {
        float acc = -INFINITY;
        if (j < cnt) {
          const float4* qh = reinterpret_cast<const float4*>(qs + h * DH);
          float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < DH / 4; ++e) {
            const float4 qv = qh[e];
            a2 = __ffma2_rn(make_float2(qv.x, qv.y), kr[2 * e], a2);
            a2 = __ffma2_rn(make_float2(qv.z, qv.w), kr[2 * e + 1], a2);
          }
          acc = (a2.x + a2.y) * p.scale_log2;
        }
        ss[h * CH + j] = acc;
      }
    } else {
      for (int i = tid; i < g * CH; i += kDecodeThreads) {
        const int h = i / CH, j = i % CH;
        float acc = -INFINITY;
        if (j < cnt) {
          const float* qh = qs + h * DH;
          const uint4* kr = reinterpret_cast<const uint4*>(kb + j * DH);
          acc = 0.f;
#pragma unroll
          for (int cc = 0; cc < VEC; ++cc) {
            const uint4 u = kr[cc];
            const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 kf = __bfloat1622float2(k2[e]);
              acc = fmaf(qh[8 * cc + 2 * e], kf.x, acc);
              acc = fmaf(qh[8 * cc + 2 * e + 1], kf.y, acc);
            }
          }
          acc *= p.scale_log2;
        }
        ss[i] = acc;
      }
    }
    __syncthreads();

    // Per head: new running maximum, weights 2^(s - m) in place, running sum.
    for (int h = warp; h < g; h += kDecodeThreads / 32) {
      float* sh = ss + h * CH;
      float m = mrun[h];
      for (int j = lane; j < CH; j += 32) m = fmaxf(m, sh[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float l = 0.f;
      for (int j = lane; j < CH; j += 32) {
        const float w = dev::ex2(sh[j] - m);  // -inf past the end gives 0
        sh[j] = w;
        l += w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) {
        const float a = mrun[h] == -INFINITY ? 0.f : dev::ex2(mrun[h] - m);
        alpha[h] = a;
        lrun[h] = lrun[h] * a + l;
        mrun[h] = m;
      }
    }
    __syncthreads();

    // Running output: o = o * alpha + sum_j w_j V_j.  With fewer outputs than
    // threads, nsub threads share one output, each over every nsub-th position.
    if (go >= kDecodeThreads) {
      for (int i = tid; i < go; i += kDecodeThreads) {
        const int h = i / DH, d = i % DH;
        const float* wh = ss + h * CH;
        float acc = 0.f;
        for (int j = 0; j < cnt; ++j) acc = fmaf(wh[j], __bfloat162float(vb[j * DH + d]), acc);
        os[i] = fmaf(os[i], alpha[h], acc);
      }
    } else {
      // Outputs in adjacent pairs (one bf16x2 load of V, one packed FMA each).
      const int gp = go / 2, nsub = kDecodeThreads / gp, o = tid % gp, sub = tid / gp;
      float2 acc = make_float2(0.f, 0.f);
      if (sub < nsub) {
        const int h = (2 * o) / DH, d = (2 * o) % DH;
        const float* wh = ss + h * CH;
        const __nv_bfloat162* vcol = reinterpret_cast<const __nv_bfloat162*>(vb + d);
        for (int j = sub; j < cnt; j += nsub) {
          const float w = wh[j];
          acc = __ffma2_rn(make_float2(w, w), __bfloat1622float2(vcol[j * (DH / 2)]), acc);
        }
      }
      red[2 * tid] = acc.x;
      red[2 * tid + 1] = acc.y;
      __syncthreads();
      if (tid < go) {
        float sum = red[tid];
        for (int k = 1; k < nsub; ++k) sum += red[tid + k * go];
        os[tid] = fmaf(os[tid], alpha[tid / DH], sum);
      }
    }
    __syncthreads();  // buffer c % 2 and the scores are free for the next chunk
  }

  for (int i = tid; i < go; i += kDecodeThreads) part[(i / DH) * (DH + 2) + i % DH] = os[i];
  for (int h = tid; h < g; h += kDecodeThreads) {
    part[h * (DH + 2) + DH] = mrun[h];
    part[h * (DH + 2) + DH + 1] = lrun[h];
  }
}

__device__ __forceinline__ float2 bf2f(uint32_t w) {
  __nv_bfloat162 h;
  memcpy(&h, &w, 4);
  return __bfloat1622float2(h);
}

// One cache row's step of the online softmax for the G heads a thread slot
// holds: scores from this lane's 8 columns summed over the L lanes of the row
// (butterfly, so every lane of the row gets the same sum), then either the
// plain update (no score above its head's running maximum anywhere in the
// warp) or the rescaling one.
template <int G, int L>
__device__ __forceinline__ void rows_update(const uint4& kc, const uint4& vc, bool valid, const float2 (&q)[G][4],
                                            float2 (&o)[G][4], float (&m)[G], float (&l)[G]) {
  const float2 k0 = bf2f(kc.x), k1 = bf2f(kc.y), k2 = bf2f(kc.z), k3 = bf2f(kc.w);
  float sc[G];
  bool up = false;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float2 a = __fmul2_rn(q[h][0], k0);
    a = __ffma2_rn(q[h][1], k1, a);
    a = __ffma2_rn(q[h][2], k2, a);
    a = __ffma2_rn(q[h][3], k3, a);
    float t = a.x + a.y;
#pragma unroll
    for (int off = 1; off < L; off <<= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    sc[h] = t;
    up |= t > m[h];
  }
  up = up && valid;
  const float2 v0 = bf2f(vc.x), v1 = bf2f(vc.y), v2 = bf2f(vc.z), v3 = bf2f(vc.w);
  if (__any_sync(0xffffffffu, up)) {
    if (valid) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mn = fmaxf(m[h], sc[h]);
        const float a = dev::ex2(m[h] - mn);  // 0 while m is -inf
        const float w = dev::ex2(sc[h] - mn);
        l[h] = fmaf(l[h], a, w);
        const float2 a2 = make_float2(a, a), w2 = make_float2(w, w);
        o[h][0] = __ffma2_rn(o[h][0], a2, __fmul2_rn(w2, v0));
        o[h][1] = __ffma2_rn(o[h][1], a2, __fmul2_rn(w2, v1));
        o[h][2] = __ffma2_rn(o[h][2], a2, __fmul2_rn(w2, v2));
        o[h][3] = __ffma2_rn(o[h][3], a2, __fmul2_rn(w2, v3));
        m[h] = mn;
      }
    }
  } else if (valid) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float w = dev::ex2(sc[h] - m[h]);
      l[h] += w;
      const float2 w2 = make_float2(w, w);
      o[h][0] = __ffma2_rn(w2, v0, o[h][0]);
      o[h][1] = __ffma2_rn(w2, v1, o[h][1]);
      o[h][2] = __ffma2_rn(w2, v2, o[h][2]);
      o[h][3] = __ffma2_rn(w2, v3, o[h][3]);
    }
  }
}

// Register-resident split path (rows_path(g, H_kv, dh) holds, G = g).
//
// The cache of one sequence is [N][H_kv][dh]: N * H_kv rows of dh elements,
// and a range of positions is one contiguous run of rows.  L = dh / 8 lanes
// share a row, so one warp load covers 32 / L whole consecutive rows (full
// 128-byte lines).  Thread slot t (L lanes) takes rows t, t + STEP, ... of
// the run; STEP is a multiple of H_kv, so the slot always meets K/V head
// t mod H_kv.  It keeps that head's G queries (its 8 columns, in log2 units),
// its own running maxima, sums and outputs in registers, and the copies of
// its next kRowsDepth rows in flight through a private ring of shared-memory
// slots; nothing is shared between threads during the run.  At the end
// the slots of each head merge (warp butterfly over slots of the same head,
// then one record per remaining slot in shared memory) into the partial
// (o, m, l) per head that the general path writes.
template <int DH, int G>
__device__ __forceinline__ void decode_split_rows(const DecodeParams& p) {
  constexpr int L = DH / 8, P = 32 / L, STEP = rows_step(DH), REC = G * (DH + 2);
  static_assert(STEP == (kDecodeThreads / 32) * P, "a step is one row per thread slot");
  const int split = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot = lane / L, col = (lane % L) * 8;
  const int t = warp * P + slot;
  const int Hkv = p.Hkv, kvh = t & (Hkv - 1);
  const int len = decode_len(p, b);
  const int j0 = split * p.span, j1 = min(len, j0 + p.span);
  const long long n_rows = static_cast<long long>(max(j1 - j0, 0)) * Hkv;
  const size_t first = (static_cast<size_t>(b) * p.N + (j0 < len ? j0 : 0)) * Hkv;
  const __nv_bfloat16* kr = p.k + first * DH + col;
  const __nv_bfloat16* vr = p.v + first * DH + col;

  float2 q[G][4], o[G][4];
  float m[G], l[G];
  {
    const __nv_bfloat16* qg = p.q + (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(kvh) * G) * DH + col;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint4 u = *reinterpret_cast<const uint4*>(qg + h * DH);
      const float2 s2 = make_float2(p.scale_log2, p.scale_log2);
      q[h][0] = __fmul2_rn(bf2f(u.x), s2);
      q[h][1] = __fmul2_rn(bf2f(u.y), s2);
      q[h][2] = __fmul2_rn(bf2f(u.z), s2);
      q[h][3] = __fmul2_rn(bf2f(u.w), s2);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[h][e] = make_float2(0.f, 0.f);
      m[h] = -INFINITY;
      l[h] = 0.f;
    }
  }

  // Each thread streams its rows through its own ring of shared-memory slots
  // with cp.async (16 bytes of K and 16 of V per row), kRowsDepth rows ahead;
  // it reads back only what it copied itself, so no barrier is needed.
  extern __shared__ __align__(16) uint8_t dsm[];
  uint4* ring_k = reinterpret_cast<uint4*>(dsm);  // [kRowsSlots][kDecodeThreads]
  uint4* ring_v = ring_k + kRowsSlots * kDecodeThreads;
  const int n_steps = static_cast<int>((n_rows + STEP - 1) / STEP);  // the same for every thread
  auto issue = [&](int st) {
    const long long r = t + static_cast<long long>(st) * STEP;
    if (r < n_rows) {
      const int sl = st % kRowsSlots;
      cp_async16(ring_k + sl * kDecodeThreads + tid, kr + r * DH);
      cp_async16(ring_v + sl * kDecodeThreads + tid, vr + r * DH);
    }
    cp_async_commit();  // one group per step, empty past the run
  };
#pragma unroll 1
  for (int i = 0; i < kRowsDepth; ++i) issue(i);
#pragma unroll 1
  for (int st = 0; st < n_steps; ++st) {
    issue(st + kRowsDepth);          // slot (st - 1) mod kRowsSlots, read in the previous step
    cp_async_wait<kRowsDepth>();     // every group but the newest kRowsDepth: step st has landed
    const int sl = st % kRowsSlots;
    const uint4 kc = ring_k[sl * kDecodeThreads + tid], vc = ring_v[sl * kDecodeThreads + tid];
    rows_update<G, L>(kc, vc, t + static_cast<long long>(st) * STEP < n_rows, q, o, m, l);
  }
  cp_async_wait<0>();

  // Merge the slots of one head inside the warp: slot offsets that are
  // multiples of H_kv (a power of two) keep the head and the columns.
  for (int off = Hkv * L; off < 32; off <<= 1) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
      const float mn = fmaxf(m[h], mo);
      const float a = m[h] == -INFINITY ? 0.f : dev::ex2(m[h] - mn);
      const float c = mo == -INFINITY ? 0.f : dev::ex2(mo - mn);
      l[h] = l[h] * a + lo * c;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float ox = __shfl_xor_sync(0xffffffffu, o[h][e].x, off);
        const float oy = __shfl_xor_sync(0xffffffffu, o[h][e].y, off);
        o[h][e] = make_float2(o[h][e].x * a + ox * c, o[h][e].y * a + oy * c);
      }
      m[h] = mn;
    }
  }

  // One record per slot that still holds a distinct part: slots below
  // min(H_kv, P) of every warp.  The records reuse the ring's memory.
  __syncthreads();
  float* rec = reinterpret_cast<float*>(dsm);  // [STEP][G][DH + 2]
  const int held = Hkv < P ? Hkv : P;
  if (slot < held) {
    float* rt = rec + t * REC;
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        rt[h * (DH + 2) + col + 2 * e] = o[h][e].x;
        rt[h * (DH + 2) + col + 2 * e + 1] = o[h][e].y;
      }
      if (col == 0) {
        rt[h * (DH + 2) + DH] = m[h];
        rt[h * (DH + 2) + DH + 1] = l[h];
      }
    }
  }
  __syncthreads();

  // Holders of head kvh: slot kvh of every warp (H_kv <= P), or the slots
  // kvh, kvh + H_kv, ... (H_kv > P).
  const int n_hold = Hkv <= P ? kDecodeThreads / 32 : STEP / Hkv;
  for (int i = tid; i < Hkv * REC; i += kDecodeThreads) {
    const int hk = i / REC, rem = i % REC, h = rem / (DH + 2), c = rem % (DH + 2);
    auto holder = [&](int k) { return Hkv <= P ? k * P + hk : hk + k * Hkv; };
    float M = -INFINITY;
    for (int k = 0; k < n_hold; ++k) M = fmaxf(M, rec[holder(k) * REC + h * (DH + 2) + DH]);
    float val = M;
    if (c != DH) {
      val = 0.f;
      for (int k = 0; k < n_hold; ++k) {
        const float* rk = rec + holder(k) * REC + h * (DH + 2);
        const float w = rk[DH] == -INFINITY ? 0.f : dev::ex2(rk[DH] - M);
        val = fmaf(rk[c], w, val);
      }
    }
    p.part[((static_cast<size_t>(b) * Hkv + hk) * p.n_split + split) * REC + rem] = val;
  }
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core split path for groups of 5 to 16 query heads (MQA-like
// layouts).  There the g queries that share a cached row make the scores and
// P V a dense contraction (16 x dh by dh x keys, then 16 x keys by keys x dh)
// that the CUDA cores cannot finish while HBM delivers the row; one
// mma.sync.m16n8k16 (bf16 in, fp32 out) computes a 16-head by 8-key block.
// The g heads are the 16 rows of the A operand (rows past g are zero).
//
// One CTA of 4 warps per (range of positions, K/V head, batch entry); the
// range streams through a ring of chunks in shared memory (16-byte cp.async
// copies; 128 keys, or 64 at dh 128 so that two CTAs fit on an SM), each warp
// taking a quarter of a chunk (32 keys, 16 at dh 128) per step:
//   S = Q K^T (B fragments by ldmatrix from the K rows), online softmax on
//   the accumulator fragments (row r = lane / 4 and r + 8; the four lanes of a
//   row reduce with shuffles; the reference maximum is raised only when a
//   step's maximum exceeds it by more than 8, so O is rarely rescaled; keys
//   are masked only in the chunk where the range ends), P re-packed as the A
//   fragments of P V (the accumulator layout of two 8-key blocks is the A
//   layout of one 16-key step), O += P V (B fragments by ldmatrix.trans from
//   the V rows).
// At the end the four warps' (m, l, O) are merged in shared memory into the
// range's partial record, in the general path's format.
constexpr int kMmaThreads = 128, kMmaStages = 3;
__host__ __device__ constexpr bool mma_path(int g) { return g >= 5 && g <= 16; }
__host__ __device__ constexpr int mma_chunk(int dh) { return dh == 128 ? 64 : 128; }
__host__ __device__ constexpr size_t mma_smem_bytes(int dh) {
  return static_cast<size_t>(kMmaStages) * 2 * mma_chunk(dh) * dh * 2;  // the ring; the merge reuses it
}
// 16-byte piece j of cached row `row` in a chunk buffer: XOR-swizzled so that
// the eight rows one ldmatrix phase reads (same piece, consecutive rows) fall
// in eight different 16-byte bank groups.
template <int DH>
__device__ __forceinline__ int mma_piece(int row, int j) {
  constexpr int P = DH / 8;  // pieces per row
  if constexpr (P >= 8) {
    return row * P + (j ^ (row & 7));
  } else {
    constexpr int SH = P == 4 ? 1 : 2;  // rows per 128 bytes: 2 or 4
    return row * P + (j ^ ((row >> SH) & (P - 1)));
  }
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* smem_row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(dev::smem_u32(smem_row)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* smem_row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(dev::smem_u32(smem_row)));
}
// d (+)= a b, m16n8k16, bf16 operands, fp32 accumulators
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int DH>
__global__ void __launch_bounds__(kMmaThreads) sqa_decode_mma_kernel(const DecodeParams p) {
  constexpr int KS = DH / 16;   // 16-wide steps over dh (scores)
  constexpr int NB = DH / 8;    // 8-wide output column blocks
  constexpr int P = DH / 8;     // 16-byte pieces per cached row
  constexpr int CH = mma_chunk(DH);
  constexpr int KW = CH / 4;    // keys per warp per chunk: 32, or 16 at dh 128
  constexpr int NKB = KW / 8;   // 8-key blocks of a warp's scores
  constexpr int CHUNK_BYTES = CH * DH * 2;
  constexpr int PIECES = CH * P / kMmaThreads;  // pieces of K (and of V) each thread copies per chunk
  static_assert(CH * P % kMmaThreads == 0 && NKB % 2 == 0, "chunk shape");
  const int split = blockIdx.x / p.Hkv, kvh = blockIdx.x % p.Hkv, b = blockIdx.y;
  const int bk = b * p.Hkv + kvh, g = p.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, c = lane & 3;  // fragment row (and row + 8) and column pair
  const int len = decode_len(p, b);
  const int r0 = split * p.span, r1 = min(len, r0 + p.span);
  float* part = p.part + (static_cast<size_t>(bk) * p.n_split + split) * g * (DH + 2);
  if (r1 <= r0) {  // range past this sequence's length: an empty partial
    for (int i = tid; i < g * (DH + 2); i += kMmaThreads) part[i] = i % (DH + 2) == DH ? -INFINITY : 0.f;
    return;
  }
  extern __shared__ __align__(128) uint8_t msm[];
  const int n_chunks = (r1 - r0 + CH - 1) / CH;
  const size_t pos_stride = static_cast<size_t>(p.Hkv) * DH;  // elements between cached positions
  const __nv_bfloat16* kg = p.k + (static_cast<size_t>(b) * p.N * p.Hkv + kvh) * DH;
  const __nv_bfloat16* vg = p.v + (static_cast<size_t>(b) * p.N * p.Hkv + kvh) * DH;
  // This thread's pieces (the same in every chunk): piece i = tid + k * threads
  // is row i / P, 16-byte piece i % P; its place in a chunk buffer and its
  // offset from the chunk's first cached row.
  uint32_t poff[PIECES];
  size_t goff[PIECES];
#pragma unroll
  for (int k = 0; k < PIECES; ++k) {
    const int i = tid + k * kMmaThreads, row = i / P, j = i % P;
    poff[k] = mma_piece<DH>(row, j) * 16;
    goff[k] = row * pos_stride + j * 8;
  }
  // chunk ci -> ring stage ci % kMmaStages: K rows at stage * 2 CHUNK_BYTES, V rows after them
  auto load_chunk = [&](int ci) {
    uint8_t* st = msm + (ci % kMmaStages) * 2 * CHUNK_BYTES;
    const int base = r0 + ci * CH;
    if (base + CH <= len) {
#pragma unroll
      for (int k = 0; k < PIECES; ++k) {
        const size_t go = base * pos_stride + goff[k];
        cp_async16(st + poff[k], kg + go);
        cp_async16(st + CHUNK_BYTES + poff[k], vg + go);
      }
    } else {  // the sequence ends in this chunk: rows past it repeat the last one (masked below)
#pragma unroll
      for (int k = 0; k < PIECES; ++k) {
        const int i = tid + k * kMmaThreads, row = i / P, j = i % P;
        const size_t go = static_cast<size_t>(min(base + row, len - 1)) * pos_stride + j * 8;
        cp_async16(st + poff[k], kg + go);
        cp_async16(st + CHUNK_BYTES + poff[k], vg + go);
      }
    }
  };
  for (int ci = 0; ci < kMmaStages - 1; ++ci) {
    if (ci < n_chunks) load_chunk(ci);
    cp_async_commit();
  }
  // A fragments of the queries, one per 16-wide dh step: rows r and r + 8 are
  // heads of the group (zero past g).
  uint32_t qa[KS][4];
  {
    const __nv_bfloat16* qh = p.q + (static_cast<size_t>(b) * p.Hq + kvh * g) * DH;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int k0 = ks * 16 + 2 * c;
      auto ld = [&](int row, int col) -> uint32_t {
        return row < g ? *reinterpret_cast<const uint32_t*>(qh + row * DH + col) : 0u;
      };
      qa[ks][0] = ld(r, k0);
      qa[ks][1] = ld(r + 8, k0);
      qa[ks][2] = ld(r, k0 + 8);
      qa[ks][3] = ld(r + 8, k0 + 8);
    }
  }
  const float sl2 = p.scale_log2;
  // Running reference maxima m (log2 units, rows r and r + 8), raised only when
  // a step's maximum exceeds them by more than 8 (P <= 256), and per-lane
  // partial sums l of 2^(s - m) over this lane's columns.
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;

  for (int ci = 0; ci < n_chunks; ++ci) {
    if (ci + kMmaStages - 1 < n_chunks) load_chunk(ci + kMmaStages - 1);
    cp_async_commit();
    cp_async_wait<kMmaStages - 1>();
    __syncthreads();
    const uint8_t* ks_base = msm + (ci % kMmaStages) * 2 * CHUNK_BYTES;
    const uint8_t* vs_base = ks_base + CHUNK_BYTES;
    const int chunk_pos = r0 + ci * CH;
    const int key0 = warp * KW;  // this warp's first key in the chunk
    // S for the warp's KW keys: NKB blocks of 8
    float s[NKB][4];
#pragma unroll
    for (int nb = 0; nb < NKB; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int h = 0; h < NKB / 2; ++h) {
        uint32_t kb[4];
        // lanes 0-7: keys 16 h + 0..7 at dh 16 ks; 8-15: same keys at 16 ks + 8;
        // 16-23 / 24-31: keys 16 h + 8..15
        const int krow = key0 + 16 * h + (lane & 7) + ((lane >> 4) << 3);
        ldmatrix_x4(kb, ks_base + mma_piece<DH>(krow, 2 * ks + ((lane >> 3) & 1)) * 16);
        mma16816(s[2 * h], qa[ks], kb[0], kb[1]);
        mma16816(s[2 * h + 1], qa[ks], kb[2], kb[3]);
      }
    }
    if (chunk_pos + CH > r1) {  // the range ends in this chunk: keys past it get -inf
#pragma unroll
      for (int nb = 0; nb < NKB; ++nb) {
        const int kp = chunk_pos + key0 + 8 * nb + 2 * c;  // key of s[nb][0] and s[nb][2]
        if (kp >= r1) s[nb][0] = s[nb][2] = -INFINITY;
        if (kp + 1 >= r1) s[nb][1] = s[nb][3] = -INFINITY;
      }
    }
    // Row maxima of the raw scores (the scale is positive), over the row's four lanes.
    float mx0 = fmaxf(s[0][0], s[0][1]), mx1 = fmaxf(s[0][2], s[0][3]);
#pragma unroll
    for (int nb = 1; nb < NKB; ++nb) {
      mx0 = dev::fmax3(mx0, s[nb][0], s[nb][1]);
      mx1 = dev::fmax3(mx1, s[nb][2], s[nb][3]);
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float t0 = mx0 * sl2, t1 = mx1 * sl2;
    const bool up0 = t0 > m0 + 8.f, up1 = t1 > m1 + 8.f;
    if (__any_sync(0xffffffffu, up0 || up1)) {
      const float a0 = (up0 && m0 != -INFINITY) ? dev::ex2(m0 - t0) : 1.f;
      const float a1 = (up1 && m1 != -INFINITY) ? dev::ex2(m1 - t1) : 1.f;
      if (up0) m0 = t0;
      if (up1) m1 = t1;
      l0 *= a0;
      l1 *= a1;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        o[nb][0] *= a0;
        o[nb][1] *= a0;
        o[nb][2] *= a1;
        o[nb][3] *= a1;
      }
    }
    // P = 2^(s sl2 - m); rows with no key seen yet (m = -inf) have only -inf scores.
    const float nm0 = m0 == -INFINITY ? 0.f : -m0, nm1 = m1 == -INFINITY ? 0.f : -m1;
    uint32_t pa[NKB / 2][4];
#pragma unroll
    for (int nb = 0; nb < NKB; ++nb) {
      const float p0 = dev::ex2(fmaf(s[nb][0], sl2, nm0)), p1 = dev::ex2(fmaf(s[nb][1], sl2, nm0));
      const float p2 = dev::ex2(fmaf(s[nb][2], sl2, nm1)), p3 = dev::ex2(fmaf(s[nb][3], sl2, nm1));
      l0 += p0 + p1;
      l1 += p2 + p3;
      // the accumulator layout of 8-key blocks 2 h and 2 h + 1 is the A layout
      // of 16-key step h: keys 0-7 in registers 0 / 1, keys 8-15 in 2 / 3
      pa[nb >> 1][(nb & 1) * 2 + 0] = dev::pack_bf16x2(p0, p1);
      pa[nb >> 1][(nb & 1) * 2 + 1] = dev::pack_bf16x2(p2, p3);
    }
#pragma unroll
    for (int h = 0; h < NKB / 2; ++h) {
#pragma unroll
      for (int nb = 0; nb < NB; nb += 2) {
        uint32_t vb[4];
        // lanes 0-7: keys 16 h + 0..7 at dh 8 nb; 8-15: keys 16 h + 8..15 at 8 nb;
        // 16-23 / 24-31: the same at dh 8 (nb + 1)
        const int vrow = key0 + 16 * h + (lane & 7) + (((lane >> 3) & 1) << 3);
        ldmatrix_x4_trans(vb, vs_base + mma_piece<DH>(vrow, nb + (lane >> 4)) * 16);
        mma16816(o[nb], pa[h], vb[0], vb[1]);
        mma16816(o[nb + 1], pa[h], vb[2], vb[3]);
      }
    }
    __syncthreads();  // the stage is reloaded next
  }
  cp_async_wait<0>();
  // Row sums over the row's four lanes.
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  // Merge the four warps: M = max of their references m, each O and l scaled by 2^(m - M).
  __syncthreads();
  float* ms = reinterpret_cast<float*>(msm);  // [4 warps][16 rows]
  float* ls = ms + 4 * 16;
  float* os = ls + 4 * 16;                    // [4 warps][16 rows][DH]
  if (c == 0) {
    ms[warp * 16 + r] = m0;
    ms[warp * 16 + r + 8] = m1;
  }
  __syncthreads();
  float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    M0 = fmaxf(M0, ms[w * 16 + r]);
    M1 = fmaxf(M1, ms[w * 16 + r + 8]);
  }
  const float f0 = m0 == -INFINITY ? 0.f : dev::ex2(m0 - M0), f1 = m1 == -INFINITY ? 0.f : dev::ex2(m1 - M1);
  if (c == 0) {
    ls[warp * 16 + r] = l0 * f0;
    ls[warp * 16 + r + 8] = l1 * f1;
  }
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int col = nb * 8 + 2 * c;
    os[(warp * 16 + r) * DH + col] = o[nb][0] * f0;
    os[(warp * 16 + r) * DH + col + 1] = o[nb][1] * f0;
    os[(warp * 16 + r + 8) * DH + col] = o[nb][2] * f1;
    os[(warp * 16 + r + 8) * DH + col + 1] = o[nb][3] * f1;
  }
  __syncthreads();
  for (int i = tid; i < g * (DH + 2); i += kMmaThreads) {
    const int h = i / (DH + 2), col = i % (DH + 2);
    float v;
    if (col < DH) {
      v = os[h * DH + col] + os[(16 + h) * DH + col] + os[(32 + h) * DH + col] + os[(48 + h) * DH + col];
    } else if (col == DH) {
      v = fmaxf(fmaxf(ms[h], ms[16 + h]), fmaxf(ms[32 + h], ms[48 + h]));
    } else {
      v = ls[h] + ls[16 + h] + ls[32 + h] + ls[48 + h];
    }
    part[i] = v;
  }
}

template <int DH, int G>
__global__ void __launch_bounds__(kDecodeThreads, G == 0 ? 1 : 2) sqa_decode_split_kernel(const DecodeParams p) {
  if constexpr (G == 0) {
    decode_split_general<DH>(p);
  } else {
    decode_split_rows<DH, G>(p);
  }
}

template <int DH>
__global__ void __launch_bounds__(kDecodeThreads) sqa_decode_combine_kernel(const DecodeParams p) {
  constexpr int DP = DH / 2, SL = kDecodeThreads / DP;  // column pairs; ranges handled side by side
  constexpr int NW = kDecodeThreads / 32;
  const int bh = blockIdx.x;                              // (batch entry, query head)
  const int b = bh / p.Hq, h = bh % p.Hq, kvh = h / p.g, hg = h % p.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, dp = tid % DP, sl = tid / DP;
  const size_t stride = static_cast<size_t>(p.g) * (DH + 2);
  const float* part =
      p.part + static_cast<size_t>(b * p.Hkv + kvh) * p.n_split * stride + static_cast<size_t>(hg) * (DH + 2);
  const int n_used = (decode_len(p, b) + p.span - 1) / p.span;
  __shared__ float2 red[kDecodeThreads];
  __shared__ float wred[NW];

  // M = largest range maximum (warp shuffles, then one value per warp).
  float m = -INFINITY;
  for (int s = tid; s < n_used; s += kDecodeThreads) m = fmaxf(m, part[s * stride + DH]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) wred[warp] = m;
  __syncthreads();
  float M = wred[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, wred[w]);

  // Columns 2 dp, 2 dp + 1 over the ranges sl, sl + SL, ..., several loads in
  // flight; the dp = 0 threads also sum L.
  float2 acc = make_float2(0.f, 0.f);
  float L = 0.f;
#pragma unroll 4
  for (int s = sl; s < n_used; s += SL) {
    const float* ps = part + s * stride;
    const float w = dev::ex2(ps[DH] - M);
    const float2 o2 = *reinterpret_cast<const float2*>(ps + 2 * dp);
    acc.x = fmaf(o2.x, w, acc.x);
    acc.y = fmaf(o2.y, w, acc.y);
    if (dp == 0) L = fmaf(ps[DH + 1], w, L);
  }
  red[tid] = acc;
  __syncthreads();
  if (sl == 0) {
    for (int k = 1; k < SL; ++k) {
      const float2 r = red[k * DP + dp];
      acc.x += r.x;
      acc.y += r.y;
    }
  }
  __syncthreads();
  if (dp == 0) red[sl] = make_float2(L, 0.f);
  __syncthreads();
  if (sl == 0) {
    L = red[0].x;
    for (int k = 1; k < SL; ++k) L += red[k].x;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* ob = p.out + static_cast<size_t>(bh) * DH + 2 * dp;  // out may be only 2-byte aligned
    ob[0] = __float2bfloat16_rn(acc.x * inv);
    ob[1] = __float2bfloat16_rn(acc.y * inv);
    if (dp == 0) p.lse[bh] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace sqa

// sqa_fwd.cuh -- Sparse Query Attention forward on sm_100a.
//
// Work item: one key/value head of one batch entry and two Q tiles.  A Q tile
// stacks the g = H_q / H_kv query heads that share the key/value head: its 128
// MMA rows are (token, head) pairs, row r = t * g + head, which is exactly how
// [B][N][H_q][dh] stores the group's heads side by side, so one TMA box
// {dh, g, T} fills it.  Every K/V tile is therefore loaded once per KV head and
// used by all heads of its group (GQA summary, "The idea": a group shares one key
// head and one value head; arXiv 2510.01817 abstract: score FLOPs scale with H_q).
//
// The kernel is persistent: one CTA per SM walks a list of work items, heaviest
// first, so the loads and the first QK^T of the next item overlap the end of
// the current one.  The K/V ring and every barrier phase run on across items.
//
// Roles (384 threads):
//   warps 0-3   softmax for Q tile 0; warps 4-7 softmax for Q tile 1 (a warp
//               reaches TMEM lanes 32*(warp%4) .. +31, so each warpgroup covers
//               the 128 rows of its tile), plus the O / lse epilogue
//   warp 8      TMA producer: Q tiles per item, 64-key K/V tiles through a ring
//   warps 9-10  MMA issuers, one thread each, for Q tiles 0 and 1 (warp 9 also
//               allocates TMEM); warp 11 idle
//                 S_t = Q_t K_j^T  (tcgen05, both operands K-major in smem)
//                 O_t += P_t V_j   (tcgen05, P from TMEM, V MN-major in smem)
// TMEM (512 columns): S_t has two 64-column buffers at 128 t + 64 (step % 2), so
// the tensor core computes S_t for the next key tile while the softmax warps work
// on the current one; O_t sits at 256 + 128 t.  P_t (bf16 pairs) overwrites the
// first 32 columns of its S buffer.
//
// With one S buffer per tile (dh 128) a tile's next S = Q K^T can only start
// after its P V, so each tile alternates between softmax and MMAs.  The two
// tiles' softmax warpgroups take turns for the exponentials (a token passed
// through two mbarriers): while one warpgroup works on the special-function
// unit, the other tile's P V and next S run on the tensor core.  Left to
// themselves the two tiles fall into step, share the special-function unit and
// then queue their MMAs together, and each unit idles while the other works.
//
// Online softmax (exact): each row keeps a reference maximum m (log2 units) and
// l = sum 2^(s*scale*log2e - m).  m is raised only when a tile's maximum exceeds
// it by more than 8, so P <= 256 and O is rescaled rarely; the final O / l and
// lse = ln2 * (m + log2 l) do not depend on which reference was used.
#pragma once

#include "sqa_device.cuh"
#include "sqa_tmem_wide.cuh"

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
  int n_items;   // n_pairs * n_bh
  int causal;
  int split;         // 1: both tile slots of a CTA work on one Q tile, even / odd key tiles
  float scale_log2;  // scale * log2(e)
  // Split mode with a workspace (chunk > 0): a work item is a range of at most
  // `chunk` key tiles of one Q tile; items of a Q tile with several ranges
  // leave partial results, and the last of them to finish merges them.
  int chunk;
  int nch_max;    // ranges of the longest Q tile (layout of the partials)
  float* part;    // [n_bh][n_qtiles][nch_max][128][dh] outputs normalised within their range
  float* part_l;  // [n_bh][n_qtiles][nch_max][128] log2 of each range's sum of exponentials (log2 units)
  int* cnt;       // [n_bh][n_qtiles][128] ranges finished per row (zero before the launch)
};

template <int DH>
struct FwdTraits {
  static constexpr int BM = 128;  // stacked rows per Q tile
  // Keys per K/V tile.  At dh = 128 a tile of 128 keys makes S = Q K^T an
  // N = 128 MMA, which reads its operands from shared memory no faster than it
  // computes (at N = 64 the reads take longer than the math); the 128 columns
  // of a tile's S region then hold one S buffer instead of two.
  static constexpr int NK = DH == 128 ? 128 : 64;
  static constexpr int NSBUF = NK == 128 ? 1 : 2;  // S buffers per Q tile
  static constexpr int PANEL = DH < 64 ? DH : 64;  // elements per swizzled row segment
  static constexpr int NPANEL = DH / PANEL;
  static constexpr int ROWB = PANEL * 2;  // bytes per row segment
  static constexpr uint32_t LAYOUT = ROWB == 32 ? 6u : (ROWB == 64 ? 4u : 2u);
  static constexpr int Q_BYTES = BM * DH * 2;
  static constexpr int KV_BYTES = NK * DH * 2;
  static constexpr int QBUF = DH <= 64 ? 2 : 1;  // Q-tile pairs in flight
  static constexpr int STAGES = DH <= 32 ? 8 : (DH == 64 ? 4 : (NK == 128 ? 2 : 3));
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBUF * 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
  // q_full[QB] | q_empty[QB] | kv_full[S] | kv_empty[S] | s_full[2][2] | p_full[2][2] |
  // o_done[2] | o_final[2] | o_free[2] | drain[2] | split_ready | split_done | turn[2]
  static constexpr int N_BARS = 2 * QBUF + 2 * STAGES + 4 + 4 + 2 + 2 + 2 + 2 + 2 + 2;
  // The softmax warpgroups take turns for the exponentials (one S buffer per tile).
  static constexpr bool TOKEN = NSBUF == 1;
  // With one Q buffer a slot cannot start the next item before the other slot
  // has passed its last turn of this one (each thread arrives on turn(t) before
  // p_full, and the Q buffer is released after the last P V), so a slot that
  // skips the other's last turns of an item (an item with one Q tile, or the
  // other tile's extra causal step) finds those phases completed: a parity wait
  // neither passes on a phase still open nor on one two ahead.  With two Q
  // buffers a slot could run a whole item ahead and alias their phases.
  static_assert(!TOKEN || QBUF == 1, "turns need one Q buffer");
  // split mode: slot 1's running maximum and sum per row, for slot 0's combine
  static constexpr int OFF_ML = OFF_BAR + N_BARS * 8 + 16;
  static constexpr int SMEM_USED = OFF_ML + 2 * BM * 4;
  // Ask for enough shared memory that only one CTA fits per SM (each CTA holds
  // all 512 TMEM columns), plus slack to align the base to 1024 bytes.
  static constexpr int SMEM_BYTES = (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) + 1024;
  __host__ __device__ static constexpr uint32_t tm_s(int t, int buf) { return 128u * t + 64u * buf; }
  __host__ __device__ static constexpr uint32_t tm_o(int t) { return 256u + 128u * t; }
  static constexpr int THREADS = 384;
  static constexpr int WARP_PRODUCER = 8, WARP_MMA = 9;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(DH % 16 == 0 && DH <= 128, "head dim");
};

__device__ __forceinline__ int fwd_item(int r, int n_items) { return dev::snake_item(r, n_items); }

struct FwdItem {
  int b, kvh, qt0, nkv0, nkv1, nkv;
  bool has1;
  int kt0;  // first key tile (split mode with ranges; 0 otherwise)
  int c;    // range index and number of ranges of the Q tile (1: no partials)
  int nch;
};

// Key tiles a Q tile needs: all of them, or under a causal mask those up to its last token.
__device__ __forceinline__ int fwd_nkv(const FwdParams& p, int qt, int NK) {
  const int end = p.causal ? min(p.N, (qt + 1) * p.T) : p.N;
  return (end + NK - 1) / NK;
}

template <bool SPLIT>
__device__ __forceinline__ FwdItem fwd_decode(const FwdParams& p, int item, int NK) {
  FwdItem it;
  const int bh = item % p.n_bh;
  it.b = bh / p.Hkv;
  it.kvh = bh % p.Hkv;
  it.kt0 = 0;
  it.c = 0;
  it.nch = 1;
  if (SPLIT) {
    // One Q tile (or, with ranges, up to `chunk` of its key tiles); slot 0
    // takes the even key tiles, slot 1 the odd ones.  Latest tokens (heaviest
    // under a causal mask) first.
    int k = item / p.n_bh;
    int qt = p.n_qtiles - 1;
    if (p.chunk > 0) {
      // the k-th range of this (batch, KV head): Q tiles from the last, ranges in key order
      int nkv = fwd_nkv(p, qt, NK), nch = (nkv + p.chunk - 1) / p.chunk;
      while (k >= nch && qt > 0) {
        k -= nch;
        --qt;
        nkv = fwd_nkv(p, qt, NK);
        nch = (nkv + p.chunk - 1) / p.chunk;
      }
      it.c = k;
      it.nch = nch;
      it.kt0 = k * p.chunk;
      it.nkv = max(0, min(nkv - it.kt0, p.chunk));
    } else {
      qt -= k;
      it.nkv = fwd_nkv(p, qt, NK);
    }
    it.qt0 = qt;
    it.nkv0 = (it.nkv + 1) / 2;
    it.nkv1 = it.nkv / 2;
    it.has1 = false;  // one Q tile to load
    return it;
  }
  const int pair = p.n_pairs - 1 - item / p.n_bh;  // latest tokens (heaviest under a causal mask) first
  it.qt0 = 2 * pair;
  it.has1 = it.qt0 + 1 < p.n_qtiles;
  const int end0 = p.causal ? min(p.N, (it.qt0 + 1) * p.T) : p.N;
  const int end1 = p.causal ? min(p.N, (it.qt0 + 2) * p.T) : p.N;
  it.nkv0 = (end0 + NK - 1) / NK;
  it.nkv1 = it.has1 ? (end1 + NK - 1) / NK : 0;
  it.nkv = max(it.nkv0, it.nkv1);
  return it;
}

// One row's result of a Q tile whose keys were split into nch ranges over
// several CTAs.  Each range leaves its output normalised within the range and
// its log2-sum-exp L_c; the row's counter in the workspace counts the ranges
// written, and the thread that completes it (seeing every other range's
// stores: each writer fences before its increment) merges them:
//   O = sum_c 2^(L_c - M) O_c / W,  W = sum_c 2^(L_c - M),  M = max_c L_c,
//   lse = ln 2 (M + log2 W),
// in one pass with a running maximum (range 0 always holds key 0, so its L_0
// is finite for every valid row), four ranges' loads in flight at a time.
// No thread waits for another CTA, so there is nothing to time out.
template <int DH>
__device__ __noinline__ void fwd_merge_ranges(const FwdParams& p, size_t slot_base, int c, int nch, int row,
                                              int* counter, float l2_own, __nv_bfloat16* dst, float* lse_dst) {
  using namespace dev;
  constexpr int BM = 128;
  p.part_l[(slot_base + c) * BM + row] = l2_own;
  __threadfence();
  if (atomicAdd(counter, 1) + 1 != nch) return;
  __threadfence();
  float acc[DH];
  const float* y0 = p.part + (slot_base * BM + row) * DH;
#pragma unroll
  for (int i = 0; i < DH; i += 4) {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(y0 + i));
    acc[i] = a.x;
    acc[i + 1] = a.y;
    acc[i + 2] = a.z;
    acc[i + 3] = a.w;
  }
  float M = __ldcg(p.part_l + slot_base * BM + row), W = 1.f;
#pragma unroll 4
  for (int cc = 1; cc < nch; ++cc) {
    const float L = __ldcg(p.part_l + (slot_base + cc) * BM + row);
    const float* y = p.part + ((slot_base + cc) * BM + row) * DH;
    const float Mn = fmaxf(M, L);
    const float a = ex2(M - Mn), b = ex2(L - Mn);  // L = -inf (no visible key in the range): b = 0
    W = fmaf(W, a, b);
#pragma unroll
    for (int i = 0; i < DH; i += 4) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(y + i));
      acc[i] = fmaf(acc[i], a, v.x * b);
      acc[i + 1] = fmaf(acc[i + 1], a, v.y * b);
      acc[i + 2] = fmaf(acc[i + 2], a, v.z * b);
      acc[i + 3] = fmaf(acc[i + 3], a, v.w * b);
    }
    M = Mn;
  }
  const float inv_w = 1.f / W;
#pragma unroll
  for (int col = 0; col < DH; col += 8) {
    uint4 o;
    o.x = pack_bf16x2(acc[col] * inv_w, acc[col + 1] * inv_w);
    o.y = pack_bf16x2(acc[col + 2] * inv_w, acc[col + 3] * inv_w);
    o.z = pack_bf16x2(acc[col + 4] * inv_w, acc[col + 5] * inv_w);
    o.w = pack_bf16x2(acc[col + 6] * inv_w, acc[col + 7] * inv_w);
    *reinterpret_cast<uint4*>(dst + col) = o;
  }
  *lse_dst = (M + __log2f(W)) * 0.69314718055994531f;
}

// SPLIT: split mode (FwdParams::split), compiled separately so that the
// ordinary kernel carries none of its code.  POLY: of every 8 pairs of scores
// in an unmasked tile, how many take the polynomial exponential (exp2_poly2)
// instead of the special-function unit.
template <int DH, bool SPLIT, int POLY = (DH <= 32 ? 2 : 0)>
__global__ void __launch_bounds__(384, 1)
    sqa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using Tr = FwdTraits<DH>;
  using namespace dev;
  constexpr int BM = Tr::BM, NK = Tr::NK, ROWB = Tr::ROWB, PANEL = Tr::PANEL, ST = Tr::STAGES, QB = Tr::QBUF;
  constexpr int NSB = Tr::NSBUF;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar0 = sbase + Tr::OFF_BAR;
  auto q_full = [&](int qb) { return bar0 + 8u * qb; };
  auto q_empty = [&](int qb) { return bar0 + 8u * (QB + qb); };
  auto kv_full = [&](int s) { return bar0 + 8u * (2 * QB + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (2 * QB + ST + s); };
  auto s_full = [&](int t, int buf) { return bar0 + 8u * (2 * QB + 2 * ST + 2 * t + buf); };
  // P of S step G is announced on the barrier of its S buffer (G % 2): with two
  // S buffers a softmax warpgroup can finish two steps before the MMA issuer
  // looks, and one barrier per buffer keeps each at most one phase ahead.
  auto p_full = [&](int t, int buf) { return bar0 + 8u * (2 * QB + 2 * ST + 4 + 2 * t + buf); };
  auto o_done = [&](int t) { return bar0 + 8u * (2 * QB + 2 * ST + 8 + t); };
  auto o_final = [&](int t) { return bar0 + 8u * (2 * QB + 2 * ST + 10 + t); };
  auto o_free = [&](int t) { return bar0 + 8u * (2 * QB + 2 * ST + 12 + t); };
  auto drain = [&](int t) { return bar0 + 8u * (2 * QB + 2 * ST + 14 + t); };
  const uint32_t split_ready = bar0 + 8u * (2 * QB + 2 * ST + 16);  // slot 1's O, m, l are final
  const uint32_t split_done = bar0 + 8u * (2 * QB + 2 * ST + 17);   // slot 0 has read them
  // turn(t): the softmax warpgroup of slot t finished the exponentials of a step
  auto turn = [&](int t) { return bar0 + 8u * (2 * QB + 2 * ST + 18 + t); };
  float* sm_m = reinterpret_cast<float*>(smem + Tr::OFF_ML);
  float* sm_l = sm_m + BM;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_BAR + Tr::N_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int qb = 0; qb < QB; ++qb) {
      mbar_init(q_full(qb), 1);
      mbar_init(q_empty(qb), 2);  // one release per MMA issuer
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 2);  // one release per MMA issuer
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t, 0), 1);
      mbar_init(s_full(t, 1), 1);
      mbar_init(p_full(t, 0), 128);
      mbar_init(p_full(t, 1), 128);
      mbar_init(o_done(t), 1);
      mbar_init(o_final(t), 1);
      mbar_init(o_free(t), 128);
    }
    mbar_init(drain(0), 1);
    mbar_init(drain(1), 1);
    mbar_init(split_ready, 128);
    mbar_init(split_done, 128);
    mbar_init(turn(0), 128);
    mbar_init(turn(1), 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Rows of a Q tile that the TMA box does not cover (when g does not divide
  // 128) stay zero, so their scores are finite; they are never stored.
  if (p.rows < BM) {
    const int pad_bytes = (BM - p.rows) * ROWB;
    for (int t = 0; t < 2 * QB; ++t)
      for (int pn = 0; pn < Tr::NPANEL; ++pn) {
        uint8_t* base = smem + Tr::OFF_Q + t * Tr::Q_BYTES + pn * BM * ROWB + p.rows * ROWB;
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
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      const uint32_t q_bytes = static_cast<uint32_t>(p.rows * ROWB * Tr::NPANEL);
      int g = 0;  // K/V tiles issued so far (across items)
      bool ok = true;
      for (int r = 0, item; ok && (item = fwd_item(r, p.n_items)) >= 0; ++r) {
        const FwdItem it = fwd_decode<SPLIT>(p, item, NK);
        const int qb = r % QB;
        if (r >= QB && !mbar_wait(q_empty(qb), ((r / QB) - 1) & 1, abort_flag, kSiteProducer)) break;
        mbar_expect_tx(q_full(qb), q_bytes * (it.has1 ? 2u : 1u));
        for (int t = 0; t < (it.has1 ? 2 : 1); ++t)
          for (int pn = 0; pn < Tr::NPANEL; ++pn)
            tma_load_4d(sbase + Tr::OFF_Q + (qb * 2 + t) * Tr::Q_BYTES + pn * BM * ROWB, &tmQ, q_full(qb),
                        pn * PANEL, it.kvh * p.g, (it.qt0 + t) * p.T, it.b);
        for (int j = 0; j < it.nkv; ++j, ++g) {
          const int s = g % ST;
          if (g >= ST && !mbar_wait(kv_empty(s), ((g / ST) - 1) & 1, abort_flag, kSiteProducer)) {
            ok = false;
            break;
          }
          mbar_expect_tx(kv_full(s), 2u * Tr::KV_BYTES);
          for (int pn = 0; pn < Tr::NPANEL; ++pn) {
            tma_load_4d(sbase + Tr::OFF_K + s * Tr::KV_BYTES + pn * NK * ROWB, &tmK, kv_full(s), pn * PANEL,
                        it.kvh, (it.kt0 + j) * NK, it.b);
            tma_load_4d(sbase + Tr::OFF_V + s * Tr::KV_BYTES + pn * NK * ROWB, &tmV, kv_full(s), pn * PANEL,
                        it.kvh, (it.kt0 + j) * NK, it.b);
          }
        }
      }
      if (*abort_flag) {  // let in-flight copies land before the CTA exits
        for (int j = max(0, g - ST); j < g; ++j) mbar_wait_drain(kv_full(j % ST), (j / ST) & 1);
      }
    }
  } else if (warp == Tr::WARP_MMA || warp == Tr::WARP_MMA + 1) {
    // ------------------------------------------------------------ MMA issuers, one warp per Q tile
    // A single issuing warp shares its sub-partition with busy softmax warps and
    // could not keep two tiles fed; two issuers also let the tiles run apart.
    // The whole warp runs the loop and one elected lane issues each MMA.
    const int t = warp - Tr::WARP_MMA;
    constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, NK, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, DH, false, true);
    // Descriptors of Q buffer 0 / stage 0; other buffers, stages and K-steps add
    // their byte offset (in 16-byte units) to the start-address field.
    // (In split mode both slots read the one Q tile, in slot 0's buffer.)
    const uint64_t dq0 = smem_desc(sbase + Tr::OFF_Q + (SPLIT ? 0 : t) * Tr::Q_BYTES, 16, 8 * ROWB, Tr::LAYOUT);
    const uint64_t dk0 = smem_desc(sbase + Tr::OFF_K, 16, 8 * ROWB, Tr::LAYOUT);
    const uint64_t dv0 = smem_desc(sbase + Tr::OFF_V, NK * ROWB, 8 * ROWB, Tr::LAYOUT);
    const uint32_t tS0 = tmem + Tr::tm_s(t, 0), tO = tmem + Tr::tm_o(t);
    auto issue_qk = [&](int qb, int s, int buf) {
      const uint64_t a0 = dq0 + static_cast<uint64_t>((qb * 2 * Tr::Q_BYTES) >> 4);
      const uint64_t b0 = dk0 + static_cast<uint64_t>((s * Tr::KV_BYTES) >> 4);
#pragma unroll
      for (int ks = 0; ks < DH / 16; ++ks) {
        const uint32_t within = ((ks * 16) % PANEL) * 2, pn = (ks * 16) / PANEL;
        mma_ss_w(tS0 + 64u * buf, a0 + ((pn * BM * ROWB + within) >> 4), b0 + ((pn * NK * ROWB + within) >> 4),
                 idesc_qk, ks > 0 ? 1u : 0u);
      }
      mma_commit_w(s_full(t, buf));
    };
    auto issue_pv = [&](int s, int buf, bool acc) {
      const uint64_t b0 = dv0 + static_cast<uint64_t>((s * Tr::KV_BYTES) >> 4);
#pragma unroll
      for (int ks = 0; ks < NK / 16; ++ks)  // P of keys 16 ks .. + 15: column 64 (ks / 4) + 8 (ks % 4)
        mma_ts_w(tO, tS0 + 64u * buf + 64u * (ks >> 2) + 8u * (ks & 3), b0 + ((ks * 16 * ROWB) >> 4), idesc_pv,
                 (acc || ks > 0) ? 1u : 0u);
      mma_commit_w(o_done(t));
    };
    int loaded = 0;  // K/V tiles whose kv_full phase this warp has observed
    int g = 0;       // first K/V tile (global index) of the current item
    // In split mode a slot releases the other slot's key tiles as soon as it
    // has observed them loaded.
    auto ensure_loaded = [&](int gj) {
      while (loaded <= gj) {
        if (!mbar_wait_warp(kv_full(loaded % ST), (loaded / ST) & 1, abort_flag, kSiteMma)) return false;
        if (SPLIT && ((loaded - g) & 1) != t) mma_commit_w(kv_empty(loaded % ST));
        ++loaded;
      }
      tc_fence_after();
      return true;
    };
    // item-relative index of this slot's j-th key tile
    auto own = [&](int j) { return SPLIT ? 2 * j + t : j; };
    int G = 0;   // S steps of this Q tile so far (across items)
    int nd = 0;  // items finished by this Q tile
    bool ok = true;
    for (int r = 0, item; ok && (item = fwd_item(r, p.n_items)) >= 0; ++r) {
      const FwdItem it = fwd_decode<SPLIT>(p, item, NK);
      const int nkv_t = t ? it.nkv1 : it.nkv0;
      const int qb = r % QB;
      // Both issuers observe this item's Q load before releasing its buffer, so a
      // release never lands in the phase of an earlier item.
      if (!mbar_wait_warp(q_full(qb), (r / QB) & 1, abort_flag, kSiteMma)) {
        ok = false;
        break;
      }
      for (int j = 0; ok && j < NSB && j < nkv_t; ++j) {  // prologue: S for the first key tiles
        ok = ensure_loaded(g + own(j));
        if (ok) issue_qk(qb, (g + own(j)) % ST, (G + j) % NSB);
      }
      for (int j = 0; ok && j < nkv_t; ++j) {
        const int Gt = G + j;
        if (!mbar_wait_warp(p_full(t, Gt % NSB), (Gt / NSB) & 1, abort_flag, kSiteMma)) {
          ok = false;
          break;
        }
        // O_t still holds the previous item until its epilogue has read it.
        if (j == 0 && nd > 0 && !mbar_wait_warp(o_free(t), (nd - 1) & 1, abort_flag, kSiteMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv((g + own(j)) % ST, Gt % NSB, j > 0);
        if (j + 1 == nkv_t) mma_commit_w(o_final(t));
        // The stage is released when the PV just issued has read V (a commit
        // covers every MMA issued before it), before waiting for a later one.
        mma_commit_w(kv_empty((g + own(j)) % ST));
        if (j + NSB < nkv_t) {
          // The next S in this buffer: the PV just issued reads P from it first
          // (MMAs from one issuer execute in order).
          if (!ensure_loaded(g + own(j + NSB))) {
            ok = false;
            break;
          }
          issue_qk(qb, (g + own(j + NSB)) % ST, Gt % NSB);
        }
      }
      if (SPLIT) {
        // the other slot's tiles after this slot's last one
        if (ok && it.nkv > 0) ok = ensure_loaded(g + it.nkv - 1);
      } else {
        // K/V tiles of this item that this Q tile does not need (causal: the other
        // tile reaches one tile further) are released too, once they are loaded.
        for (int j = nkv_t; ok && j < it.nkv; ++j) {
          ok = ensure_loaded(g + j);
          if (ok) mma_commit_w(kv_empty((g + j) % ST));
        }
      }
      if (!ok) break;
      mma_commit_w(q_empty(qb));
      G += nkv_t;
      nd += nkv_t > 0 ? 1 : 0;
      g += it.nkv;
    }
    if (!ok) {  // wait for issued MMAs before TMEM is released
      mma_commit_w(drain(t));
      mbar_wait_drain(drain(t), 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax and epilogue
    const int t = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t tO = lane_addr + Tr::tm_o(t);
    const float sl2 = p.scale_log2;
    int G = 0, nd = 0;
    int nc = 0;  // split mode: combines done (phases of split_ready / split_done)
    // Token order within an item: slot 0's step j follows slot 1's step j - 1,
    // slot 1's step j follows slot 0's step j, where the other slot has such a
    // step.  (Across items there is no order: the next item's Q tile may wait
    // for this item's last steps to release the Q buffer.)  Phases of turn(t)
    // count slot t's steps over all items; G_other is the other slot's count
    // before this item.
    int G_other = 0;
    bool ok = true;
    for (int r = 0, item; ok && (item = fwd_item(r, p.n_items)) >= 0; ++r) {
      const FwdItem it = fwd_decode<SPLIT>(p, item, NK);
      const int nkv_t = t ? it.nkv1 : it.nkv0;
      const int nkv_o = Tr::TOKEN ? (t ? it.nkv0 : it.nkv1) : 0;
      const int G_o = G_other;
      if constexpr (Tr::TOKEN) G_other += nkv_o;
      if (nkv_t == 0) continue;
      const int qt = SPLIT ? it.qt0 : it.qt0 + t;
      const bool combine = SPLIT && it.nkv1 > 0;  // slot 1 holds part of this row's sums
      const int tok = qt * p.T + row / p.g;
      const int head = it.kvh * p.g + row % p.g;
      const bool row_valid = row < p.rows && tok < p.N;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv_t; ++j) {
        const int Gt = G + j;
        // Every lane waits; the verdict is made warp-uniform so that the
        // warp-wide TMEM instructions below are never reached divergently.
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(t, Gt % NSB), (Gt / NSB) & 1, abort_flag, kSiteSoftmax));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = lane_addr + Tr::tm_s(t, Gt % NSB);
        const int k0 = (it.kt0 + (SPLIT ? 2 * j + t : j)) * NK;
        const bool masked = (k0 + NK > p.N) || (p.causal && k0 + NK - 1 > qt * p.T);
        // The tile's scores are handled 64 columns (a half at NK = 128) at a time.
        // last visible key of this tile, relative to k0 (may be negative)
        const int last = min(p.N - 1, p.causal ? tok : p.N - 1) - k0;
        uint32_t sr[64];
        auto load64 = [&](int h) {
          tmem_ld32x2(tS + 64 * h, tS + 64 * h + 32, sr);
          if (masked) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (i + 64 * h > last) sr[i] = __float_as_uint(-INFINITY);
          }
        };
        // Row maximum: eight independent chains of three-input maxima per half.
        auto max64 = [&]() {
          float acc[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            acc[c] = fmax3(__uint_as_float(sr[c]), __uint_as_float(sr[8 + c]), __uint_as_float(sr[16 + c]));
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            acc[c] = fmax3(acc[c], __uint_as_float(sr[24 + c]), __uint_as_float(sr[32 + c]));
            acc[c] = fmax3(acc[c], __uint_as_float(sr[40 + c]), __uint_as_float(sr[48 + c]));
            acc[c] = fmaxf(acc[c], __uint_as_float(sr[56 + c]));
          }
          return fmax3(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], acc[5]), fmaxf(acc[6], acc[7]));
        };
        float mx = -INFINITY;
#pragma unroll
        for (int h = 0; h < NK / 64; ++h) {
          load64(h);
          mx = fmaxf(mx, max64());
        }
        const float mnew = fmaxf(m, mx * sl2);
        const bool raise = mnew > m + 8.f;
        const float alpha = (raise && m != -INFINITY) ? ex2(m - mnew) : 1.f;
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          // O must hold P*V of every earlier step of this item before it is
          // rescaled: wait for the PV of step Gt - 1 (o_done is at most one phase
          // behind here; alpha is 1 at an item's first step).
          ok = __all_sync(0xffffffffu, mbar_wait(o_done(t), (Gt - 1) & 1, abort_flag, kSiteSoftmax));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < DH; c += 16) {
            uint32_t rr[16];
            tmem_ld16(tO + c, rr);
#pragma unroll
            for (int i = 0; i < 16; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
            tmem_st16(tO + c, rr);
          }
        }
        l *= alpha;
        if (raise) m = mnew;
        if constexpr (Tr::TOKEN) {
          const int k_other = t ? j : j - 1;  // the other slot's step of this item that goes first
          if (k_other >= 0 && k_other < nkv_o) {
            ok = __all_sync(0xffffffffu, mbar_wait(turn(1 - t), (G_o + k_other) & 1, abort_flag, kSiteSoftmax));
            if (!ok) break;
          }
        }
        // Masked scores are -inf, so their P is exactly 0 (the scale is positive).
        const float nref = m == -INFINITY ? 0.f : -m;
        float sum0[8], sum1[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) sum0[c] = sum1[c] = 0.f;
        // P (bf16 pairs) of the 64 keys of half h goes to columns 64 h .. 64 h + 31,
        // over scores already consumed.  At NK = 128 the second half is still in
        // registers from the maximum pass and goes first, then the first half is
        // loaded again.
#pragma unroll
        for (int hh = 0; hh < NK / 64; ++hh) {
          const int h = NK / 64 - 1 - hh;
          if (hh > 0) load64(h);
          uint32_t pk[32];
          if (!masked) {
            // POLY of every 8 pairs take the FMA-pipe exponential, the rest the
            // special-function unit, so that neither pipe alone sets the pace.
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float x0, x1, p0, p1;
              ffma2(x0, x1, __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]), sl2, sl2, nref, nref);
              if ((i & 7) * POLY % 8 + POLY >= 8) {  // POLY evenly spread indices of 0..7
                const float2 pp = exp2_poly2(x0, x1);
                p0 = pp.x;
                p1 = pp.y;
              } else {
                p0 = ex2(x0);
                p1 = ex2(x1);
              }
              fadd2(sum0[i & 7], sum1[i & 7], sum0[i & 7], sum1[i & 7], p0, p1);
              pk[i] = pack_bf16x2(p0, p1);
            }
          } else {
            // Masked scores are -inf: the special-function unit gives exactly 0 there.
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float x0, x1;
              ffma2(x0, x1, __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]), sl2, sl2, nref, nref);
              const float p0 = ex2(x0), p1 = ex2(x1);
              fadd2(sum0[i & 7], sum1[i & 7], sum0[i & 7], sum1[i & 7], p0, p1);
              pk[i] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st32(tS + 64 * h, pk);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) fadd2(sum0[c], sum1[c], sum0[c], sum1[c], sum0[c + 4], sum1[c + 4]);
        l += ((sum0[0] + sum1[0]) + (sum0[1] + sum1[1])) + ((sum0[2] + sum1[2]) + (sum0[3] + sum1[3]));
        tmem_wait_st();
        tc_fence_before();
        // The turn goes before P: the MMA issuer releases the Q buffer only after
        // the last P of the item, so every turn of an item has completed before
        // either slot starts the next one.
        if constexpr (Tr::TOKEN) mbar_arrive(turn(t));
        mbar_arrive(p_full(t, Gt % NSB));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(o_final(t), nd & 1, abort_flag, kSiteEpilogue));
      if (!ok) break;
      tc_fence_after();
      if (combine && t == 1) {
        // Slot 1 hands its row statistics to slot 0, which reads O_1 from TMEM
        // too; O_1 stays until slot 0 is done with it.
        sm_m[row] = m;
        sm_l[row] = l;
        tc_fence_before();
        mbar_arrive(split_ready);
        ok = __all_sync(0xffffffffu, mbar_wait(split_done, nc & 1, abort_flag, kSiteEpilogue));
        if (!ok) break;
        tc_fence_before();
        mbar_arrive(o_free(t));
        G += nkv_t;
        ++nd;
        ++nc;
        continue;
      }
      // Split mode: O = O_0 2^(m_0 - M) + O_1 2^(m_1 - M) over L = l_0 2^(m_0 - M) +
      // l_1 2^(m_1 - M), M = max(m_0, m_1).
      float a0 = 1.f, a1 = 0.f;
      const uint32_t tO1 = lane_addr + Tr::tm_o(1);
      if (combine) {
        ok = __all_sync(0xffffffffu, mbar_wait(split_ready, nc & 1, abort_flag, kSiteEpilogue));
        if (!ok) break;
        tc_fence_after();
        const float m1 = sm_m[row], l1 = sm_l[row];
        const float M = fmaxf(m, m1);
        a0 = M == -INFINITY ? 0.f : ex2(m - M);
        a1 = M == -INFINITY ? 0.f : ex2(m1 - M);
        l = l * a0 + l1 * a1;
        m = M;
      }
      // (With key ranges a row may see no key of its range: l = 0, output 0.)
      const float inv_l = (row_valid && l > 0.f) ? 1.f / l : 0.f;
      const float c0 = a0 * inv_l, c1 = a1 * inv_l;
      __nv_bfloat16* dst =
          p.out + ((static_cast<size_t>(it.b) * p.N + (row_valid ? tok : 0)) * p.Hq + head) * DH;
      // One range of several: the fp32 result normalised within the range goes
      // to the workspace instead, for the merge below.
      const bool partial = SPLIT && it.nch > 1;
      const size_t slot_base =
          partial ? (static_cast<size_t>(it.b * p.Hkv + it.kvh) * p.n_qtiles + qt) * p.nch_max : 0;
      float* pdst = partial ? p.part + ((slot_base + it.c) * BM + row) * DH : nullptr;
#pragma unroll 1
      for (int c = 0; c < DH; c += 16) {
        uint32_t rr[16];
        float y[16];
        tmem_ld16(tO + c, rr);  // warp-wide: every lane loads, only valid rows store
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = __uint_as_float(rr[i]) * c0;
        if (combine) {
          tmem_ld16(tO1 + c, rr);
#pragma unroll
          for (int i = 0; i < 16; ++i) y[i] = fmaf(__uint_as_float(rr[i]), c1, y[i]);
        }
        if (partial) {
          if (row_valid) {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
              *reinterpret_cast<float4*>(pdst + c + i) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
          }
          continue;
        }
        uint4 lo, hi;
        lo.x = pack_bf16x2(y[0], y[1]);
        lo.y = pack_bf16x2(y[2], y[3]);
        lo.z = pack_bf16x2(y[4], y[5]);
        lo.w = pack_bf16x2(y[6], y[7]);
        hi.x = pack_bf16x2(y[8], y[9]);
        hi.y = pack_bf16x2(y[10], y[11]);
        hi.z = pack_bf16x2(y[12], y[13]);
        hi.w = pack_bf16x2(y[14], y[15]);
        if (row_valid) {
          *reinterpret_cast<uint4*>(dst + c) = lo;
          *reinterpret_cast<uint4*>(dst + c + 8) = hi;
        }
      }
      // O has been read: the next item's first PV may overwrite it (and, in
      // split mode, slot 1's).
      tc_fence_before();
      mbar_arrive(o_free(t));
      if (combine) {
        mbar_arrive(split_done);
        ++nc;
      }
      float* lse_dst = p.lse + (static_cast<size_t>(it.b) * p.Hq + head) * p.N + tok;
      if (partial) {
        if (row_valid)
          fwd_merge_ranges<DH>(p, slot_base, it.c, it.nch, row,
                               p.cnt + (static_cast<size_t>(it.b * p.Hkv + it.kvh) * p.n_qtiles + qt) * BM + row,
                               l > 0.f ? m + __log2f(l) : -INFINITY, dst, lse_dst);
      } else if (row_valid) {
        *lse_dst = (m + __log2f(l)) * 0.69314718055994531f;
      }
      G += nkv_t;
      ++nd;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Tr::WARP_MMA) tmem_dealloc(tmem, 512);
}

}  // namespace sqa

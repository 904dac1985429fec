// sqa_api.cu -- host side of the C ABI declared in include/sqa.h: argument
// validation, TMA tensor-map encoding and kernel launches on the caller's
// stream.  This is the only translation unit of libsqa.so.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "sqa.h"
#include "sqa_block.cuh"
#include "sqa_bwd.cuh"
#include "sqa_bwd_bf16.cuh"
#include "sqa_bwd_tf32.cuh"
#include "sqa_decode.cuh"
#include "sqa_fwd.cuh"
#include "sqa_gemm.cuh"

namespace {

thread_local std::string g_last_error;
thread_local cudaEvent_t g_timing[3][2] = {{nullptr, nullptr}, {nullptr, nullptr}, {nullptr, nullptr}};

sqa_status record_timing(int kernel, int which, cudaStream_t stream);

sqa_status fail(sqa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

sqa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SQA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map over a contiguous bf16 tensor [B][N][H][dh], seen by TMA as the
// 4-D array {dh, H, N, B} (innermost first), with a box {panel, box_h, box_n, 1}.
sqa_status make_map(CUtensorMap* map, const void* ptr, int B, int N, int H, int dh, int panel,
                    int box_h, int box_n) {
  auto fn = encode_fn();
  if (!fn) return fail(SQA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[4] = {(cuuint64_t)dh, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)dh * 2, (cuuint64_t)H * dh * 2, (cuuint64_t)N * H * dh * 2};
  const cuuint32_t box[4] = {(cuuint32_t)panel, (cuuint32_t)box_h, (cuuint32_t)box_n, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapSwizzle swz = panel * 2 == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                                 : panel * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                   : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SQA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return SQA_OK;
}

sqa_status record_timing(int kernel, int which, cudaStream_t stream) {
  cudaEvent_t ev = g_timing[kernel][which];
  if (!ev) return SQA_OK;
  cudaError_t e = cudaEventRecord(ev, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord (timing hook)");
  return SQA_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sqa_status check_shape(const sqa_shape& s) {
  if (s.B < 1 || s.N < 1 || s.H_q < 1 || s.H_kv < 1 || s.dh < 1)
    return fail(SQA_ERR_INVALID_ARG, "sizes must be positive (B=%d N=%d H_q=%d H_kv=%d dh=%d)", s.B, s.N,
                s.H_q, s.H_kv, s.dh);
  if (s.H_q % s.H_kv != 0)
    return fail(SQA_ERR_INVALID_ARG, "H_q=%d is not a multiple of H_kv=%d", s.H_q, s.H_kv);
  if (s.dh != 16 && s.dh != 32 && s.dh != 64 && s.dh != 128)
    return fail(SQA_ERR_UNSUPPORTED, "head dim %d not supported (16, 32, 64 or 128)", s.dh);
  if (s.H_q / s.H_kv > 128)
    return fail(SQA_ERR_UNSUPPORTED, "group size H_q/H_kv=%d exceeds 128", s.H_q / s.H_kv);
  if (s.B > 65535 || s.H_q > 65535)
    return fail(SQA_ERR_UNSUPPORTED, "B and H_q must be at most 65535");
  return SQA_OK;
}

sqa_status resolve_scale(float scale, int dh, float* out) {
  if (std::isnan(scale) || std::isinf(scale)) return fail(SQA_ERR_INVALID_ARG, "scale is not finite");
  *out = scale > 0.f ? scale : 1.f / std::sqrt(static_cast<float>(dh));
  return SQA_OK;
}

template <typename Kernel>
sqa_status set_smem(Kernel k, int bytes) {
  // The attribute is per device; setting it on every call costs little.
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  return SQA_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

// SMs of the current device (148 on B200; also the answer when no device can
// be queried, so that workspace sizes can be computed without a GPU).
int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return 148;
  }
  return sms;
}

// How the forward splits its work.  Pairs of Q tiles per CTA; for problems
// whose pairs would fill less than half the SMs, one Q tile per CTA with its
// key tiles shared between the two tile slots (split mode, dh <= 64); and when
// even single Q tiles fill less than half the SMs and the caller gives a
// workspace, ranges of `chunk` key tiles of a Q tile as separate work items,
// merged by the last range to finish.  chunk: the smallest even count whose
// items do not outnumber the SMs (a second item on an SM costs more than
// longer ranges).  Ranges are used only if they shorten the longest Q tile's
// walk by at least kMinRangeSaving key tiles per slot: the memset (a second
// node when a step is replayed as a graph), the partials and the merge cost
// about as much as four to six key-tile steps.
struct FwdPlan {
  int g, T, n_qtiles, n_pairs, n_bh, split, chunk, nch_max;
  long long items;
  size_t part_off, part_l_off, cnt_off, ws_bytes;
};

FwdPlan fwd_plan(const sqa_shape& s, int causal, int sms, bool ranges_allowed) {
  FwdPlan P{};
  const int NK = s.dh == 128 ? 128 : 64;
  P.g = s.H_q / s.H_kv;
  P.T = 128 / P.g;
  P.n_qtiles = (s.N + P.T - 1) / P.T;
  P.n_pairs = (P.n_qtiles + 1) / 2;
  P.n_bh = s.B * s.H_kv;
  P.split = (s.dh <= 64 && static_cast<long long>(P.n_pairs) * P.n_bh < sms / 2) ? 1 : 0;
  P.items = static_cast<long long>(P.split ? P.n_qtiles : P.n_pairs) * P.n_bh;
  if (!P.split || !ranges_allowed || static_cast<long long>(P.n_qtiles) * P.n_bh >= sms / 2) return P;
  auto nkv_of = [&](int qt) {
    const long long end = causal ? std::min<long long>(s.N, static_cast<long long>(qt + 1) * P.T) : s.N;
    return static_cast<int>((end + NK - 1) / NK);
  };
  constexpr int kMinRangeSaving = 6;
  const int nkv_max = nkv_of(P.n_qtiles - 1);
  auto items_of = [&](int chunk) {
    long long n = 0;
    for (int qt = 0; qt < P.n_qtiles; ++qt) n += (nkv_of(qt) + chunk - 1) / chunk;
    return n * P.n_bh;
  };
  int chunk = 2;
  while (chunk < nkv_max && items_of(chunk) > sms) chunk += 2;
  if ((nkv_max + 1) / 2 - chunk / 2 < kMinRangeSaving) return P;
  P.chunk = chunk;
  P.nch_max = (nkv_max + chunk - 1) / chunk;
  P.items = items_of(chunk);
  const size_t slots = static_cast<size_t>(P.n_bh) * P.n_qtiles * P.nch_max * 128;
  P.part_off = 0;
  P.part_l_off = sqa::align256(slots * s.dh * sizeof(float));
  P.cnt_off = P.part_l_off + sqa::align256(slots * sizeof(float));
  P.ws_bytes = P.cnt_off + sqa::align256(static_cast<size_t>(P.n_bh) * P.n_qtiles * 128 * sizeof(int));
  return P;
}

template <int DH>
sqa_status launch_fwd(const void* q, const void* k, const void* v, void* out, float* lse, const sqa_shape& s,
                      int causal, float scale, cudaStream_t stream, void* workspace = nullptr) {
  using Tr = sqa::FwdTraits<DH>;
  sqa::FwdParams p{};
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.N = s.N;
  p.Hq = s.H_q;
  p.Hkv = s.H_kv;
  p.g = s.H_q / s.H_kv;
  p.T = Tr::BM / p.g;
  p.rows = p.T * p.g;
  p.n_qtiles = (s.N + p.T - 1) / p.T;
  p.n_pairs = (p.n_qtiles + 1) / 2;
  p.n_bh = s.B * s.H_kv;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * kLog2e;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "querying the SM count");
  // Split mode (one Q tile per CTA, key tiles shared by the two slots) needs a
  // K/V ring of at least four stages: dh <= 64.  Key ranges need the workspace.
  const FwdPlan P = fwd_plan(s, causal, sms, workspace != nullptr);
  p.split = P.split;
  const long long items = P.items;
  if (items > 0x7fffffffLL) return fail(SQA_ERR_UNSUPPORTED, "problem too large for one launch");
  p.n_items = static_cast<int>(items);
  if (P.chunk > 0) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.chunk = P.chunk;
    p.nch_max = P.nch_max;
    p.part = reinterpret_cast<float*>(ws + P.part_off);
    p.part_l = reinterpret_cast<float*>(ws + P.part_l_off);
    p.cnt = reinterpret_cast<int*>(ws + P.cnt_off);
    e = cudaMemsetAsync(p.cnt, 0, P.ws_bytes - P.cnt_off, stream);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the forward's range counters");
  }
  // Persistent kernel: at most one CTA per SM, each walking several work items.
  const long long grid = items < sms ? items : sms;

  CUtensorMap mq, mk, mv;
  sqa_status st;
  if ((st = make_map(&mq, q, s.B, s.N, s.H_q, DH, Tr::PANEL, p.g, p.T)) != SQA_OK) return st;
  if ((st = make_map(&mk, k, s.B, s.N, s.H_kv, DH, Tr::PANEL, 1, Tr::NK)) != SQA_OK) return st;
  if ((st = make_map(&mv, v, s.B, s.N, s.H_kv, DH, Tr::PANEL, 1, Tr::NK)) != SQA_OK) return st;
  // split mode is compiled as its own kernel (dh <= 64 only)
  auto kernel = p.split ? sqa::sqa_fwd_kernel<DH, DH <= 64> : sqa::sqa_fwd_kernel<DH, false>;
  if ((st = set_smem(kernel, Tr::SMEM_BYTES)) != SQA_OK) return st;
  if ((st = record_timing(0, 0, stream)) != SQA_OK) return st;
  kernel<<<static_cast<unsigned>(grid), Tr::THREADS, Tr::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sqa_fwd launch");
  return record_timing(0, 1, stream);
}

// Ranges per sequence of the decoding split kernel: the general path's fixed
// span, or (register-resident path) about four waves of resident CTAs over the
// whole batch, each range at least rows_min_span positions.  The workspace is
// sized for the most ranges either path can take.
size_t decode_workspace(const sqa_shape& s) {
  const int g = s.H_q / s.H_kv;
  size_t n_split = (static_cast<size_t>(s.N) + sqa::decode_span(s.dh) - 1) / sqa::decode_span(s.dh);
  if (sqa::rows_path(g, s.H_kv, s.dh)) {
    const int ms = sqa::rows_min_span(s.dh, s.H_kv);
    const size_t n_rows = (static_cast<size_t>(s.N) + ms - 1) / ms;
    if (n_rows > n_split) n_split = n_rows;
  }
  return sqa::align256(static_cast<size_t>(s.B) * s.H_kv * n_split * g * (s.dh + 2) * sizeof(float));
}

int decode_rows_span(const sqa_shape& s, int ctas_per_sm) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (4LL * sms * ctas_per_sm + s.B - 1) / s.B;  // ranges per sequence
  const int unit = sqa::rows_step(s.dh) / s.H_kv;                     // positions per CTA step
  long long span = (s.N + want - 1) / want;
  span = (span + unit - 1) / unit * unit;
  const int ms = sqa::rows_min_span(s.dh, s.H_kv);
  return static_cast<int>(span < ms ? ms : span);
}

constexpr int kMaxDevices = 128;

// Resident CTAs per SM of the register-resident split kernel on the current
// device, queried once per device.  The kernel's shared-memory limit must be
// raised first: asked before that, the query sees no resident CTA at all.
template <int DH, int G>
sqa_status decode_rows_occupancy(int smem, int* occ) {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SQA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  int o = cache[dev].load(std::memory_order_relaxed);
  if (o == 0) {
    sqa_status st = set_smem(sqa::sqa_decode_split_kernel<DH, G>, smem);
    if (st != SQA_OK) return st;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, sqa::sqa_decode_split_kernel<DH, G>, sqa::kDecodeThreads,
                                                      smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (o < 1) o = 1;
    cache[dev].store(o, std::memory_order_relaxed);
  }
  *occ = o;
  return SQA_OK;
}

template <int DH, int G>
sqa_status launch_decode_rows(sqa::DecodeParams& p, const sqa_shape& s, cudaStream_t stream) {
  const int smem = static_cast<int>(sqa::rows_smem_bytes(G, DH));
  sqa_status st;
  if ((st = set_smem(sqa::sqa_decode_split_kernel<DH, G>, smem)) != SQA_OK) return st;
  int occ = 1;
  if ((st = decode_rows_occupancy<DH, G>(smem, &occ)) != SQA_OK) return st;
  p.span = decode_rows_span(s, occ);
  p.n_split = (s.N + p.span - 1) / p.span;
  if ((st = record_timing(2, 0, stream)) != SQA_OK) return st;
  sqa::sqa_decode_split_kernel<DH, G>
      <<<dim3(static_cast<unsigned>(p.n_split), static_cast<unsigned>(s.B)), sqa::kDecodeThreads, smem, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sqa_decode split launch");
  return SQA_OK;
}

template <int DH>
sqa_status launch_decode(const void* q, const void* k, const void* v, const int* lens, void* out, float* lse,
                         void* workspace, const sqa_shape& s, float scale, cudaStream_t stream) {
  sqa::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.lens = lens;
  p.part = static_cast<float*>(workspace);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.N = s.N;
  p.Hq = s.H_q;
  p.Hkv = s.H_kv;
  p.g = s.H_q / s.H_kv;
  p.scale_log2 = scale * kLog2e;
  sqa_status st;
  if (sqa::rows_path(p.g, s.H_kv, DH) && aligned(q, 16)) {
    switch (p.g) {
      case 1: st = launch_decode_rows<DH, 1>(p, s, stream); break;
      case 2: st = launch_decode_rows<DH, 2>(p, s, stream); break;
      case 3: st = launch_decode_rows<DH, 3>(p, s, stream); break;
      default: st = launch_decode_rows<DH, 4>(p, s, stream); break;
    }
    if (st != SQA_OK) return st;
  } else if (sqa::mma_path(p.g) && aligned(q, 4)) {
    p.span = sqa::decode_span(DH);
    p.n_split = (s.N + p.span - 1) / p.span;
    const int smem = static_cast<int>(sqa::mma_smem_bytes(DH));
    if ((st = set_smem(sqa::sqa_decode_mma_kernel<DH>, smem)) != SQA_OK) return st;
    const dim3 grid(static_cast<unsigned>(p.n_split * s.H_kv), static_cast<unsigned>(s.B));
    if ((st = record_timing(2, 0, stream)) != SQA_OK) return st;
    sqa::sqa_decode_mma_kernel<DH><<<grid, sqa::kMmaThreads, smem, stream>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "sqa_decode mma split launch");
  } else {
    p.span = sqa::decode_span(DH);
    p.n_split = (s.N + p.span - 1) / p.span;
    const int smem = static_cast<int>(sqa::decode_smem_bytes(p.g, DH));
    if ((st = set_smem(sqa::sqa_decode_split_kernel<DH, 0>, smem)) != SQA_OK) return st;
    const dim3 grid(static_cast<unsigned>(p.n_split * s.H_kv), static_cast<unsigned>(s.B));
    if ((st = record_timing(2, 0, stream)) != SQA_OK) return st;
    sqa::sqa_decode_split_kernel<DH, 0><<<grid, sqa::kDecodeThreads, smem, stream>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "sqa_decode split launch");
  }
  if ((st = record_timing(2, 1, stream)) != SQA_OK) return st;
  sqa::sqa_decode_combine_kernel<DH><<<static_cast<unsigned>(s.B * s.H_q), sqa::kDecodeThreads, 0, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sqa_decode combine launch");
  return SQA_OK;
}

// y = exp2_poly2(x) elementwise (the forward's polynomial exponential), for tests.
__global__ void exp2_poly_kernel(const float* x, float* y, int n) {
  const int pairs = (n + 1) / 2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < pairs; i += gridDim.x * blockDim.x) {
    const int j = 2 * i;
    const float2 r = sqa::dev::exp2_poly2(x[j], j + 1 < n ? x[j + 1] : 0.f);
    y[j] = r.x;
    if (j + 1 < n) y[j + 1] = r.y;
  }
}

// Exponential throughput: 8 independent chains of dependent ex2.approx per
// thread, so the special-function unit, not latency, sets the pace.
__global__ void __launch_bounds__(256) exp2_rate_kernel(float* out, int iters) {
  float v[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) v[c] = -0.5f + 0.01f * c + 1e-6f * threadIdx.x;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int c = 0; c < 8; ++c) v[c] = sqa::dev::ex2(v[c]) - 1.5f;  // stays in [-1, 0.5]
  }
  out[blockIdx.x * 256 + threadIdx.x] = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing
// ever arrives on, with the given limit, through the same slow path the
// kernels use; it gives up, records `site` in the device status word and the
// timeout record, and the kernel returns.
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, unsigned site) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sqa::dev::mbar_init(sqa::dev::smem_u32(&bar), 1);
    abort_flag = 0;
    sqa::dev::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    sqa::dev::mbar_wait_slow(sqa::dev::smem_u32(&bar), 0, &abort_flag, site, limit_ns);
  __syncthreads();
}

int grid_for(long long work, int threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks = (work + threads - 1) / threads;
  const long long cap = static_cast<long long>(sms) * 8;
  return static_cast<int>(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

template <int DH>
sqa_status launch_bwd(const void* dout, const void* q, const void* k, const void* v, const void* out,
                      const float* lse, void* dq, void* dk, void* dv, void* workspace, const sqa_shape& s,
                      int causal, float scale, cudaStream_t stream) {
  const sqa::BwdLayout L = sqa::bwd_layout(s.B, s.N, s.H_q, s.H_kv, DH);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* lse2 = reinterpret_cast<float*>(ws);
  float* Dst = reinterpret_cast<float*>(ws + L.off_D);
  float* dq_acc = DH <= 32 ? reinterpret_cast<float*>(ws + L.off_dq) : nullptr;
  const long long grid_main = static_cast<long long>(L.n_kt) * s.B * s.H_kv;
  const long long grid_q = static_cast<long long>(L.n_qt) * s.B * s.H_kv;
  if (grid_main > 0x7fffffffLL || grid_q > 0x7fffffffLL)
    return fail(SQA_ERR_UNSUPPORTED, "problem too large for one launch");

  sqa::BwdPrepParams pp{};
  pp.dout = static_cast<const __nv_bfloat16*>(dout);
  pp.out = static_cast<const __nv_bfloat16*>(out);
  pp.lse = lse;
  pp.lse2 = lse2;
  pp.D = Dst;
  pp.dq_acc = dq_acc;
  pp.N = s.N;
  pp.Hq = s.H_q;
  pp.Hkv = s.H_kv;
  pp.g = L.g;
  pp.T = L.T;
  pp.rows = L.rows;
  pp.n_qt = L.n_qt;
  pp.n_slots = static_cast<long long>(L.n_slots);
  pp.dq_vec4 = DH <= 32 ? static_cast<long long>(s.B) * s.N * s.H_q * DH / 4 : 0;
  const long long prep_work = pp.n_slots > pp.dq_vec4 ? pp.n_slots : pp.dq_vec4;
  sqa::sqa_bwd_prep_kernel<DH><<<grid_for(prep_work, 256), 256, 0, stream>>>(pp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sqa_bwd prep launch");

  CUtensorMap mq, mdo, mk, mv;
  sqa_status st;
  // Tensor maps: boxes of one 32-, 64- or 128-byte swizzled row segment of dh
  // (all of dh up to 64 elements, a 64-element panel at dh 128).
  constexpr int PANEL = DH < 64 ? DH : 64;
  if ((st = make_map(&mq, q, s.B, s.N, s.H_q, DH, PANEL, L.g, L.T)) != SQA_OK) return st;
  if ((st = make_map(&mdo, dout, s.B, s.N, s.H_q, DH, PANEL, L.g, L.T)) != SQA_OK) return st;
  if ((st = make_map(&mk, k, s.B, s.N, s.H_kv, DH, PANEL, 1, sqa::kBwdTile)) != SQA_OK) return st;
  if ((st = make_map(&mv, v, s.B, s.N, s.H_kv, DH, PANEL, 1, sqa::kBwdTile)) != SQA_OK) return st;
  sqa::BwdParams p{};
  p.lse2 = lse2;
  p.D = Dst;
  p.dq_acc = dq_acc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.N = s.N;
  p.Hq = s.H_q;
  p.Hkv = s.H_kv;
  p.g = L.g;
  p.T = L.T;
  p.rows = L.rows;
  p.n_qt = L.n_qt;
  p.n_bh = s.B * s.H_kv;
  p.causal = causal;
  p.scale_log2 = scale * kLog2e;
  p.scale = scale;
  if constexpr (DH <= 32) {
    // dh 16 and 32: tf32 gradient contractions, half-tile pipelining, dQ added
    // to an fp32 accumulator and converted by a third kernel.
    // Persistent: one CTA per SM walks the items.
    using T32 = sqa::BwdTf32Traits<DH>;
    const int sms = sm_count();
    p.n_items = static_cast<int>(grid_main);
    const unsigned grid = static_cast<unsigned>(grid_main < sms ? grid_main : sms);
    if ((st = set_smem(sqa::sqa_bwd_tf32_kernel<DH>, T32::SMEM_BYTES)) != SQA_OK) return st;
    if ((st = record_timing(1, 0, stream)) != SQA_OK) return st;
    sqa::sqa_bwd_tf32_kernel<DH><<<grid, T32::THREADS, T32::SMEM_BYTES, stream>>>(mq, mdo, mk, mv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "sqa_bwd main launch");
    if ((st = record_timing(1, 1, stream)) != SQA_OK) return st;
    const long long n_vec8 = static_cast<long long>(s.B) * s.N * s.H_q * DH / 8;
    sqa::sqa_bwd_dq_kernel<<<grid_for(n_vec8, 256), 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq),
                                                                      n_vec8, scale);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "sqa_bwd dq launch");
    return SQA_OK;
  } else {
    // dh 64 and 128: dK / dV key-major, then dQ query-major (one CTA per item,
    // heaviest items first); the timing hook brackets both.
    constexpr int D2 = DH < 64 ? 64 : DH;
    using Tr = sqa::BwdBf16Traits<D2>;
    using TQ = sqa::BwdQTraits<D2>;
    CUtensorMap mk64, mv64;
    if ((st = make_map(&mk64, k, s.B, s.N, s.H_kv, DH, PANEL, 1, TQ::NK)) != SQA_OK) return st;
    if ((st = make_map(&mv64, v, s.B, s.N, s.H_kv, DH, PANEL, 1, TQ::NK)) != SQA_OK) return st;
    sqa::BwdQParams pq{};
    pq.q = static_cast<const __nv_bfloat16*>(q);
    pq.dout = static_cast<const __nv_bfloat16*>(dout);
    pq.lse2 = lse2;
    pq.D = Dst;
    pq.dq = static_cast<__nv_bfloat16*>(dq);
    pq.N = s.N;
    pq.Hq = s.H_q;
    pq.Hkv = s.H_kv;
    pq.g = L.g;
    pq.T = L.T;
    pq.rows = L.rows;
    pq.n_qt = L.n_qt;
    pq.n_bh = s.B * s.H_kv;
    pq.causal = causal;
    pq.scale_log2 = scale * kLog2e;
    pq.scale = scale;
    auto kern_kv = L.g >= sqa::kBwdSplitGroup ? sqa::sqa_bwd_kernel<D2, true> : sqa::sqa_bwd_kernel<D2, false>;
    if ((st = set_smem(kern_kv, Tr::SMEM_BYTES)) != SQA_OK) return st;
    if ((st = set_smem(sqa::sqa_bwd_q_kernel<D2>, TQ::SMEM_BYTES)) != SQA_OK) return st;
    if ((st = record_timing(1, 0, stream)) != SQA_OK) return st;
    kern_kv<<<static_cast<unsigned>(grid_main), Tr::THREADS, Tr::SMEM_BYTES, stream>>>(mq, mdo, mk, mv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "sqa_bwd dK/dV launch");
    sqa::sqa_bwd_q_kernel<D2><<<static_cast<unsigned>(grid_q), TQ::THREADS, TQ::SMEM_BYTES, stream>>>(mk64, mv64,
                                                                                                     pq);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "sqa_bwd dQ launch");
    return record_timing(1, 1, stream);
  }
}

// Scratch for sqa_bwd_static_scratch: one device array per GPU that loads the
// library.  In host code the name is only a handle; its device address comes
// from cudaGetSymbolAddress with the device current.  Outside a stream capture
// the address is looked up on every call (cheap), so a context torn down and
// rebuilt between calls (cudaDeviceReset) never leaves a stale pointer; inside
// a capture the address from the last call outside one is used.
static __device__ __align__(256) unsigned char g_static_scratch[SQA_STATIC_SCRATCH_BYTES];

std::mutex g_static_scratch_mu;
void* g_static_scratch_addr[kMaxDevices] = {};

sqa_status static_scratch_address(cudaStream_t stream, void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SQA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cap);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress (static scratch)");
    g_static_scratch_addr[dev] = p;
  } else if (!g_static_scratch_addr[dev]) {
    return fail(SQA_ERR_INVALID_ARG,
                "sqa_bwd_static_scratch: the first call on a device must come before any stream capture");
  }
  *addr = g_static_scratch_addr[dev];
  return SQA_OK;
}

// ---------------------------------------------------------------------------
// The full layer: projections around the attention core.

// 2-D tensor map over a row-major bf16 matrix [rows][cols] whose rows are ld
// elements apart, box {64 columns, box_rows rows}, 128-byte swizzle (64 bf16
// columns per swizzled row).
sqa_status make_map_2d(CUtensorMap* map, const void* ptr, long long rows, long long cols, long long ld,
                       int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(SQA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SQA_ERR_CUDA, "cuTensorMapEncodeTiled (2-D) failed (CUresult %d)", (int)r);
  return SQA_OK;
}

// One K segment of a GEMM: A (K-major [M][k] or MN-major [k][M]) and B
// (K-major [N][k] or MN-major [k][N]), row-major bf16 with row strides lda, ldb.
struct GemmSeg {
  const void* a;
  const void* b;
  int k;
  long long lda, ldb;
};

// D[M x N] = sum_s A_s B_s with the epilogue in `p` (mode and outputs set by
// the caller).  split_k > 1 only with the fp32 reduction epilogue.
template <int BN, bool A_MN, bool B_MN>
sqa_status launch_gemm(int M, int N, const GemmSeg* segs, int n_seg, int split_k, sqa::GemmParams p,
                       cudaStream_t stream) {
  using Tr = sqa::GemmTraits<BN>;
  CUtensorMap ma[3], mb[3];
  sqa_status st;
  int blocks = 0;
  for (int i = 0; i < 3; ++i) {
    // kSwiGLU reads a second B operand (W3) from segs[1] over the same K.
    const int n_maps = p.mode == sqa::kSwiGLU ? 2 : n_seg;
    const GemmSeg& sg = segs[i < n_maps ? i : 0];
    if ((st = A_MN ? make_map_2d(&ma[i], sg.a, sg.k, M, sg.lda, 64) : make_map_2d(&ma[i], sg.a, M, sg.k, sg.lda, 128)) !=
        SQA_OK)
      return st;
    if ((st = B_MN ? make_map_2d(&mb[i], sg.b, sg.k, N, sg.ldb, 64) : make_map_2d(&mb[i], sg.b, N, sg.k, sg.ldb, BN)) !=
        SQA_OK)
      return st;
    if (i < n_seg) {
      p.kseg[i] = sg.k;
      p.kblk0[i] = blocks;
      blocks += (sg.k + Tr::BK - 1) / Tr::BK;
    }
  }
  p.kblk0[n_seg] = blocks;
  p.M = M;
  p.N = N;
  p.n_seg = n_seg;
  p.tiles_m = (M + Tr::BM - 1) / Tr::BM;
  const int tile_cols = p.mode == sqa::kSwiGLU ? BN / 2 : BN;  // output columns per tile
  p.tiles_n = (N + tile_cols - 1) / tile_cols;
  p.split_k = split_k < 1 ? 1 : (split_k > blocks ? blocks : split_k);
  const long long items = static_cast<long long>(p.tiles_m) * p.tiles_n * p.split_k;
  if (items > 0x7fffffffLL) return fail(SQA_ERR_UNSUPPORTED, "GEMM too large for one launch");
  p.n_items = static_cast<int>(items);
  const int sms = sm_count();
  const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  if ((st = set_smem(sqa::sqa_gemm_kernel<BN, A_MN, B_MN>, Tr::SMEM_BYTES)) != SQA_OK) return st;
  sqa::sqa_gemm_kernel<BN, A_MN, B_MN>
      <<<grid, Tr::THREADS, Tr::SMEM_BYTES, stream>>>(ma[0], ma[1], ma[2], mb[0], mb[1], mb[2], p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sqa_gemm launch");
  return SQA_OK;
}

// Column tile width for an output of N columns.
template <bool A_MN, bool B_MN>
sqa_status gemm(int M, int N, const GemmSeg* segs, int n_seg, int split_k, const sqa::GemmParams& p,
                cudaStream_t stream) {
  if (N > 128) return launch_gemm<256, A_MN, B_MN>(M, N, segs, n_seg, split_k, p, stream);
  if (N > 64) return launch_gemm<128, A_MN, B_MN>(M, N, segs, n_seg, split_k, p, stream);
  return launch_gemm<64, A_MN, B_MN>(M, N, segs, n_seg, split_k, p, stream);
}

// K splits for a reduction GEMM with few output tiles: about one item per SM,
// at least four K blocks per item.
int split_for(int M, int N, int K) {
  const long long tiles = static_cast<long long>((M + 127) / 128) * ((N + 255) / 256);
  const int kblocks = (K + 63) / 64;
  long long s = (sm_count() + tiles - 1) / tiles;
  if (s > kblocks / 4) s = kblocks / 4;
  return s < 1 ? 1 : static_cast<int>(s);
}

struct LayerLayout {
  size_t off_dout, off_dq, off_dk, off_dv, off_core, fwd_bytes, bwd_bytes;
};

LayerLayout layer_layout(const sqa_layer_shape& s) {
  LayerLayout L{};
  const size_t M = static_cast<size_t>(s.B) * s.N;
  const size_t table = sqa::align256(static_cast<size_t>(s.N) * (s.dh / 2) * sizeof(float2));
  L.fwd_bytes = table;
  L.off_dout = table;
  L.off_dq = L.off_dout + sqa::align256(M * s.H_q * s.dh * 2);
  L.off_dk = L.off_dq + sqa::align256(M * s.H_q * s.dh * 2);
  L.off_dv = L.off_dk + sqa::align256(M * s.H_kv * s.dh * 2);
  L.off_core = L.off_dv + sqa::align256(M * s.H_kv * s.dh * 2);
  L.bwd_bytes = L.off_core + sqa::bwd_workspace_bytes(s.B, s.N, s.H_q, s.H_kv, s.dh);
  return L;
}

sqa_status check_layer_shape(const sqa_layer_shape& s) {
  const sqa_shape core{s.B, s.N, s.H_q, s.H_kv, s.dh};
  sqa_status st = check_shape(core);
  if (st != SQA_OK) return st;
  if (s.d < 1) return fail(SQA_ERR_INVALID_ARG, "model width d=%d must be positive", s.d);
  if (s.d % 8 != 0) return fail(SQA_ERR_UNSUPPORTED, "model width d=%d must be a multiple of 8", s.d);
  if (static_cast<long long>(s.B) * s.N > 0x7fffffffLL)
    return fail(SQA_ERR_UNSUPPORTED, "B * N must fit in a 32-bit int");
  return SQA_OK;
}

sqa_status rope_table(float2* cs, const sqa_layer_shape& s, float base, cudaStream_t stream) {
  const long long n = static_cast<long long>(s.N) * (s.dh / 2);
  sqa::sqa_rope_table_kernel<<<grid_for(n, 256), 256, 0, stream>>>(cs, s.N, s.dh, static_cast<double>(base));
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rotary table launch");
  return SQA_OK;
}

// The layer forward after validation: Q | K | V = X W_qkv with the rotation in
// the epilogue, the attention core, Y = O W_o (+ resid when given).
sqa_status layer_forward(const void* x, const void* w_qkv, const void* w_o, void* y, const void* resid, void* q,
                         void* k, void* v, void* out, float* lse, float2* table, const sqa_layer_shape& s,
                         int causal, float sc, float rope_base, cudaStream_t cs) {
  sqa_status st;
  const int M = s.B * s.N, nq = s.H_q * s.dh, nk = s.H_kv * s.dh, wqkv = nq + 2 * nk;
  if (rope_base > 0.f && (st = rope_table(table, s, rope_base, cs)) != SQA_OK) return st;
  sqa::GemmParams gp{};
  gp.mode = sqa::kQkvRope;
  gp.q = static_cast<__nv_bfloat16*>(q);
  gp.k = static_cast<__nv_bfloat16*>(k);
  gp.v = static_cast<__nv_bfloat16*>(v);
  gp.nq = nq;
  gp.nk = nk;
  gp.nv = nk;
  gp.dh = s.dh;
  gp.n_tokens = s.N;
  gp.rope_cs = rope_base > 0.f ? table : nullptr;
  const GemmSeg g_qkv{x, w_qkv, s.d, s.d, wqkv};
  if ((st = gemm<false, true>(M, wqkv, &g_qkv, 1, 1, gp, cs)) != SQA_OK) return st;
  const sqa_shape core{s.B, s.N, s.H_q, s.H_kv, s.dh};
  switch (s.dh) {
    case 16: st = launch_fwd<16>(q, k, v, out, lse, core, causal, sc, cs); break;
    case 32: st = launch_fwd<32>(q, k, v, out, lse, core, causal, sc, cs); break;
    case 64: st = launch_fwd<64>(q, k, v, out, lse, core, causal, sc, cs); break;
    default: st = launch_fwd<128>(q, k, v, out, lse, core, causal, sc, cs); break;
  }
  if (st != SQA_OK) return st;
  sqa::GemmParams go{};
  go.mode = sqa::kStoreBf16;
  go.out = static_cast<__nv_bfloat16*>(y);
  go.ld_out = s.d;
  go.resid = static_cast<const __nv_bfloat16*>(resid);
  const GemmSeg g_o{out, w_o, nq, nq, s.d};
  return gemm<false, true>(M, s.d, &g_o, 1, 1, go, cs);
}

// ---------------------------------------------------------------------------
// One decoder block: RMSNorm, the layer, residuals, SwiGLU feed-forward.

sqa_status check_block_shape(const sqa_block_shape& s) {
  const sqa_layer_shape ls{s.B, s.N, s.d, s.H_q, s.H_kv, s.dh};
  sqa_status st = check_layer_shape(ls);
  if (st != SQA_OK) return st;
  if (s.hidden < 1) return fail(SQA_ERR_INVALID_ARG, "hidden width %d must be positive", s.hidden);
  if (s.hidden % 8 != 0) return fail(SQA_ERR_UNSUPPORTED, "hidden width %d must be a multiple of 8", s.hidden);
  if (s.d > 8192) return fail(SQA_ERR_UNSUPPORTED, "model width d=%d exceeds 8192", s.d);
  return SQA_OK;
}

sqa_status check_block_weights(const sqa_block_weights* w) {
  const void* all[] = {w->g1, w->w_qkv, w->w_o, w->g2, w->w1, w->w3, w->w2};
  for (const void* ptr : all) {
    if (!ptr) return fail(SQA_ERR_INVALID_ARG, "null weight pointer");
    if (!aligned(ptr, 16)) return fail(SQA_ERR_UNSUPPORTED, "weights must be 16-byte aligned");
  }
  return SQA_OK;
}

struct BlockLayout {
  size_t n1, rstd1, q, k, v, out, lse, h, n2, rstd2, a, b, act, da, db, dn, dh, layer_ws, layer_ws_bytes, bytes;
};

BlockLayout block_layout(const sqa_block_shape& s) {
  BlockLayout L{};
  const size_t M = static_cast<size_t>(s.B) * s.N, bf = 2;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += sqa::align256(bytes);
    return at;
  };
  L.n1 = take(M * s.d * bf);
  L.rstd1 = take(M * sizeof(float));
  L.q = take(M * s.H_q * s.dh * bf);
  L.k = take(M * s.H_kv * s.dh * bf);
  L.v = take(M * s.H_kv * s.dh * bf);
  L.out = take(M * s.H_q * s.dh * bf);
  L.lse = take(M * s.H_q * sizeof(float));
  L.h = take(M * s.d * bf);
  L.n2 = take(M * s.d * bf);
  L.rstd2 = take(M * sizeof(float));
  L.a = take(M * s.hidden * bf);
  L.b = take(M * s.hidden * bf);
  L.act = take(M * s.hidden * bf);
  L.da = take(M * s.hidden * bf);
  L.db = take(M * s.hidden * bf);
  L.dn = take(M * s.d * bf);
  L.dh = take(M * s.d * bf);
  const sqa_layer_shape ls{s.B, s.N, s.d, s.H_q, s.H_kv, s.dh};
  L.layer_ws_bytes = layer_layout(ls).bwd_bytes;
  L.layer_ws = take(L.layer_ws_bytes);
  L.bytes = o;
  return L;
}

struct BlockPtrs {
  void *n1, *q, *k, *v, *out, *h, *n2, *a, *b, *act, *da, *db, *dn, *dh, *layer_ws;
  float *rstd1, *rstd2, *lse;
  float2* table;
};

BlockPtrs block_ptrs(void* state, const sqa_block_shape& s, const BlockLayout& L) {
  uint8_t* base = static_cast<uint8_t*>(state);
  BlockPtrs b;
  b.n1 = base + L.n1;
  b.q = base + L.q;
  b.k = base + L.k;
  b.v = base + L.v;
  b.out = base + L.out;
  b.h = base + L.h;
  b.n2 = base + L.n2;
  b.a = base + L.a;
  b.b = base + L.b;
  b.act = base + L.act;
  b.da = base + L.da;
  b.db = base + L.db;
  b.dn = base + L.dn;
  b.dh = base + L.dh;
  b.layer_ws = base + L.layer_ws;
  b.rstd1 = reinterpret_cast<float*>(base + L.rstd1);
  b.rstd2 = reinterpret_cast<float*>(base + L.rstd2);
  b.lse = reinterpret_cast<float*>(base + L.lse);
  b.table = reinterpret_cast<float2*>(base + L.layer_ws);  // the layer workspace starts with the rotary table
  (void)s;
  return b;
}

sqa_status rmsnorm(const void* x, const void* g, void* n, float* rstd, int M, int d, cudaStream_t cs) {
  const int blocks = grid_for(static_cast<long long>(M) * 32, 256);
  sqa::sqa_rmsnorm_kernel<<<blocks, 256, 0, cs>>>(static_cast<const __nv_bfloat16*>(x),
                                                  static_cast<const __nv_bfloat16*>(g),
                                                  static_cast<__nv_bfloat16*>(n), rstd, M, d);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
  return SQA_OK;
}

sqa_status rmsnorm_bwd(const void* x, const void* g, const float* rstd, const void* dn, const void* resid, void* dx,
                       float* dg, int M, int d, cudaStream_t cs) {
  const int blocks = grid_for(static_cast<long long>(M) * 32, 256);
  const int smem = d * static_cast<int>(sizeof(float));
  sqa_status st;
  if (smem > 48 * 1024 && (st = set_smem(sqa::sqa_rmsnorm_bwd_kernel, smem)) != SQA_OK) return st;
  sqa::sqa_rmsnorm_bwd_kernel<<<blocks, 256, smem, cs>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(g), rstd,
      static_cast<const __nv_bfloat16*>(dn), static_cast<const __nv_bfloat16*>(resid),
      static_cast<__nv_bfloat16*>(dx), dg, M, d);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm backward launch");
  return SQA_OK;
}

}  // namespace

extern "C" {

sqa_status sqa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, sqa_shape s, int causal,
                   float scale, sqa_stream_t stream) {
  g_last_error.clear();
  if (!q || !k || !v || !out || !lse) return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  sqa_status st = check_shape(s);
  if (st != SQA_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return fail(SQA_ERR_UNSUPPORTED, "q, k, v, out must be 16-byte aligned and lse 4-byte aligned");
  float sc;
  if ((st = resolve_scale(scale, s.dh, &sc)) != SQA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  switch (s.dh) {
    case 16: return launch_fwd<16>(q, k, v, out, lse, s, causal, sc, cs);
    case 32: return launch_fwd<32>(q, k, v, out, lse, s, causal, sc, cs);
    case 64: return launch_fwd<64>(q, k, v, out, lse, s, causal, sc, cs);
    default: return launch_fwd<128>(q, k, v, out, lse, s, causal, sc, cs);
  }
}

size_t sqa_fwd_workspace_bytes(sqa_shape s, int causal) {
  if (check_shape(s) != SQA_OK) return 0;
  return fwd_plan(s, causal, sm_count(), true).ws_bytes;
}

sqa_status sqa_fwd_with_workspace(const void* q, const void* k, const void* v, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes, sqa_shape s, int causal, float scale,
                                  sqa_stream_t stream) {
  g_last_error.clear();
  if (!q || !k || !v || !out || !lse) return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  sqa_status st = check_shape(s);
  if (st != SQA_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return fail(SQA_ERR_UNSUPPORTED, "q, k, v, out must be 16-byte aligned and lse 4-byte aligned");
  const size_t need = fwd_plan(s, causal, sm_count(), true).ws_bytes;
  if (need > 0) {
    if (!workspace) return fail(SQA_ERR_INVALID_ARG, "null workspace (%zu bytes needed)", need);
    if (!aligned(workspace, 256)) return fail(SQA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
    if (workspace_bytes < need)
      return fail(SQA_ERR_INVALID_ARG, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
  }
  float sc;
  if ((st = resolve_scale(scale, s.dh, &sc)) != SQA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  void* ws = need > 0 ? workspace : nullptr;
  switch (s.dh) {
    case 16: return launch_fwd<16>(q, k, v, out, lse, s, causal, sc, cs, ws);
    case 32: return launch_fwd<32>(q, k, v, out, lse, s, causal, sc, cs, ws);
    case 64: return launch_fwd<64>(q, k, v, out, lse, s, causal, sc, cs, ws);
    default: return launch_fwd<128>(q, k, v, out, lse, s, causal, sc, cs, ws);
  }
}

size_t sqa_bwd_workspace_bytes(sqa_shape s) {
  if (check_shape(s) != SQA_OK) return 0;
  return sqa::bwd_workspace_bytes(s.B, s.N, s.H_q, s.H_kv, s.dh);
}

sqa_status sqa_bwd(const void* dout, const void* q, const void* k, const void* v, const void* out, const float* lse,
                   void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, sqa_shape s, int causal,
                   float scale, sqa_stream_t stream) {
  g_last_error.clear();
  if (!dout || !q || !k || !v || !out || !lse || !dq || !dk || !dv || !workspace)
    return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  sqa_status st = check_shape(s);
  if (st != SQA_OK) return st;
  const void* bf[] = {dout, q, k, v, out, dq, dk, dv};
  for (const void* ptr : bf)
    if (!aligned(ptr, 16)) return fail(SQA_ERR_UNSUPPORTED, "bf16 tensors must be 16-byte aligned");
  if (!aligned(lse, 4)) return fail(SQA_ERR_UNSUPPORTED, "lse must be 4-byte aligned");
  if (!aligned(workspace, 256)) return fail(SQA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
  const size_t need = sqa::bwd_workspace_bytes(s.B, s.N, s.H_q, s.H_kv, s.dh);
  if (workspace_bytes < need)
    return fail(SQA_ERR_INVALID_ARG, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
  float sc;
  if ((st = resolve_scale(scale, s.dh, &sc)) != SQA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int c = causal ? 1 : 0;
  switch (s.dh) {
    case 16: return launch_bwd<16>(dout, q, k, v, out, lse, dq, dk, dv, workspace, s, c, sc, cs);
    case 32: return launch_bwd<32>(dout, q, k, v, out, lse, dq, dk, dv, workspace, s, c, sc, cs);
    case 64: return launch_bwd<64>(dout, q, k, v, out, lse, dq, dk, dv, workspace, s, c, sc, cs);
    default: return launch_bwd<128>(dout, q, k, v, out, lse, dq, dk, dv, workspace, s, c, sc, cs);
  }
}

size_t sqa_decode_workspace_bytes(sqa_shape s) {
  if (check_shape(s) != SQA_OK || s.B * static_cast<long long>(s.H_kv) > 65535) return 0;
  return decode_workspace(s);
}

sqa_status sqa_decode(const void* q, const void* k_cache, const void* v_cache, const int* seq_lens, void* out,
                      float* lse, void* workspace, size_t workspace_bytes, sqa_shape s, float scale,
                      sqa_stream_t stream) {
  g_last_error.clear();
  if (!q || !k_cache || !v_cache || !out || !lse || !workspace) return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  sqa_status st = check_shape(s);
  if (st != SQA_OK) return st;
  if (s.B * static_cast<long long>(s.H_kv) > 65535) return fail(SQA_ERR_UNSUPPORTED, "B * H_kv must be at most 65535");
  if (!aligned(q, 2) || !aligned(out, 2)) return fail(SQA_ERR_UNSUPPORTED, "q and out must be 2-byte aligned");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16))
    return fail(SQA_ERR_UNSUPPORTED, "the key/value caches must be 16-byte aligned");
  if (!aligned(lse, 4) || (seq_lens && !aligned(seq_lens, 4)))
    return fail(SQA_ERR_UNSUPPORTED, "lse and seq_lens must be 4-byte aligned");
  if (!aligned(workspace, 256)) return fail(SQA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
  const size_t need = decode_workspace(s);
  if (workspace_bytes < need)
    return fail(SQA_ERR_INVALID_ARG, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
  float sc;
  if ((st = resolve_scale(scale, s.dh, &sc)) != SQA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  switch (s.dh) {
    case 16: return launch_decode<16>(q, k_cache, v_cache, seq_lens, out, lse, workspace, s, sc, cs);
    case 32: return launch_decode<32>(q, k_cache, v_cache, seq_lens, out, lse, workspace, s, sc, cs);
    case 64: return launch_decode<64>(q, k_cache, v_cache, seq_lens, out, lse, workspace, s, sc, cs);
    default: return launch_decode<128>(q, k_cache, v_cache, seq_lens, out, lse, workspace, s, sc, cs);
  }
}

sqa_status sqa_bwd_static_scratch(const void* dout, const void* q, const void* k, const void* v, const void* out,
                                  const float* lse, void* dq, void* dk, void* dv, sqa_shape s, int causal,
                                  float scale, sqa_stream_t stream) {
  g_last_error.clear();
  sqa_status st = check_shape(s);
  if (st != SQA_OK) return st;
  const size_t need = sqa::bwd_workspace_bytes(s.B, s.N, s.H_q, s.H_kv, s.dh);
  if (need > SQA_STATIC_SCRATCH_BYTES)
    return fail(SQA_ERR_UNSUPPORTED, "this shape needs %zu bytes of scratch; the static scratch holds %u (use sqa_bwd)",
                need, SQA_STATIC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if ((st = static_scratch_address(reinterpret_cast<cudaStream_t>(stream), &scratch)) != SQA_OK) return st;
  return sqa_bwd(dout, q, k, v, out, lse, dq, dk, dv, scratch, SQA_STATIC_SCRATCH_BYTES, s, causal, scale, stream);
}

size_t sqa_layer_workspace_bytes(sqa_layer_shape s, int backward) {
  if (check_layer_shape(s) != SQA_OK) return 0;
  const LayerLayout L = layer_layout(s);
  return backward ? L.bwd_bytes : L.fwd_bytes;
}

sqa_status sqa_layer_fwd(const void* x, const void* w_qkv, const void* w_o, void* y, void* q, void* k, void* v,
                         void* out, float* lse, void* workspace, size_t workspace_bytes, sqa_layer_shape s,
                         int causal, float scale, float rope_base, sqa_stream_t stream) {
  g_last_error.clear();
  if (!x || !w_qkv || !w_o || !y || !q || !k || !v || !out || !lse || !workspace)
    return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  sqa_status st = check_layer_shape(s);
  if (st != SQA_OK) return st;
  const void* bf[] = {x, w_qkv, w_o, y, q, k, v, out};
  for (const void* ptr : bf)
    if (!aligned(ptr, 16)) return fail(SQA_ERR_UNSUPPORTED, "bf16 tensors must be 16-byte aligned");
  if (!aligned(lse, 4)) return fail(SQA_ERR_UNSUPPORTED, "lse must be 4-byte aligned");
  if (!aligned(workspace, 256)) return fail(SQA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
  const LayerLayout L = layer_layout(s);
  if (workspace_bytes < L.fwd_bytes)
    return fail(SQA_ERR_INVALID_ARG, "workspace holds %zu bytes, %zu needed", workspace_bytes, L.fwd_bytes);
  if (std::isnan(rope_base) || std::isinf(rope_base) || rope_base < 0.f)
    return fail(SQA_ERR_INVALID_ARG, "rope_base must be finite and non-negative");
  float sc;
  if ((st = resolve_scale(scale, s.dh, &sc)) != SQA_OK) return st;
  return layer_forward(x, w_qkv, w_o, y, nullptr, q, k, v, out, lse, static_cast<float2*>(workspace), s, causal, sc,
                       rope_base, reinterpret_cast<cudaStream_t>(stream));
}

sqa_status sqa_layer_bwd(const void* dy, const void* x, const void* w_qkv, const void* w_o, const void* q,
                         const void* k, const void* v, const void* out, const float* lse, void* dx, float* dw_qkv,
                         float* dw_o, void* workspace, size_t workspace_bytes, sqa_layer_shape s, int causal,
                         float scale, float rope_base, sqa_stream_t stream) {
  g_last_error.clear();
  if (!dy || !x || !w_qkv || !w_o || !q || !k || !v || !out || !lse || !dx || !dw_qkv || !dw_o || !workspace)
    return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  sqa_status st = check_layer_shape(s);
  if (st != SQA_OK) return st;
  const void* bf[] = {dy, x, w_qkv, w_o, q, k, v, out, dx, dw_qkv, dw_o};
  for (const void* ptr : bf)
    if (!aligned(ptr, 16)) return fail(SQA_ERR_UNSUPPORTED, "tensors must be 16-byte aligned");
  if (!aligned(lse, 4)) return fail(SQA_ERR_UNSUPPORTED, "lse must be 4-byte aligned");
  if (!aligned(workspace, 256)) return fail(SQA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
  const LayerLayout L = layer_layout(s);
  if (workspace_bytes < L.bwd_bytes)
    return fail(SQA_ERR_INVALID_ARG, "workspace holds %zu bytes, %zu needed", workspace_bytes, L.bwd_bytes);
  if (std::isnan(rope_base) || std::isinf(rope_base) || rope_base < 0.f)
    return fail(SQA_ERR_INVALID_ARG, "rope_base must be finite and non-negative");
  float sc;
  if ((st = resolve_scale(scale, s.dh, &sc)) != SQA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int M = s.B * s.N, nq = s.H_q * s.dh, nk = s.H_kv * s.dh, wqkv = nq + 2 * nk;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float2* table = reinterpret_cast<float2*>(ws);
  void* dout = ws + L.off_dout;
  void* dq = ws + L.off_dq;
  void* dk = ws + L.off_dk;
  void* dv = ws + L.off_dv;
  void* core_ws = ws + L.off_core;
  if (rope_base > 0.f && (st = rope_table(table, s, rope_base, cs)) != SQA_OK) return st;
  // dO = dY W_o^T (W_o is [H_q dh][d]: K-major for this product)
  sqa::GemmParams p1{};
  p1.mode = sqa::kStoreBf16;
  p1.out = static_cast<__nv_bfloat16*>(dout);
  p1.ld_out = nq;
  const GemmSeg g1{dy, w_o, s.d, s.d, s.d};
  if ((st = gemm<false, false>(M, nq, &g1, 1, 1, p1, cs)) != SQA_OK) return st;
  // dW_o = O^T dY, reduced over all tokens (split over K, fp32 reductions)
  cudaError_t e = cudaMemsetAsync(dw_o, 0, static_cast<size_t>(nq) * s.d * sizeof(float), cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(dw_qkv, 0, static_cast<size_t>(s.d) * wqkv * sizeof(float), cs);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (weight gradients)");
  sqa::GemmParams p2{};
  p2.mode = sqa::kAtomicF32;
  p2.out32 = dw_o;
  p2.ld_out32 = s.d;
  const GemmSeg g2{out, dy, M, nq, s.d};
  if ((st = gemm<true, true>(nq, s.d, &g2, 1, split_for(nq, s.d, M), p2, cs)) != SQA_OK) return st;
  // the attention core's backward, then the rotation undone on dQ and dK
  const sqa_shape core{s.B, s.N, s.H_q, s.H_kv, s.dh};
  const size_t core_bytes = sqa::bwd_workspace_bytes(s.B, s.N, s.H_q, s.H_kv, s.dh);
  if ((st = sqa_bwd(dout, q, k, v, out, lse, dq, dk, dv, core_ws, core_bytes, core, causal, scale, stream)) !=
      SQA_OK)
    return st;
  if (rope_base > 0.f) {
    sqa::sqa_rope_inverse_kernel<<<grid_for(static_cast<long long>(M) * nq / 8, 256), 256, 0, cs>>>(
        static_cast<__nv_bfloat16*>(dq), M, nq, s.dh, s.N, table);
    sqa::sqa_rope_inverse_kernel<<<grid_for(static_cast<long long>(M) * nk / 8, 256), 256, 0, cs>>>(
        static_cast<__nv_bfloat16*>(dk), M, nk, s.dh, s.N, table);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "inverse rotary launch");
  }
  // dW_qkv = X^T [dQ | dK | dV], one product per part into its columns
  const void* parts[3] = {dq, dk, dv};
  const int widths[3] = {nq, nk, nk}, col0[3] = {0, nq, nq + nk};
  for (int i = 0; i < 3; ++i) {
    sqa::GemmParams p3{};
    p3.mode = sqa::kAtomicF32;
    p3.out32 = dw_qkv + col0[i];
    p3.ld_out32 = wqkv;
    const GemmSeg g3{x, parts[i], M, s.d, widths[i]};
    if ((st = gemm<true, true>(s.d, widths[i], &g3, 1, split_for(s.d, widths[i], M), p3, cs)) != SQA_OK) return st;
  }
  // dX = dQ W_q^T + dK W_k^T + dV W_v^T: three K segments, W_qkv's column
  // blocks as K-major B operands
  sqa::GemmParams p4{};
  p4.mode = sqa::kStoreBf16;
  p4.out = static_cast<__nv_bfloat16*>(dx);
  p4.ld_out = s.d;
  const __nv_bfloat16* w = static_cast<const __nv_bfloat16*>(w_qkv);
  const GemmSeg g4[3] = {{dq, w, nq, nq, wqkv}, {dk, w + nq, nk, nk, wqkv}, {dv, w + nq + nk, nk, nk, wqkv}};
  return gemm<false, false>(M, s.d, g4, 3, 1, p4, cs);
}

size_t sqa_block_state_bytes(sqa_block_shape s) {
  if (check_block_shape(s) != SQA_OK) return 0;
  return block_layout(s).bytes;
}

sqa_status sqa_block_fwd(const void* x, const sqa_block_weights* w, void* y, void* state, size_t state_bytes,
                         sqa_block_shape s, int causal, float scale, float rope_base, sqa_stream_t stream) {
  g_last_error.clear();
  if (!x || !w || !y || !state) return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  sqa_status st = check_block_shape(s);
  if (st != SQA_OK) return st;
  if ((st = check_block_weights(w)) != SQA_OK) return st;
  if (!aligned(x, 16) || !aligned(y, 16)) return fail(SQA_ERR_UNSUPPORTED, "x and y must be 16-byte aligned");
  if (!aligned(state, 256)) return fail(SQA_ERR_UNSUPPORTED, "state must be 256-byte aligned");
  const BlockLayout L = block_layout(s);
  if (state_bytes < L.bytes) return fail(SQA_ERR_INVALID_ARG, "state holds %zu bytes, %zu needed", state_bytes, L.bytes);
  if (std::isnan(rope_base) || std::isinf(rope_base) || rope_base < 0.f)
    return fail(SQA_ERR_INVALID_ARG, "rope_base must be finite and non-negative");
  float sc;
  if ((st = resolve_scale(scale, s.dh, &sc)) != SQA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const BlockPtrs b = block_ptrs(state, s, L);
  const sqa_layer_shape ls{s.B, s.N, s.d, s.H_q, s.H_kv, s.dh};
  const int M = s.B * s.N;
  // n1 = RMSNorm(x; g1); h = x + SQA(n1)
  if ((st = rmsnorm(x, w->g1, b.n1, b.rstd1, M, s.d, cs)) != SQA_OK) return st;
  if ((st = layer_forward(b.n1, w->w_qkv, w->w_o, b.h, x, b.q, b.k, b.v, b.out, b.lse, b.table, ls, causal, sc,
                          rope_base, cs)) != SQA_OK)
    return st;
  // n2 = RMSNorm(h; g2); a = n2 W1, b = n2 W3, m = silu(a) * b; y = h + m W2
  if ((st = rmsnorm(b.h, w->g2, b.n2, b.rstd2, M, s.d, cs)) != SQA_OK) return st;
  sqa::GemmParams p1{};
  p1.mode = sqa::kSwiGLU;
  p1.out = static_cast<__nv_bfloat16*>(b.act);
  p1.sw_a = static_cast<__nv_bfloat16*>(b.a);
  p1.sw_b = static_cast<__nv_bfloat16*>(b.b);
  p1.ld_out = s.hidden;
  const GemmSeg g1[2] = {{b.n2, w->w1, s.d, s.d, s.hidden}, {b.n2, w->w3, s.d, s.d, s.hidden}};
  if ((st = launch_gemm<256, false, true>(M, s.hidden, g1, 1, 1, p1, cs)) != SQA_OK) return st;
  sqa::GemmParams p2{};
  p2.mode = sqa::kStoreBf16;
  p2.out = static_cast<__nv_bfloat16*>(y);
  p2.ld_out = s.d;
  p2.resid = static_cast<const __nv_bfloat16*>(b.h);
  const GemmSeg g2{b.act, w->w2, s.hidden, s.hidden, s.d};
  return gemm<false, true>(M, s.d, &g2, 1, 1, p2, cs);
}

sqa_status sqa_block_bwd(const void* dy, const void* x, const sqa_block_weights* w, void* state, size_t state_bytes,
                         void* dx, const sqa_block_grads* gr, sqa_block_shape s, int causal, float scale,
                         float rope_base, sqa_stream_t stream) {
  g_last_error.clear();
  if (!dy || !x || !w || !state || !dx || !gr) return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  if (!gr->g1 || !gr->w_qkv || !gr->w_o || !gr->g2 || !gr->w1 || !gr->w3 || !gr->w2)
    return fail(SQA_ERR_INVALID_ARG, "null gradient pointer");
  sqa_status st = check_block_shape(s);
  if (st != SQA_OK) return st;
  if ((st = check_block_weights(w)) != SQA_OK) return st;
  const void* al[] = {dy, x, dx, gr->g1, gr->w_qkv, gr->w_o, gr->g2, gr->w1, gr->w3, gr->w2};
  for (const void* ptr : al)
    if (!aligned(ptr, 16)) return fail(SQA_ERR_UNSUPPORTED, "tensors must be 16-byte aligned");
  if (!aligned(state, 256)) return fail(SQA_ERR_UNSUPPORTED, "state must be 256-byte aligned");
  const BlockLayout L = block_layout(s);
  if (state_bytes < L.bytes) return fail(SQA_ERR_INVALID_ARG, "state holds %zu bytes, %zu needed", state_bytes, L.bytes);
  if (std::isnan(rope_base) || std::isinf(rope_base) || rope_base < 0.f)
    return fail(SQA_ERR_INVALID_ARG, "rope_base must be finite and non-negative");
  float sc;
  if ((st = resolve_scale(scale, s.dh, &sc)) != SQA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const BlockPtrs b = block_ptrs(state, s, L);
  const int M = s.B * s.N;
  const size_t dsz = static_cast<size_t>(s.d) * sizeof(float);
  const size_t whid = static_cast<size_t>(s.d) * s.hidden * sizeof(float);
  cudaError_t e = cudaMemsetAsync(gr->g1, 0, dsz, cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->g2, 0, dsz, cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->w1, 0, whid, cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->w3, 0, whid, cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(gr->w2, 0, whid, cs);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (block gradients)");
  // dM = dY W2^T, and with the saved a, b: da = dM b silu'(a), db = dM silu(a)
  sqa::GemmParams p1{};
  p1.mode = sqa::kSwiGLUBwd;
  p1.out = static_cast<__nv_bfloat16*>(b.da);
  p1.out2 = static_cast<__nv_bfloat16*>(b.db);
  p1.sw_a = static_cast<__nv_bfloat16*>(b.a);
  p1.sw_b = static_cast<__nv_bfloat16*>(b.b);
  p1.ld_out = s.hidden;
  const GemmSeg g1{dy, w->w2, s.d, s.d, s.d};
  if ((st = gemm<false, false>(M, s.hidden, &g1, 1, 1, p1, cs)) != SQA_OK) return st;
  // dW2 = m^T dY; dW1 = n2^T da; dW3 = n2^T db (fp32 reductions over the tokens)
  sqa::GemmParams pw{};
  pw.mode = sqa::kAtomicF32;
  pw.out32 = gr->w2;
  pw.ld_out32 = s.d;
  const GemmSeg gw2{b.act, dy, M, s.hidden, s.d};
  if ((st = gemm<true, true>(s.hidden, s.d, &gw2, 1, split_for(s.hidden, s.d, M), pw, cs)) != SQA_OK) return st;
  pw.ld_out32 = s.hidden;
  pw.out32 = gr->w1;
  const GemmSeg gw1{b.n2, b.da, M, s.d, s.hidden};
  if ((st = gemm<true, true>(s.d, s.hidden, &gw1, 1, split_for(s.d, s.hidden, M), pw, cs)) != SQA_OK) return st;
  pw.out32 = gr->w3;
  const GemmSeg gw3{b.n2, b.db, M, s.d, s.hidden};
  if ((st = gemm<true, true>(s.d, s.hidden, &gw3, 1, split_for(s.d, s.hidden, M), pw, cs)) != SQA_OK) return st;
  // dn2 = da W1^T + db W3^T
  sqa::GemmParams p2{};
  p2.mode = sqa::kStoreBf16;
  p2.out = static_cast<__nv_bfloat16*>(b.dn);
  p2.ld_out = s.d;
  const GemmSeg g2[2] = {{b.da, w->w1, s.hidden, s.hidden, s.hidden}, {b.db, w->w3, s.hidden, s.hidden, s.hidden}};
  if ((st = gemm<false, false>(M, s.d, g2, 2, 1, p2, cs)) != SQA_OK) return st;
  // dh = dY + RMSNorm'(h; g2) dn2
  if ((st = rmsnorm_bwd(b.h, w->g2, b.rstd2, b.dn, dy, b.dh, gr->g2, M, s.d, cs)) != SQA_OK) return st;
  // the layer's backward with X = n1, dY = dh: dn1, dW_qkv, dW_o
  const sqa_layer_shape ls{s.B, s.N, s.d, s.H_q, s.H_kv, s.dh};
  if ((st = sqa_layer_bwd(b.dh, b.n1, w->w_qkv, w->w_o, b.q, b.k, b.v, b.out, b.lse, b.dn, gr->w_qkv, gr->w_o,
                          b.layer_ws, L.layer_ws_bytes, ls, causal, scale, rope_base, stream)) != SQA_OK)
    return st;
  // dx = dh + RMSNorm'(x; g1) dn1
  return rmsnorm_bwd(x, w->g1, b.rstd1, b.dn, b.dh, dx, gr->g1, M, s.d, cs);
}

sqa_status sqa_selftest_exp2_poly(const float* x, float* y, int n, sqa_stream_t stream) {
  g_last_error.clear();
  if (n <= 0) return SQA_OK;
  if (!x || !y) return fail(SQA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(x, 8) || !aligned(y, 8)) return fail(SQA_ERR_INVALID_ARG, "x and y must be 8-byte aligned");
  const int pairs = (n + 1) / 2;
  exp2_poly_kernel<<<grid_for(pairs, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sqa_selftest_exp2_poly launch");
  return SQA_OK;
}

sqa_status sqa_selftest_exp2_rate(float* out, int n_blocks, int iters, sqa_stream_t stream) {
  g_last_error.clear();
  if (!out) return fail(SQA_ERR_INVALID_ARG, "null pointer");
  if (n_blocks < 1 || n_blocks > 65535) return fail(SQA_ERR_INVALID_ARG, "n_blocks must be in [1, 65535]");
  if (iters < 1 || iters > (1 << 20)) return fail(SQA_ERR_INVALID_ARG, "iters must be in [1, 1048576]");
  exp2_rate_kernel<<<n_blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(out, iters);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sqa_selftest_exp2_rate launch");
  return SQA_OK;
}

sqa_status sqa_selftest_wait_timeout(unsigned int limit_us, unsigned int site, sqa_stream_t stream) {
  g_last_error.clear();
  if (limit_us < 1 || limit_us > 100000) return fail(SQA_ERR_INVALID_ARG, "limit_us must be in [1, 100000]");
  if (site > 4) return fail(SQA_ERR_INVALID_ARG, "site must be in [0, 4]");
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * limit_us, site);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sqa_selftest_wait_timeout launch");
  return SQA_OK;
}

const char* sqa_status_string(sqa_status status) {
  switch (status) {
    case SQA_OK: return "ok";
    case SQA_ERR_INVALID_ARG: return "invalid argument";
    case SQA_ERR_UNSUPPORTED: return "unsupported";
    case SQA_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* sqa_last_error(void) { return g_last_error.c_str(); }

sqa_status sqa_device_status(unsigned int* word, int clear) {
  g_last_error.clear();
  if (!word) return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaMemcpyFromSymbol(word, sqa::g_wait_status, sizeof(unsigned int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(sqa::g_wait_status, &zero, sizeof(unsigned int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  }
  return SQA_OK;
}

sqa_status sqa_device_timeout_info(unsigned int info[4], int clear) {
  g_last_error.clear();
  if (!info) return fail(SQA_ERR_INVALID_ARG, "null pointer argument");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaMemcpyFromSymbol(info, sqa::g_timeout_info, 4 * sizeof(unsigned int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the timeout record");
  if (clear) {
    const unsigned int zero[4] = {0, 0, 0, 0};
    e = cudaMemcpyToSymbol(sqa::g_timeout_info, zero, sizeof(zero));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "clearing the timeout record");
  }
  return SQA_OK;
}

sqa_status sqa_set_timing_events(int kernel, void* start, void* stop) {
  g_last_error.clear();
  if (kernel < 0 || kernel > 2)
    return fail(SQA_ERR_INVALID_ARG, "kernel index %d is not 0 (fwd), 1 (bwd) or 2 (decode)", kernel);
  if ((start == nullptr) != (stop == nullptr)) return fail(SQA_ERR_INVALID_ARG, "give both events or neither");
  g_timing[kernel][0] = static_cast<cudaEvent_t>(start);
  g_timing[kernel][1] = static_cast<cudaEvent_t>(stop);
  return SQA_OK;
}

int sqa_version(void) { return 100; }

}  // extern "C"

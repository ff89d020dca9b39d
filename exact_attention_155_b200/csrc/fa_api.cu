// C ABI of libfa.so: argument checking, TMA descriptor encoding and kernel launch.
// Declarations and the contract of every entry point are in include/fa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <set>
#include <utility>
#include <string>

#include "fa.h"
#include "ptx.cuh"
#include "fwd.cuh"
#include "bwd.cuh"
#include "bwd_det.cuh"
#include "decode.cuh"
#include "merge.cuh"
#include "accumulate.cuh"

namespace {

constexpr int kAbiVersion = 2;
thread_local std::string g_last_error;

fa_status fail(fa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

fa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Largest divisor of n that is <= cap: the number of heads whose CTAs are scheduled
// together so their K/V (or Q/dO) stay resident in L2.
int head_group_for(int n, int cap) {
  for (int g = cap < n ? cap : n; g > 1; --g)
    if (n % g == 0) return g;
  return 1;
}
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// ---------------------------------------------------------------- device info
struct DeviceInfo {
  bool queried = false;
  bool supported = false;
  int sms = 0;
  std::string why;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

fa_status current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.queried) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    di.queried = true;
    di.sms = sms;
    di.supported = (major == 10 && minor == 0);
    if (!di.supported) {
      char buf[128];
      snprintf(buf, sizeof(buf), "device %d is sm_%d%d; this library is built for sm_100a only", dev,
               major, minor);
      di.why = buf;
    }
  }
  if (!di.supported) return fail(FA_ERR_UNSUPPORTED, "%s", di.why.c_str());
  if (dev_out) *dev_out = dev;
  if (sms_out) *sms_out = di.sms;
  return FA_OK;
}

// ------------------------------------------------------------- TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

fa_status get_encoder(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!cached) {
    if (err != cudaSuccess) return cuda_fail(err, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
    return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  }
  *fn = cached;
  return FA_OK;
}

// Row layout shared by every [*, H, d] bf16 operand of one call: dense batches of N
// rows (row (b, n) is token b*N + n) or one packed batch of `total` tokens split into
// sequences by cu_seqlens. Consecutive tokens of an operand are `rs` elements apart.
struct RowLayout {
  int B, N, H, d;
  const int* cu_seqlens;  // NULL: dense
  int total;              // variable length only
};

// 4-D map over one operand; one box = 128 rows of one head x 64 columns of d, stored
// with the 128-byte swizzle the UMMA descriptors expect. Dense: dims (d, H, N, B) with
// row coordinate n and batch coordinate b. Variable length: dims (d, H, total, 1) with
// row coordinate = token.
fa_status map_rows(CUtensorMap* map, const void* ptr, const RowLayout& lay, long long rs) {
  EncodeTiledFn enc;
  fa_status st = get_encoder(&enc);
  if (st != FA_OK) return st;
  const bool var = lay.cu_seqlens != nullptr;
  const cuuint64_t rows = static_cast<cuuint64_t>(var ? lay.total : lay.N);
  const cuuint64_t gdim[4] = {static_cast<cuuint64_t>(lay.d), static_cast<cuuint64_t>(lay.H), rows,
                              static_cast<cuuint64_t>(var ? 1 : lay.B)};
  const cuuint64_t gstride[3] = {static_cast<cuuint64_t>(lay.d) * 2, static_cast<cuuint64_t>(rs) * 2,
                                 rows * static_cast<cuuint64_t>(rs) * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estride[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), gdim, gstride,
                   box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FA_OK;
}

// ------------------------------------------------------------ launch helpers
std::mutex g_attr_mu;
std::set<std::pair<const void*, int>> g_attr_done;

// Raises a kernel's dynamic shared-memory limit once per (kernel, device).
template <typename Kern>
fa_status set_smem(Kern kernel, int bytes, int dev) {
  const void* key = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (g_attr_done.count({key, dev})) return FA_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  g_attr_done.insert({key, dev});
  return FA_OK;
}

fa_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return FA_OK;
}

// Work-unit tickets of the persistent forward: one counter per launch, taken round
// robin from a small pool in the library's device image and zeroed on the launch's
// stream right before the kernel (so launches on different streams use different
// counters unless more than kTicketSlots are in flight at once).
constexpr int kTicketSlots = 64;
__device__ unsigned int g_fwd_tickets[kTicketSlots];
std::atomic<unsigned int> g_ticket_next{0};

template <int D, bool CAUSAL, bool GENERAL>
fa_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     fa::FwdParams p, int dev, int sms, cudaStream_t stream) {
  using L = fa::FwdLayout<D>;
  auto kern = fa::fwd_kernel<D, CAUSAL, GENERAL>;
  fa_status st = set_smem(kern, L::kAlloc, dev);
  if (st != FA_OK) return st;
  void* tickets = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&tickets, g_fwd_tickets);
  if (e != cudaSuccess) return cuda_fail(e, "fa_fwd: cudaGetSymbolAddress(tickets)");
  p.ticket = static_cast<unsigned int*>(tickets) + (g_ticket_next.fetch_add(1) % kTicketSlots);
  if ((e = cudaMemsetAsync(p.ticket, 0, sizeof(unsigned int), stream)) != cudaSuccess)
    return cuda_fail(e, "fa_fwd: reset the work-unit ticket");
  // One CTA per SM (the shared memory and TMEM of a CTA fill one), each taking units
  // until none are left.
  const unsigned grid = static_cast<unsigned>(std::min(p.num_units, std::max(1, sms)));
  kern<<<grid, L::kThreads, L::kAlloc, stream>>>(mq, mk, mv, p);
  return check_launch("fa_fwd kernel launch");
}


template <int D, bool CAUSAL, bool GENERAL>
fa_status launch_bwd_main(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const CUtensorMap& mdo, const fa::BwdParams& p, int dev, int sms,
                          cudaStream_t stream) {
  using L = fa::BwdLayout<D>;
  auto kern = fa::bwd_kernel<D, CAUSAL, GENERAL>;
  fa_status st = set_smem(kern, L::kBytes, dev);
  if (st != FA_OK) return st;
  // Persistent: one CTA per SM (its shared memory and TMEM fill one), each taking
  // units from the workspace counter until none are left.
  const unsigned grid = static_cast<unsigned>(std::min(p.num_units, std::max(1, sms)));
  kern<<<grid, L::kThreads, L::kBytes, stream>>>(mq, mk, mv, mdo, p);
  return check_launch("fa_bwd main kernel launch");
}

template <int D, bool CAUSAL, bool GENERAL>
fa_status launch_bwd_det(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                             const CUtensorMap& mdo, fa::BwdParams p, int dev, cudaStream_t stream) {
  using LA = fa::BwdKVLayout<D>;
  using LB = fa::BwdQLayout<D>;
  auto ka = fa::bwd_dkdv_kernel<D, CAUSAL, GENERAL>;
  auto kb = fa::bwd_dq_kernel<D, CAUSAL, GENERAL>;
  fa_status st = set_smem(ka, LA::kBytes, dev);
  if (st != FA_OK) return st;
  if ((st = set_smem(kb, LB::kBytes, dev)) != FA_OK) return st;
  const unsigned grid = static_cast<unsigned>(p.nqt) * p.B * p.H;
  // dK/dV: four heads per group (their Q and dO, 4 x 8 MiB at N = 16384, stay in L2).
  p.head_group = head_group_for(p.B * p.H, 4);
  ka<<<grid, LA::kThreads, LA::kBytes, stream>>>(mq, mk, mv, mdo, p);
  if ((st = check_launch("fa_bwd dK/dV kernel launch")) != FA_OK) return st;
  // dQ: eight heads per group (their K and V, 8 x 8 MiB at N = 16384, stay in L2).
  p.head_group = head_group_for(p.B * p.H, 8);
  kb<<<grid, LB::kThreads, LB::kBytes, stream>>>(mq, mk, mv, mdo, p);
  return check_launch("fa_bwd dQ kernel launch");
}

// Strides (elements between consecutive tokens) of the eight row-major operands of a
// backward call, in the order q, k, v, out, dout, dq, dk, dv.
struct BwdStrides {
  long long q, k, v, o, dout, dq, dk, dv;
};

fa_status run_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, const RowLayout& lay,
                  const BwdStrides& rs, int wl, int wr, float scale, void* workspace,
                  const fa::BwdWorkspace& ws, bool deterministic, int dev, int sms, cudaStream_t stream,
                  cudaEvent_t ev_start, cudaEvent_t ev_stop) {
  const int B = lay.B, H = lay.H, N = lay.N, d = lay.d;
  CUtensorMap mq, mk, mv, mdo;
  fa_status st;
  if ((st = map_rows(&mq, q, lay, rs.q)) != FA_OK) return st;
  if ((st = map_rows(&mk, k, lay, rs.k)) != FA_OK) return st;
  if ((st = map_rows(&mv, v, lay, rs.v)) != FA_OK) return st;
  if ((st = map_rows(&mdo, dout, lay, rs.dout)) != FA_OK) return st;
  fa::BwdParams p;
  p.B = B;
  p.H = H;
  p.N = N;
  p.Np = (N + 127) / 128 * 128;
  p.nqt = p.Np / 128;
  // Four heads: their Q, dO and fp32 dQ accumulator (4 x 16 MiB at N = 16384) fit in L2.
  p.head_group = head_group_for(B * H, 4);
  p.window_left = wl;
  p.window_right = wr;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.cu_seqlens = lay.cu_seqlens;
  p.total = lay.total;
  p.rs_o = rs.o;
  p.rs_do = rs.dout;
  p.rs_dq = rs.dq;
  p.rs_dk = rs.dk;
  p.rs_dv = rs.dv;
  p.out = static_cast<const uint16_t*>(out);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  char* w = static_cast<char*>(workspace);
  // The deterministic kernels write dq directly: no fp32 accumulator to zero or convert.
  p.dq_acc = deterministic ? nullptr : reinterpret_cast<float*>(w + ws.dq_off);
  p.num_units = p.nqt * B * H;  // < 2^31: checked by the callers
  p.ticket = deterministic ? nullptr : reinterpret_cast<unsigned int*>(w + ws.ticket_off);
  p.lse2 = reinterpret_cast<float*>(w + ws.lse2_off);
  p.dvec = reinterpret_cast<float*>(w + ws.dvec_off);
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  const long long tpr = d / 8;
  const long long pre_threads = static_cast<long long>(B) * H * p.Np * tpr;
  const unsigned pre_blocks = static_cast<unsigned>((pre_threads + 255) / 256);
  if (d == 64) fa::bwd_pre_kernel<64><<<pre_blocks, 256, 0, stream>>>(p);
  else fa::bwd_pre_kernel<128><<<pre_blocks, 256, 0, stream>>>(p);
  if ((st = check_launch("fa_bwd preprocess launch")) != FA_OK) return st;
  cudaError_t e;
  if (ev_start && (e = cudaEventRecord(ev_start, stream)) != cudaSuccess)
    return cuda_fail(e, "fa_bwd_profiled: record start event");
  const bool general = lay.cu_seqlens != nullptr || wl >= 0 || wr > 0;
  if (deterministic) {
    if (d == 64)
      st = general ? launch_bwd_det<64, false, true>(mq, mk, mv, mdo, p, dev, stream)
           : wr == 0 ? launch_bwd_det<64, true, false>(mq, mk, mv, mdo, p, dev, stream)
                     : launch_bwd_det<64, false, false>(mq, mk, mv, mdo, p, dev, stream);
    else
      st = general ? launch_bwd_det<128, false, true>(mq, mk, mv, mdo, p, dev, stream)
           : wr == 0 ? launch_bwd_det<128, true, false>(mq, mk, mv, mdo, p, dev, stream)
                     : launch_bwd_det<128, false, false>(mq, mk, mv, mdo, p, dev, stream);
    if (st != FA_OK) return st;
    if (ev_stop && (e = cudaEventRecord(ev_stop, stream)) != cudaSuccess)
      return cuda_fail(e, "fa_bwd_profiled: record stop event");
    return FA_OK;
  }
  if (d == 64)
    st = general ? launch_bwd_main<64, false, true>(mq, mk, mv, mdo, p, dev, sms, stream)
         : wr == 0 ? launch_bwd_main<64, true, false>(mq, mk, mv, mdo, p, dev, sms, stream)
                   : launch_bwd_main<64, false, false>(mq, mk, mv, mdo, p, dev, sms, stream);
  else
    st = general ? launch_bwd_main<128, false, true>(mq, mk, mv, mdo, p, dev, sms, stream)
         : wr == 0 ? launch_bwd_main<128, true, false>(mq, mk, mv, mdo, p, dev, sms, stream)
                   : launch_bwd_main<128, false, false>(mq, mk, mv, mdo, p, dev, sms, stream);
  if (st != FA_OK) return st;
  if (ev_stop && (e = cudaEventRecord(ev_stop, stream)) != cudaSuccess)
    return cuda_fail(e, "fa_bwd_profiled: record stop event");
  const long long cv_threads = static_cast<long long>(B) * N * H * tpr;
  const unsigned cv_blocks = static_cast<unsigned>((cv_threads + 255) / 256);
  if (d == 64) fa::bwd_dq_convert_kernel<64><<<cv_blocks, 256, 0, stream>>>(p);
  else fa::bwd_dq_convert_kernel<128><<<cv_blocks, 256, 0, stream>>>(p);
  return check_launch("fa_bwd dq convert launch");
}

fa_status run_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                  const RowLayout& lay, long long rs_q, long long rs_k, long long rs_v,
                  long long rs_o, int wl, int wr, float scale, int dev, int sms,
                  cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  fa_status st;
  if ((st = map_rows(&mq, q, lay, rs_q)) != FA_OK) return st;
  if ((st = map_rows(&mk, k, lay, rs_k)) != FA_OK) return st;
  if ((st = map_rows(&mv, v, lay, rs_v)) != FA_OK) return st;
  fa::FwdParams p;
  p.B = lay.B;
  p.H = lay.H;
  p.N = lay.N;
  p.num_qblocks = (lay.N + 255) / 256;
  p.num_units = p.num_qblocks * lay.B * lay.H;  // < 2^31: checked by the callers
  p.ticket = nullptr;
  // Eight heads: their K and V (8 x 4 MiB at N = 8192) stay in L2 while their CTAs run.
  p.head_group = head_group_for(lay.B * lay.H, 8);
  p.window_left = wl;
  p.window_right = wr;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.cu_seqlens = lay.cu_seqlens;
  p.total = lay.total;
  p.o_rs = rs_o;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  // Plain dense problems (no sequence offsets, no window beyond causal) take the
  // kernel instance with those tests compiled out.
  const bool general = lay.cu_seqlens != nullptr || wl >= 0 || wr > 0;
  if (lay.d == 64) {
    if (general) return launch_fwd<64, false, true>(mq, mk, mv, p, dev, sms, stream);
    return wr == 0 ? launch_fwd<64, true, false>(mq, mk, mv, p, dev, sms, stream)
                   : launch_fwd<64, false, false>(mq, mk, mv, p, dev, sms, stream);
  }
  if (general) return launch_fwd<128, false, true>(mq, mk, mv, p, dev, sms, stream);
  return wr == 0 ? launch_fwd<128, true, false>(mq, mk, mv, p, dev, sms, stream)
                 : launch_fwd<128, false, false>(mq, mk, mv, p, dev, sms, stream);
}

// Checks shared by the extended entry points; on success fills `lay`, `wr_eff` (the
// right window edge with causal folded in) and returns FA_OK. `*empty` is set when the
// call has no work.
fa_status check_ex(const char* who, const int* cu_seqlens, int total_tokens, int B, int H, int N,
                   int d, int causal, int window_left, int window_right, float scale,
                   const long long* strides, int nstrides, RowLayout* lay, int* wr_eff, bool* empty) {
  if (B < 0 || H < 0 || N < 0 || total_tokens < 0)
    return fail(FA_ERR_INVALID_ARG, "%s: negative size B=%d H=%d N=%d total=%d", who, B, H, N, total_tokens);
  if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "%s: head dim %d not supported (64 or 128)", who, d);
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "%s: scale must be finite", who);
  if (window_left < -1 || window_right < -1)
    return fail(FA_ERR_INVALID_ARG, "%s: window edges must be >= 0, or -1 for unbounded", who);
  if (causal && window_right > 0)
    return fail(FA_ERR_INVALID_ARG, "%s: causal attention needs window_right 0 or -1 (got %d)", who,
                window_right);
  for (int i = 0; i < nstrides; ++i)
    if (strides[i] < static_cast<long long>(H) * d || strides[i] % 8 != 0)
      return fail(FA_ERR_INVALID_ARG,
                  "%s: row stride %lld must be a multiple of 8 elements and at least H*d = %d", who,
                  strides[i], H * d);
  const long long nkb = (static_cast<long long>(N) + 127) / 128;  // backward grid per (b, h)
  if (nkb * B * H >= (1LL << 31) || N > (1 << 30) || H > (1 << 20))
    return fail(FA_ERR_INVALID_ARG, "%s: problem too large (B=%d H=%d N=%d)", who, B, H, N);
  lay->B = B;
  lay->N = N;
  lay->H = H;
  lay->d = d;
  lay->cu_seqlens = cu_seqlens;
  lay->total = cu_seqlens ? total_tokens : 0;
  *wr_eff = causal ? 0 : window_right;
  *empty = B == 0 || H == 0 || N == 0 || (cu_seqlens && total_tokens == 0);
  if (cu_seqlens && !aligned4(cu_seqlens))
    return fail(FA_ERR_INVALID_ARG, "%s: cu_seqlens must be 4-byte aligned", who);
  return FA_OK;
}

// CTAs per (batch, head) for decode: a power of two <= 8 (one portable cluster)
// so the grid is about one wave (6 CTAs per SM), with at least 64 keys per CTA.
int decode_splits(int B, int H, int Ncap, int sms, int* chunk_out) {
  const long long heads = static_cast<long long>(B) * H;
  const long long want = (static_cast<long long>(sms) * FA_DECODE_CTAS_PER_SM + heads - 1) / std::max(1LL, heads);
  int ns = 1;
  while (ns < fa::kDecodeMaxSplits && ns < want && static_cast<long long>(ns) * 2 * 64 <= Ncap) ns *= 2;
  const int chunk = (Ncap + ns - 1) / ns;
  if (chunk_out) *chunk_out = chunk;
  return ns;
}

__global__ void timeout_probe_kernel(long long limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    fa::mbar_init(fa::smem_u32(&bar), 1);
    fa::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on this barrier: the bounded wait must give up.
    const long long t0 = clock64();
    while (!fa::mbar_try_wait(fa::smem_u32(&bar), 0)) {
      if (clock64() - t0 > limit) {
        fa::report(fa::kDevTimeout, 0x7FFu, 0u);
        break;
      }
    }
  }
}

// Scratch for fa_bwd_noalloc, for callers that cannot allocate device memory: a
// fixed-size array in the library's own device image (held by every GPU while the
// library is loaded). Host code must not use the symbol as a pointer; the device
// address is looked up with cudaGetSymbolAddress in the current context.
static __device__ __align__(256) unsigned char g_bwd_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the current device's context. Looked up on
// every call (cudaGetSymbolAddress allocates nothing): the address belongs to the
// context that loaded the library's device code, so a cached value would go stale if
// the caller reset the device and a new primary context loaded the code elsewhere.
fa_status noalloc_scratch(void** out) {
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_bwd_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "fa_bwd_noalloc: cudaGetSymbolAddress(scratch)");
  *out = ptr;
  return FA_OK;
}

}  // namespace

// =============================================================================
extern "C" {

int fa_abi_version(void) { return kAbiVersion; }

const char* fa_last_error(void) { return g_last_error.c_str(); }

fa_status fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
                 int N, int d, int causal, float scale, void* stream) {
  if (B < 0 || H < 0 || N < 0) return fail(FA_ERR_INVALID_ARG, "fa_fwd: negative size B=%d H=%d N=%d", B, H, N);
  if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "fa_fwd: head dim %d not supported (64 or 128)", d);
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "fa_fwd: scale must be finite");
  if (B == 0 || H == 0 || N == 0) return FA_OK;
  if (!q || !k || !v || !out || !lse) return fail(FA_ERR_INVALID_ARG, "fa_fwd: null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(lse))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd: q/k/v/out must be 16-byte aligned, lse 4-byte aligned");
  const long long nqb = (static_cast<long long>(N) + 255) / 256;
  if (nqb * B * H >= (1LL << 31) || N > (1 << 30) || H > (1 << 20))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd: problem too large (B=%d H=%d N=%d)", B, H, N);
  int dev = 0, sms = 0;
  fa_status st = current_device(&dev, &sms);
  if (st != FA_OK) return st;
  const RowLayout lay{B, N, H, d, nullptr, 0};
  const long long rs = static_cast<long long>(H) * d;
  return run_fwd(q, k, v, out, lse, lay, rs, rs, rs, rs, -1, causal ? 0 : -1, scale, dev, sms,
                 static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse,
                    const int* cu_seqlens, int total_tokens, int B, int H, int N, int d,
                    long long q_row_stride, long long k_row_stride, long long v_row_stride,
                    long long out_row_stride, int causal, int window_left, int window_right,
                    float scale, void* stream) {
  const long long strides[4] = {q_row_stride, k_row_stride, v_row_stride, out_row_stride};
  RowLayout lay;
  int wr = -1;
  bool empty = false;
  fa_status st = check_ex("fa_fwd_ex", cu_seqlens, total_tokens, B, H, N, d, causal, window_left,
                          window_right, scale, strides, 4, &lay, &wr, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !out || !lse) return fail(FA_ERR_INVALID_ARG, "fa_fwd_ex: null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(lse))
    return fail(FA_ERR_INVALID_ARG, "fa_fwd_ex: q/k/v/out must be 16-byte aligned, lse 4-byte aligned");
  int dev = 0, sms = 0;
  if ((st = current_device(&dev, &sms)) != FA_OK) return st;
  return run_fwd(q, k, v, out, lse, lay, q_row_stride, k_row_stride, v_row_stride, out_row_stride,
                 window_left, wr, scale, dev, sms, static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || (d != 64 && d != 128)) return 0;
  return fa::bwd_ws_layout(B, H, N, d).total;
}

fa_status fa_bwd_profiled(const void* q, const void* k, const void* v, const void* out,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                          int H, int N, int d, int causal, float scale, void* workspace,
                          size_t workspace_bytes, void* stream, void* main_start,
                          void* main_stop) {
  if (B < 0 || H < 0 || N < 0) return fail(FA_ERR_INVALID_ARG, "fa_bwd: negative size B=%d H=%d N=%d", B, H, N);
  if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "fa_bwd: head dim %d not supported (64 or 128)", d);
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "fa_bwd: scale must be finite");
  if (B == 0 || H == 0 || N == 0) return FA_OK;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv)
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned4(lse))
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: tensors must be 16-byte aligned, lse 4-byte aligned");
  const long long nkb = (static_cast<long long>(N) + 127) / 128;
  if (nkb * B * H >= (1LL << 31) || N > (1 << 30) || H > (1 << 20))
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: problem too large (B=%d H=%d N=%d)", B, H, N);
  const fa::BwdWorkspace ws = fa::bwd_ws_layout(B, H, N, d);
  if (!workspace || workspace_bytes < ws.total)
    return fail(FA_ERR_WORKSPACE, "fa_bwd: workspace needs %zu bytes, got %zu", ws.total, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(FA_ERR_INVALID_ARG, "fa_bwd: workspace must be 256-byte aligned");
  int dev = 0, sms = 0;
  fa_status st = current_device(&dev, &sms);
  if (st != FA_OK) return st;
  const RowLayout lay{B, N, H, d, nullptr, 0};
  const long long rs = static_cast<long long>(H) * d;
  const BwdStrides strides{rs, rs, rs, rs, rs, rs, rs, rs};
  return run_bwd(q, k, v, out, dout, lse, dq, dk, dv, lay, strides, -1, causal ? 0 : -1, scale,
                 workspace, ws, false, dev, sms, static_cast<cudaStream_t>(stream),
                 static_cast<cudaEvent_t>(main_start), static_cast<cudaEvent_t>(main_stop));
}

fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* out, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens,
                    int total_tokens, int B, int H, int N, int d, const long long* row_strides,
                    int causal, int window_left, int window_right, float scale, int deterministic,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!row_strides) return fail(FA_ERR_INVALID_ARG, "fa_bwd_ex: row_strides is null");
  RowLayout lay;
  int wr = -1;
  bool empty = false;
  fa_status st = check_ex("fa_bwd_ex", cu_seqlens, total_tokens, B, H, N, d, causal, window_left,
                          window_right, scale, row_strides, 8, &lay, &wr, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv)
    return fail(FA_ERR_INVALID_ARG, "fa_bwd_ex: null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned4(lse))
    return fail(FA_ERR_INVALID_ARG, "fa_bwd_ex: tensors must be 16-byte aligned, lse 4-byte aligned");
  const fa::BwdWorkspace ws = fa::bwd_ws_layout(B, H, N, d);
  if (!workspace || workspace_bytes < ws.total)
    return fail(FA_ERR_WORKSPACE, "fa_bwd_ex: workspace needs %zu bytes, got %zu", ws.total, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(FA_ERR_INVALID_ARG, "fa_bwd_ex: workspace must be 256-byte aligned");
  int dev = 0, sms = 0;
  if ((st = current_device(&dev, &sms)) != FA_OK) return st;
  const BwdStrides strides{row_strides[0], row_strides[1], row_strides[2], row_strides[3],
                           row_strides[4], row_strides[5], row_strides[6], row_strides[7]};
  return run_bwd(q, k, v, out, dout, lse, dq, dk, dv, lay, strides, window_left, wr, scale, workspace,
                 ws, deterministic != 0, dev, sms, static_cast<cudaStream_t>(stream), nullptr, nullptr);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return fa_bwd_profiled(q, k, v, out, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, workspace,
                         workspace_bytes, stream, nullptr, nullptr);
}

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* out,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, int causal, float scale, void* stream) {
  if (B < 0 || H < 0 || N < 0)
    return fail(FA_ERR_INVALID_ARG, "fa_bwd_noalloc: negative size B=%d H=%d N=%d", B, H, N);
  if (d != 64 && d != 128)
    return fail(FA_ERR_UNSUPPORTED, "fa_bwd_noalloc: head dim %d not supported (64 or 128)", d);
  if (B == 0 || H == 0 || N == 0) return FA_OK;
  const size_t need = fa::bwd_ws_layout(B, H, N, d).total;
  if (need > FA_BWD_NOALLOC_SCRATCH_BYTES)
    return fail(FA_ERR_WORKSPACE,
                "fa_bwd_noalloc: this problem needs %zu bytes of scratch but the built-in "
                "scratch holds %u; call fa_bwd with a caller-provided workspace instead",
                need, FA_BWD_NOALLOC_SCRATCH_BYTES);
  fa_status st = current_device(nullptr, nullptr);
  if (st != FA_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != FA_OK) return st;
  return fa_bwd(q, k, v, out, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, scratch,
                FA_BWD_NOALLOC_SCRATCH_BYTES, stream);
}

size_t fa_decode_workspace_size(int B, int H, int Ncap, int d) {
  (void)B;
  (void)H;
  (void)Ncap;
  (void)d;
  return 0;  // split partials are combined on chip (cluster shared memory)
}

}  // extern "C"

namespace {

// Shared by fa_decode and fa_decode_paged: argument checks, split choice and the
// cluster launch. block_table == NULL selects the contiguous cache layout.
fa_status run_decode(const char* who, const void* q, void* k_cache, void* v_cache,
                     const int* cache_seqlens, const void* k_new, const void* v_new, void* out,
                     float* lse, int B, int H, int Ncap, int d, float scale,
                     const int* block_table, int max_blocks, int page_shift, int num_pages,
                     void* stream) {
  if (B < 0 || H < 0) return fail(FA_ERR_INVALID_ARG, "%s: negative size B=%d H=%d", who, B, H);
  if (Ncap <= 0) return fail(FA_ERR_INVALID_ARG, "%s: cache capacity must be >= 1 (got %d)", who, Ncap);
  if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "%s: head dim %d not supported (64 or 128)", who, d);
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "%s: scale must be finite", who);
  if (B == 0 || H == 0) return FA_OK;
  if (!q || !k_cache || !v_cache || !cache_seqlens || !out)
    return fail(FA_ERR_INVALID_ARG, "%s: null pointer", who);
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(FA_ERR_INVALID_ARG, "%s: k_new and v_new must both be given or both be NULL", who);
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (k_new && (!aligned16(k_new) || !aligned16(v_new))) || !aligned4(cache_seqlens) ||
      (lse && !aligned4(lse)) || (block_table && !aligned4(block_table)))
    return fail(FA_ERR_INVALID_ARG, "%s: bf16 tensors must be 16-byte aligned, int/float 4-byte", who);
  if (H > 65535 || B > 65535) return fail(FA_ERR_INVALID_ARG, "%s: B and H must be <= 65535", who);
  int dev = 0, sms = 0;
  fa_status st = current_device(&dev, &sms);
  if (st != FA_OK) return st;
  int chunk = 0;
  const int ns = decode_splits(B, H, Ncap, sms, &chunk);
  fa::DecodeParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.k_cache = static_cast<uint16_t*>(k_cache);
  p.v_cache = static_cast<uint16_t*>(v_cache);
  p.seqlens = cache_seqlens;
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.v_new = static_cast<const uint16_t*>(v_new);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Ncap = Ncap;
  p.nsplit = ns;
  p.chunk = chunk;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.block_table = block_table;
  p.max_blocks = max_blocks;
  p.num_pages = num_pages;
  p.page_shift = page_shift;
  // The `ns` CTAs of one (batch, head) run as one thread-block cluster.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ns, H, B);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ns;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (block_table)
    e = (d == 64) ? cudaLaunchKernelEx(&cfg, fa::decode_kernel<64, true>, p)
                  : cudaLaunchKernelEx(&cfg, fa::decode_kernel<128, true>, p);
  else
    e = (d == 64) ? cudaLaunchKernelEx(&cfg, fa::decode_kernel<64, false>, p)
                  : cudaLaunchKernelEx(&cfg, fa::decode_kernel<128, false>, p);
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  return check_launch("decode kernel launch");
}

}  // namespace

extern "C" {

fa_status fa_decode(const void* q, void* k_cache, void* v_cache, const int* cache_seqlens,
                    const void* k_new, const void* v_new, void* out, float* lse, int B, int H,
                    int Ncap, int d, int causal, float scale, void* workspace,
                    size_t workspace_bytes, void* stream) {
  (void)causal;  // one query at the end of the sequence sees every valid key
  (void)workspace;
  (void)workspace_bytes;
  return run_decode("fa_decode", q, k_cache, v_cache, cache_seqlens, k_new, v_new, out, lse, B, H,
                    Ncap, d, scale, nullptr, 0, 0, 0, stream);
}

fa_status fa_decode_paged(const void* q, void* k_pages, void* v_pages, const int* block_table,
                          int max_blocks, int page_size, int num_pages, const int* cache_seqlens,
                          const void* k_new, const void* v_new, void* out, float* lse, int B,
                          int H, int d, int causal, float scale, void* stream) {
  (void)causal;
  if (page_size < 1 || page_size > (1 << 16) || (page_size & (page_size - 1)) != 0)
    return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: page_size must be a power of two in [1, 65536] (got %d)",
                page_size);
  if (max_blocks < 1 || num_pages < 1)
    return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: max_blocks and num_pages must be >= 1");
  const long long cap = static_cast<long long>(max_blocks) * page_size;
  if (cap > (1LL << 30)) return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: capacity too large");
  if (B > 0 && H > 0 && !block_table) return fail(FA_ERR_INVALID_ARG, "fa_decode_paged: null block_table");
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  return run_decode("fa_decode_paged", q, k_pages, v_pages, cache_seqlens, k_new, v_new, out, lse, B,
                    H, static_cast<int>(cap), d, scale, block_table, max_blocks, shift, num_pages,
                    stream);
}

fa_status fa_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                            void* out, int B, int N, int H, int d, void* stream) {
  if (B < 0 || N < 0 || H < 0) return fail(FA_ERR_INVALID_ARG, "fa_merge_partials: negative size");
  if (d != 64 && d != 128)
    return fail(FA_ERR_UNSUPPORTED, "fa_merge_partials: head dim %d not supported (64 or 128)", d);
  if (B == 0 || N == 0 || H == 0) return FA_OK;
  if (!o_acc || !lse_acc || !o_part || !lse_part)
    return fail(FA_ERR_INVALID_ARG, "fa_merge_partials: null pointer");
  if (!aligned16(o_acc) || !aligned16(o_part) || !aligned4(lse_acc) || !aligned4(lse_part) ||
      (out && !aligned16(out)))
    return fail(FA_ERR_INVALID_ARG, "fa_merge_partials: o tensors 16-byte aligned, lse 4-byte");
  const long long threads = static_cast<long long>(B) * N * H * (d / 8);
  if (threads / 256 >= (1LL << 31)) return fail(FA_ERR_INVALID_ARG, "fa_merge_partials: too large");
  int dev = 0;
  fa_status st = current_device(&dev, nullptr);
  if (st != FA_OK) return st;
  fa::MergeParams p;
  p.o_acc = o_acc;
  p.lse_acc = lse_acc;
  p.o_part = static_cast<const uint16_t*>(o_part);
  p.lse_part = lse_part;
  p.out = static_cast<uint16_t*>(out);
  p.B = B;
  p.N = N;
  p.H = H;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64) fa::merge_kernel<64><<<blocks, 256, 0, s>>>(p);
  else fa::merge_kernel<128><<<blocks, 256, 0, s>>>(p);
  return check_launch("fa_merge_partials launch");
}

fa_status fa_accumulate(float* acc, const void* part, void* out, long long n, void* stream) {
  if (n < 0) return fail(FA_ERR_INVALID_ARG, "fa_accumulate: n < 0");
  if (n == 0) return FA_OK;
  if (!acc) return fail(FA_ERR_INVALID_ARG, "fa_accumulate: null acc");
  if (!part && !out) return fail(FA_ERR_INVALID_ARG, "fa_accumulate: part and out are both NULL");
  if (n % 8 != 0) return fail(FA_ERR_INVALID_ARG, "fa_accumulate: n (%lld) must be a multiple of 8", n);
  if (!aligned16(acc) || (part && !aligned16(part)) || (out && !aligned16(out)))
    return fail(FA_ERR_INVALID_ARG, "fa_accumulate: acc, part and out must be 16-byte aligned");
  const long long n8 = n / 8;
  const long long blocks = (n8 + 255) / 256;
  if (blocks >= (1LL << 31)) return fail(FA_ERR_INVALID_ARG, "fa_accumulate: n too large");
  fa_status st = current_device(nullptr, nullptr);
  if (st != FA_OK) return st;
  fa::AccumParams p;
  p.acc = acc;
  p.part = static_cast<const uint16_t*>(part);
  p.out = static_cast<uint16_t*>(out);
  p.n8 = n8;
  fa::accumulate_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return check_launch("fa_accumulate launch");
}

fa_status fa_device_status(void* stream, unsigned int* site_out, unsigned int* info_out) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fa_device_status: stream synchronize");
  unsigned int w[4] = {0, 0, 0, 0};
  e = cudaMemcpyFromSymbol(w, fa::g_status, sizeof(w));
  if (e != cudaSuccess) return cuda_fail(e, "fa_device_status: read status word");
  if (site_out) *site_out = w[1];
  if (info_out) *info_out = w[2];
  if (w[0] == 0) return FA_OK;
  const unsigned int zero[4] = {0, 0, 0, 0};
  e = cudaMemcpyToSymbol(fa::g_status, zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "fa_device_status: clear status word");
  if (w[0] == fa::kDevTimeout)
    return fail(FA_ERR_TIMEOUT, "device pipeline wait timed out (site 0x%x, info %u)", w[1], w[2]);
  if (w[0] == fa::kDevBadInput)
    return fail(FA_ERR_DEVICE_INPUT, "device input out of range (site 0x%x, batch %u)", w[1], w[2]);
  return fail(FA_ERR_CUDA, "unknown device status %u", w[0]);
}

fa_status fa_debug_timeout_probe(long long limit_cycles, void* stream) {
  if (limit_cycles < 1000) limit_cycles = 1000;
  if (limit_cycles > 4000000000LL) limit_cycles = 4000000000LL;
  fa_status st = current_device(nullptr, nullptr);
  if (st != FA_OK) return st;
  timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return check_launch("fa_debug_timeout_probe launch");
}

}  // extern "C"

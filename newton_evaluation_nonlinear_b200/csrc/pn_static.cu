// pn_static.cu -- pn_eval_static: an evaluation that allocates no memory.
//
// Some callers cannot call cudaMalloc: code that must not touch the device
// allocator once it is running (a real-time or embedded loop with its memory
// budget fixed at start-up, a process whose device memory is owned by another
// framework's allocator, a plug-in that may not grow its footprint).  For them
// this entry point runs the FP32 fused diagonal-family iteration kernel of the
// tanh RNN with all of its scratch -- second iterate buffer, projected inputs,
// packed weights, scan descriptors, control block, residual history -- carved
// out of one file-scope device array of fixed size, reserved when the library
// is loaded and kept until the process exits.  The caller passes inputs and
// outputs only.  The loop is driven from the host (one launch per iteration,
// the stop decision read back after each).
#include <cuda_runtime.h>

#include <climits>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <mutex>

#include "pn_dispatch.cuh"

namespace pn {
const void* aux_kernel(int which);           // pn_api.cu
void set_thread_error(const char* msg);      // pn_api.cu: the text of pn_last_error(NULL)
}
using namespace pn;

// 24 MiB of scratch for every call of pn_eval_static, on every device that loads
// the library.  Host code may not use this name as an address: the device
// address comes from cudaGetSymbolAddress (see static_scratch_base).
constexpr size_t kStaticScratchBytes = size_t(24) << 20;
static __device__ __align__(256) unsigned char pn_static_scratch[kStaticScratchBytes];

namespace {

pn_status static_fail(pn_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  set_thread_error(buf);
  return st;
}

// Device address of the scratch array on the current device, looked up once
// per device (the first call on each device does this, with that device current).
pn_status static_scratch_base(int dev, unsigned char** out) {
  static std::mutex mu;
  static unsigned char* base[64] = {nullptr};
  if (dev < 0 || dev >= 64) return static_fail(PN_ERR_INVALID, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!base[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, pn_static_scratch);
    if (e != cudaSuccess || !p)
      return static_fail(PN_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
    base[dev] = static_cast<unsigned char*>(p);
  }
  *out = base[dev];
  return PN_OK;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// wt[k * DP + j] = W[j][k] (transposed recurrent weights, zero-padded to DP).
__global__ void static_pack_kernel(const float* __restrict__ params, float* __restrict__ wt, int D, int DP) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < DP * DP; e += gridDim.x * blockDim.x) {
    const int k = e / DP, j = e % DP;
    wt[e] = (j < D && k < D) ? params[(size_t)j * D + k] : 0.0f;
  }
}

bool device_ptr(const void* p, int dev) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeManaged || (at.type == cudaMemoryTypeDevice && at.device == dev);
}

}  // namespace

extern "C" {

PN_API pn_status pn_eval_static(const float* params, size_t n_params, int D, int d_in, int T, int B,
                                const float* x, const float* s0, pn_mode mode, int max_iters, float tol,
                                float* states, int* iters_out, float* resid_out, void* cuda_stream) {
  set_thread_error("");
  if (D < 1 || D > 64) return static_fail(PN_ERR_INVALID, "pn_eval_static: D=%d outside 1..64", D);
  if (d_in < 1 || d_in > 1024) return static_fail(PN_ERR_INVALID, "pn_eval_static: d_in=%d outside 1..1024", d_in);
  if (T < 1 || B < 1 || (long long)B * T > INT_MAX) return static_fail(PN_ERR_INVALID, "pn_eval_static: bad T or B");
  if (mode != PN_JACOBI && mode != PN_PICARD && mode != PN_QUASI)
    return static_fail(PN_ERR_INVALID, "pn_eval_static: mode must be jacobi, picard or quasi");
  if (max_iters < 0 || !(tol >= 0.0f) || !std::isfinite(tol))
    return static_fail(PN_ERR_INVALID, "pn_eval_static: need max_iters >= 0 and a finite tol >= 0");
  const size_t need_params = (size_t)D * D + (size_t)D * d_in + D;
  if (!params || n_params != need_params)
    return static_fail(PN_ERR_INVALID, "pn_eval_static: n_params=%zu, the tanh RNN needs %zu", n_params, need_params);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return static_fail(PN_ERR_CUDA, "pn_eval_static: no CUDA device");
  if (!x || !s0 || !states || (((uintptr_t)x | (uintptr_t)s0 | (uintptr_t)states) & 15u) ||
      !device_ptr(x, dev) || !device_ptr(s0, dev) || !device_ptr(states, dev))
    return static_fail(PN_ERR_INVALID, "pn_eval_static: x, s0 and states must be 16-byte aligned device memory");

  int DP = 4;
  while (DP < D) DP <<= 1;
  const KInfo ki = lookup(PN_CELL_TANH_RNN, mode, DP, false, false);
  if (!ki.fn) return static_fail(PN_ERR_INVALID, "pn_eval_static: no kernel for D=%d", D);
  const int G = ki.G;   // DP <= 64: one channel group
  const int nchunks = (T + ki.L - 1) / ki.L;
  const size_t ntiles = (size_t)B * nchunks;
  const size_t nstate = (size_t)B * T * D;

  // scratch layout, 256-byte aligned regions
  size_t off = 0;
  const size_t o_ctrl = off;  off = align256(off + sizeof(Ctrl));
  const size_t o_args = off;  off = align256(off + sizeof(Args));
  const size_t o_hist = off;  off = align256(off + sizeof(float) * kHistCap);
  const size_t o_par = off;   off = align256(off + sizeof(float) * need_params);
  const size_t o_wt = off;    off = align256(off + sizeof(float) * (size_t)DP * DP);
  const size_t o_bhn = off;   off = align256(off + sizeof(float) * DP);
  const size_t o_flags = off; off = align256(off + sizeof(unsigned) * ntiles);
  const size_t o_agg = off;   off = align256(off + sizeof(float) * ntiles * 2 * G);
  const size_t o_pref = off;  off = align256(off + sizeof(float) * ntiles * G);
  const size_t o_u = off;     off = align256(off + sizeof(float) * nstate);
  const size_t o_buf1 = off;  off = align256(off + sizeof(float) * nstate);
  if (off > kStaticScratchBytes)
    return static_fail(PN_ERR_INVALID,
                       "pn_eval_static: D=%d, T=%d, B=%d needs %zu bytes of scratch; the static buffer holds %zu "
                       "(about B*T*D <= 2.9M states at D=64)",
                       D, T, B, off, kStaticScratchBytes);

  unsigned char* base = nullptr;
  pn_status st = static_scratch_base(dev, &base);
  if (st != PN_OK) return st;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(base + o_ctrl);
  Args* args = reinterpret_cast<Args*>(base + o_args);
  cudaStream_t stream = (cudaStream_t)cuda_stream;

#define PN_STATIC_CUDA(call)                                                                               \
  do {                                                                                                     \
    cudaError_t e_ = (call);                                                                               \
    if (e_ != cudaSuccess) return static_fail(PN_ERR_CUDA, "pn_eval_static: %s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

  // The scratch keeps the previous call's contents, and the region this call reads as look-back
  // flags may have held another shape's floats or flags: clear this call's flags on every call (a
  // few KB), and restart the look-back epochs well before they wrap.
  Ctrl hc;
  PN_STATIC_CUDA(cudaMemcpyAsync(&hc, ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, stream));
  PN_STATIC_CUDA(cudaStreamSynchronize(stream));
  PN_STATIC_CUDA(cudaMemsetAsync(base + o_flags, 0, sizeof(unsigned) * ntiles, stream));
  if (hc.epoch > (1u << 29)) PN_STATIC_CUDA(cudaMemsetAsync(&ctrl->epoch, 0, sizeof(unsigned), stream));
  PN_STATIC_CUDA(cudaMemcpyAsync(base + o_par, params, sizeof(float) * need_params, cudaMemcpyHostToDevice, stream));
  PN_STATIC_CUDA(cudaMemsetAsync(base + o_bhn, 0, sizeof(float) * DP, stream));
  {
    const float* pp = reinterpret_cast<const float*>(base + o_par);
    float* wt = reinterpret_cast<float*>(base + o_wt);
    int d = D, dp = DP;
    void* kargs[] = {(void*)&pp, (void*)&wt, (void*)&d, (void*)&dp};
    PN_STATIC_CUDA(cudaLaunchKernel((const void*)&static_pack_kernel, dim3(16), dim3(256), kargs, 0, stream));
  }
  Args ha{};
  ha.x = x;
  ha.s0 = s0;
  ha.states = states;
  ha.tol = tol;
  ha.max_iters = max_iters;
  ha.timeout_ns = 1000000000LL;
  ha.stall_ticket = -1;
  ha.use_cond = 0;
  ha.newton_band = -1;
  ha.damping = 1.0f;
  PN_STATIC_CUDA(cudaMemcpyAsync(args, &ha, sizeof(Args), cudaMemcpyHostToDevice, stream));

  // u = U x + b, s^(0) = s0
  {
    const Args* a_d = args;
    const float* U = reinterpret_cast<const float*>(base + o_par) + (size_t)D * D;
    const float* bias = U + (size_t)D * d_in;
    float* u = reinterpret_cast<float*>(base + o_u);
    int M = B * T, N = D, K = d_in;
    void* kargs[] = {(void*)&a_d, (void*)&U, (void*)&bias, (void*)&u, (void*)&M, (void*)&N, (void*)&K};
    PN_STATIC_CUDA(cudaLaunchKernel(aux_kernel(0), dim3((unsigned)((M + 63) / 64), (unsigned)((N + 63) / 64)), dim3(256),
                                    kargs, 0, stream));
    Ctrl* c = ctrl;
    int d = D, t = T, b = B;
    void* kargs2[] = {(void*)&a_d, (void*)&c, (void*)&d, (void*)&t, (void*)&b};
    const unsigned g = (unsigned)std::min<size_t>((nstate + 255) / 256, 148u * 16u);
    PN_STATIC_CUDA(cudaLaunchKernel(aux_kernel(1), dim3(g), dim3(256), kargs2, 0, stream));
  }

  IterParams P{};
  P.wt = reinterpret_cast<const float*>(base + o_wt);
  P.wdiag = nullptr;
  P.bhn = reinterpret_cast<const float*>(base + o_bhn);
  P.xin = reinterpret_cast<const float*>(base + o_u);
  P.buf1 = reinterpret_cast<float*>(base + o_buf1);
  P.flags = reinterpret_cast<unsigned*>(base + o_flags);
  P.agg = reinterpret_cast<float*>(base + o_agg);
  P.pref = reinterpret_cast<float*>(base + o_pref);
  P.ctrl = ctrl;
  P.args = args;
  P.hist = reinterpret_cast<float*>(base + o_hist);
  P.eps = 0.0f;
  P.D = D;
  P.d_in = d_in;
  P.T = T;
  P.B = B;
  P.ngroups = 1;
  P.nchunks = nchunks;
  P.tiles_per_group = (int)ntiles;
  P.agg_stride = 2 * G;
  P.pref_stride = G;
  P.cond = 0;
  if (ki.smem > 0)   // also below 48 KB: dynamic plus static shared memory above it needs the opt-in
    PN_STATIC_CUDA(cudaFuncSetAttribute(ki.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ki.smem));
  int per_sm = 0, nsm = 0;
  PN_STATIC_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ki.fn, ki.nt, ki.smem));
  PN_STATIC_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
  const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>((long long)per_sm * nsm, (long long)ntiles));
  for (long it = 0;; ++it) {
    void* kargs[] = {(void*)&P};
    PN_STATIC_CUDA(cudaLaunchKernel(ki.fn, dim3(grid), dim3(ki.nt), kargs, ki.smem, stream));
    PN_STATIC_CUDA(cudaMemcpyAsync(&hc, ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, stream));
    PN_STATIC_CUDA(cudaStreamSynchronize(stream));
    if (hc.status != kRunning) break;
    if (it > (long)max_iters + 2) return static_fail(PN_ERR_CUDA, "pn_eval_static: the loop did not stop");
  }
  {
    const Args* a_d = args;
    const Ctrl* c = ctrl;
    float* b1 = P.buf1;
    size_t n = nstate;
    int pass = 1;   // float32 storage: one pass
    void* kargs[] = {(void*)&a_d, (void*)&c, (void*)&b1, (void*)&n, (void*)&pass};
    const unsigned g = (unsigned)std::min<size_t>(n / 4 / 256 + 1, 148u * 16u);
    PN_STATIC_CUDA(cudaLaunchKernel(aux_kernel(2), dim3(g), dim3(256), kargs, 0, stream));
  }
  PN_STATIC_CUDA(cudaMemcpyAsync(&hc, ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, stream));
  PN_STATIC_CUDA(cudaStreamSynchronize(stream));
#undef PN_STATIC_CUDA
  if (iters_out) *iters_out = hc.final_iter;
  if (resid_out) *resid_out = hc.final_resid;
  if (hc.status == PN_ERR_TIMEOUT) return static_fail(PN_ERR_TIMEOUT, "pn_eval_static: a bounded device wait gave up");
  if (hc.status == PN_ERR_NONFINITE) return static_fail(PN_ERR_NONFINITE, "pn_eval_static: non-finite residual");
  return (pn_status)hc.status;
}

}  // extern "C"

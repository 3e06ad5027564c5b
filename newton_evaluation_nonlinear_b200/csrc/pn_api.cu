// pn_api.cu -- the C ABI of libpn (declared in include/pn.h).
//
// Host side of the solver: argument validation, weight packing, device buffer
// ownership, the CUDA graph that holds the device-side convergence loop (a
// conditional WHILE node around the fused iteration kernel), and the
// host-driven loop used when the device loop is switched off.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>
#include <vector>

#include "pn_aux.cuh"
#include "pn_dispatch.cuh"

using namespace pn;

namespace {

thread_local std::string g_create_error;

int padded_width(int D) {
  int dp = 4;
  while (dp < D) dp <<= 1;
  return dp;
}

int cell_R(int cell) { return cell == PN_CELL_GRU ? 3 : 1; }

struct Family {
  KInfo k[4];        // per mode (jacobi, picard, quasi, newton); fn == nullptr if unsupported
  int ngroups[4];
  int nchunks[4];
  int ntiles[4];     // ngroups * B * nchunks
  int grid[4];       // persistent CTAs: a multiple of ngroups, at most ntiles
  int resident[4];   // CTAs that can be resident at once (occupancy query x SM count)
  int run[4];        // chunks per ticket
};

}  // namespace

struct pn_ctx {
  int cell = 0, D = 0, d_in = 0, T = 0, B = 0, DP = 0, device = 0;
  float eps = 0.0f;
  cudaStream_t stream = nullptr;
  Family fam{};
  // device memory
  float* wt_diag = nullptr;    // [ngroups][DP][R*G] transposed recurrent weights
  float* wt_dense = nullptr;   // [DP][R*DP] transposed + [R][DP][DP] row-major
  float* wt_tc = nullptr;      // [W ; W_lo] rows of W_q, TF32-rounded, K-major core-matrix layout
  float* wt_tct = nullptr;     // banded [Z; W_hi; Z; W_lo; Z] (one-gate cells; no Z for D = 64), same layout
  float* wdiag = nullptr;      // [R][DP] diagonal entries W_q[c][c]
  float* bhn = nullptr;        // [DP]
  float* proj_w = nullptr;     // U [D][d_in] or W_ih [3D][d_in]
  float* proj_b = nullptr;     // b [D] or b_ih + [b_hr; b_hz; 0] [3D]
  float* xin = nullptr;        // hoisted step inputs [B][T][R*D]
  float* buf1 = nullptr;       // second iterate buffer [B][T][D]
  unsigned* flags = nullptr;
  float* agg = nullptr;
  float* pref = nullptr;
  size_t agg_floats = 0, pref_floats = 0, nflags = 0;        // what the selected tilings need
  size_t agg_cap = 0, pref_cap = 0, flags_cap = 0;            // what is allocated
  Ctrl* ctrl = nullptr;
  Args* args = nullptr;
  float* hist = nullptr;
  CUtensorMap* tmaps = nullptr;   // TMA descriptors of the tensor-core kernels: kTcMaps per mode (see IterParams)
  // wide one-gate cells (D = 128, 256): the tensor-core product Y = S W^T before each iteration
  bool wide_capable = false;
  float* wt_hi = nullptr;          // TF32 split of W, row-major [D][D]
  float* wt_lo = nullptr;
  float* ypre = nullptr;           // [B*T][D]
  CUtensorMap* wmaps = nullptr;    // kWideMaps: [0]/[1] S of iterate buffer 0 / 1, [2] W_hi, [3] W_lo, [4] Y
                                   // stores; the per-channel kernel's tiles: [5] Y, [6] step inputs, [7]/[8] s^(i)
  CUtensorMap* wmaps_h = nullptr;
  // the input projection on the tensor cores (N = R*D a multiple of 16 up to 256, d_in % 4 == 0)
  const void* proj_gemm = nullptr;
  size_t proj_gemm_smem = 0;
  float* proj_hi = nullptr;        // TF32 split of U (or W_ih), row-major [R*D][d_in]
  float* proj_lo = nullptr;
  CUtensorMap* pmaps = nullptr;    // kProjMaps: [0], [1] x, [2] U_hi, [3] U_lo, [4] u stores
  CUtensorMap* pmaps_h = nullptr;
  // host pinned mirrors
  Args* args_h = nullptr;
  Ctrl* ctrl_h = nullptr;
  CUtensorMap* tmaps_h = nullptr;
  // host-buffer evaluation staging (allocated on first pn_eval_host)
  float* hx = nullptr;
  float* hs0 = nullptr;
  float* hst = nullptr;
  // pipelined host-buffer evaluation (pn_eval_host_many): two staging slots, copy streams, events
  float* px[2] = {nullptr, nullptr};
  float* ps0[2] = {nullptr, nullptr};
  float* pst[2] = {nullptr, nullptr};
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_done[2] = {nullptr, nullptr}, ev_out[2] = {nullptr, nullptr};
  // graphs, one per mode, built on first use; the adaptive ones (one per starting mode) hold an
  // IF node per mode inside the WHILE node
  cudaGraph_t graph[4] = {nullptr, nullptr, nullptr, nullptr};
  cudaGraphExec_t exec[4] = {nullptr, nullptr, nullptr, nullptr};
  cudaGraph_t graph_ad[4] = {nullptr, nullptr, nullptr, nullptr};
  cudaGraphExec_t exec_ad[4] = {nullptr, nullptr, nullptr, nullptr};
  int* mode_hist_d = nullptr;  // [kHistCap] modes of the kept updates (adaptive graph)
  // options
  long long timeout_ns = 1000000000LL;
  int stall_ticket = -1;
  int newton_band = -1;        // PN_OPT_NEWTON_BAND
  int run_opt = 0;             // PN_OPT_RUN_LENGTH (0: automatic)
  int small_opt = 1;           // PN_OPT_SMALL_SOLVE
  KInfo small_k{nullptr, 0, 0, 0, 0, 0};   // the single-CTA Newton solve, when the problem fits
  float damping = 1.0f;        // pn_set_damping
  int store_fmt = 0;           // pn_set_storage: PN_STORE_F32 / _BF16 / _F16
  float store_until = 0.0f;
  float adapt_stall = -1.0f;   // pn_set_adaptive: < 0 off
  std::vector<int> mode_hist;  // mode of every update of the last evaluation
  int device_loop = 1;
  bool use_tma = false;        // pipelined bulk-copy kernels (D % 4 == 0, DP >= 32)
  bool tc_opt = true;          // PN_OPT_TENSOR_CORES
  bool use_tc = false;         // tensor-core matvec kernels (D == DP in {32, 64})
  bool tc_capable = false;
  long long evals = 0;
  int last_iters = -1;
  int last_kind = -1;          // kernel kind of the last iteration launch (look-back buffer format)
  std::string err;
};

namespace {

pn_status fail(pn_ctx* h, pn_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (h) h->err = buf;
  else g_create_error = buf;
  return st;
}

#define PN_CUDA(h, call)                                                                  \
  do {                                                                                    \
    cudaError_t e_ = (call);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return fail((h), e_ == cudaErrorMemoryAllocation ? PN_ERR_NOMEM : PN_ERR_CUDA,      \
                  "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__); \
  } while (0)

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
    else prev = -1;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

template <class T>
pn_status dalloc(pn_ctx* h, T** p, size_t count) {
  *p = nullptr;
  if (count == 0) count = 1;
  cudaError_t e = cudaMalloc((void**)p, count * sizeof(T));
  if (e != cudaSuccess) {
    *p = nullptr;
    return fail(h, PN_ERR_NOMEM, "cudaMalloc of %zu bytes failed: %s", count * sizeof(T),
                cudaGetErrorString(e));
  }
  return PN_OK;
}

void destroy_graphs(pn_ctx* h) {
  for (int m = 0; m < 4; ++m) {
    if (h->exec[m]) cudaGraphExecDestroy(h->exec[m]);
    if (h->graph[m]) cudaGraphDestroy(h->graph[m]);
    if (h->exec_ad[m]) cudaGraphExecDestroy(h->exec_ad[m]);
    if (h->graph_ad[m]) cudaGraphDestroy(h->graph_ad[m]);
    h->exec[m] = nullptr;
    h->graph[m] = nullptr;
    h->exec_ad[m] = nullptr;
    h->graph_ad[m] = nullptr;
  }
}

void free_all(pn_ctx* h) {
  destroy_graphs(h);
  if (h->mode_hist_d) cudaFree(h->mode_hist_d);
  h->mode_hist_d = nullptr;
  float** fbufs[] = {&h->wt_diag, &h->wt_dense, &h->wt_tc, &h->wt_tct, &h->wdiag, &h->bhn,    &h->proj_w,
                     &h->proj_b,  &h->xin,      &h->buf1,  &h->agg,    &h->pref,  &h->hist, &h->hx,
                     &h->hs0,     &h->hst,      &h->px[0], &h->px[1],  &h->ps0[0], &h->ps0[1], &h->pst[0],
                     &h->pst[1]};
  for (int q = 0; q < 2; ++q) {
    if (h->ev_in[q]) cudaEventDestroy(h->ev_in[q]);
    if (h->ev_done[q]) cudaEventDestroy(h->ev_done[q]);
    if (h->ev_out[q]) cudaEventDestroy(h->ev_out[q]);
    h->ev_in[q] = h->ev_done[q] = h->ev_out[q] = nullptr;
  }
  if (h->s_in) cudaStreamDestroy(h->s_in);
  if (h->s_out) cudaStreamDestroy(h->s_out);
  h->s_in = h->s_out = nullptr;
  for (float** p : fbufs) {
    if (*p) cudaFree(*p);
    *p = nullptr;
  }
  if (h->pmaps) cudaFree(h->pmaps);
  if (h->pmaps_h) cudaFreeHost(h->pmaps_h);
  h->pmaps = nullptr;
  h->pmaps_h = nullptr;
  for (float** p : {&h->wt_hi, &h->wt_lo, &h->ypre, &h->proj_hi, &h->proj_lo}) {
    if (*p) cudaFree(*p);
    *p = nullptr;
  }
  if (h->wmaps) cudaFree(h->wmaps);
  if (h->wmaps_h) cudaFreeHost(h->wmaps_h);
  h->wmaps = nullptr;
  h->wmaps_h = nullptr;
  if (h->flags) cudaFree(h->flags);
  if (h->tmaps) cudaFree(h->tmaps);
  if (h->tmaps_h) cudaFreeHost(h->tmaps_h);
  h->tmaps = nullptr;
  h->tmaps_h = nullptr;
  if (h->ctrl) cudaFree(h->ctrl);
  if (h->args) cudaFree(h->args);
  if (h->args_h) cudaFreeHost(h->args_h);
  if (h->ctrl_h) cudaFreeHost(h->ctrl_h);
  h->flags = nullptr;
  h->ctrl = nullptr;
  h->args = nullptr;
  h->args_h = nullptr;
  h->ctrl_h = nullptr;
}

// Recurrent weight block q of the cell, element [row][col] (rows, cols < D).
float w_block(const pn_ctx* h, const float* params, int q, int row, int col) {
  const int D = h->D;
  if (h->cell == PN_CELL_GRU) return params[(size_t)3 * D * h->d_in + ((size_t)q * D + row) * D + col];
  return params[(size_t)row * D + col];
}

IterParams make_params(const pn_ctx* h, int mode) {
  IterParams P{};
  const bool dense = (mode == PN_NEWTON);
  const int kind = h->fam.k[mode].kind;
  P.wt = (dense || kind == kKindDiagPost)
             ? h->wt_dense
             : (kind == kKindDiagTc ? h->wt_tc : (kind == kKindDiagTct ? h->wt_tct : h->wt_diag));
  P.wt_tc = h->wt_tc;
  P.ypre = h->ypre;
  P.mode_hist = h->mode_hist_d;
  P.wdiag = h->wdiag;
  P.bhn = h->bhn;
  P.xin = h->xin;
  P.buf1 = h->buf1;
  P.flags = h->flags;
  P.agg = h->agg;
  P.pref = h->pref;
  P.ctrl = h->ctrl;
  P.args = h->args;
  P.hist = h->hist;
  P.tmaps = h->tmaps ? h->tmaps + (size_t)mode * kTcMaps : nullptr;   // each mode's kernel has its own maps
  if (kind == kKindDiagPost) P.tmaps = h->wmaps ? h->wmaps + 5 : nullptr;   // its tile loads
  P.eps = h->eps;
  P.D = h->D;
  P.d_in = h->d_in;
  P.T = h->T;
  P.B = h->B;
  P.ngroups = h->fam.ngroups[mode];
  P.nchunks = h->fam.nchunks[mode];
  P.tiles_per_group = h->B * h->fam.nchunks[mode];
  P.run = h->fam.run[mode];
  P.tc = h->tc_opt ? 1 : 0;
  const int G = h->fam.k[mode].G;
  // the wide per-channel kernel keeps two (A, B) pairs per channel: the tile's and its first half's
  P.agg_stride = dense ? G * (G + 1) : (kind == kKindDiagPost ? 4 * G : 2 * G);
  P.pref_stride = G;
  P.cond = 0;
  return P;
}

unsigned grid_1d(size_t n, int threads, unsigned cap) {
  size_t g = (n + threads - 1) / threads;
  if (g < 1) g = 1;
  if (g > cap) g = cap;
  return (unsigned)g;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// Map over an fp32 array [B][T][cols] (one sequence after the other) whose
// box is box_rows steps of box_cols floats of one sequence.  Box elements
// outside the array (columns >= cols, steps < 0 or >= T) read as zero and are
// not written by stores, so a box never reaches into the next sequence.
bool encode_seq(CUtensorMap* m, const void* base, int cols, int T, int B, int box_cols, int box_rows, bool swizzle128) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn || !base) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)cols * sizeof(float), (cuuint64_t)cols * sizeof(float) * (cuuint64_t)T};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over a row-major fp32 matrix [rows][cols] whose box is box_rows x box_cols,
// 128-byte swizzled (the tensor cores' K-major operand layout for 32-float rows).
bool encode_2d_sw128(CUtensorMap* m, const void* base, int cols, long long rows, int box_cols, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn || !base) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * sizeof(float)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The wide product's maps for the current call: S of both iterate buffers (128 rows x 32
// floats per box) and W_hi, W_lo (D rows x 32 floats); then the per-channel kernel's tile loads
// (G channels of L steps of one sequence): Y (row b T + t - 1 read as step t - 1 of sequence b),
// the step inputs, and s^(i) of both iterate buffers (L + 1 steps, from t0 - 1).
bool encode_wide_maps(const pn_ctx* h, CUtensorMap* out, int G, int L) {
  const long long rows = (long long)h->B * h->T;
  const int D = h->D, T = h->T, B = h->B;
  const void* xs = (h->cell == PN_CELL_EULER_TANH) ? (const void*)h->args_h->x : (const void*)h->xin;
  return encode_2d_sw128(&out[0], h->args_h->states, D, rows, 32, 128) &&
         encode_2d_sw128(&out[1], h->buf1, D, rows, 32, 128) &&
         encode_2d_sw128(&out[2], h->wt_hi, D, D, 32, D) &&
         encode_2d_sw128(&out[3], h->wt_lo, D, D, 32, D) &&
         encode_2d_sw128(&out[4], h->ypre, D, rows, 32, 128) &&
         encode_seq(&out[5], h->ypre, D, T, B, G, L, false) &&
         encode_seq(&out[6], xs, D, T, B, G, L, false) &&
         encode_seq(&out[7], h->args_h->states, D, T, B, G, L + 1, false) &&
         encode_seq(&out[8], h->buf1, D, T, B, G, L + 1, false);
}

// Fills the pinned mirror of the maps of the tensor-core kernels for the
// buffers of the current call (iterate buffer 0 is the caller's states,
// buffer 1 is buf1; the step inputs are the hoisted projection, or x itself
// for the Euler cell):
//   [0], [1]  s^(i) loads from buffer 0 / 1: 32-float column halves of L+1
//             steps, 128-byte swizzled (the tensor cores' operand layout);
//   [2]       step-input loads: rows padded by 4 floats through the box width
//             for the row-major kernel, plain rows for the channel-major one;
//   [3], [4]  state stores into buffer 0 / 1, from rows padded by 4 floats
//             (row-major kernel).
bool encode_tc_maps(const pn_ctx* h, int mode, CUtensorMap* out) {
  const int L = h->fam.k[mode].L;
  const bool padded_x = (h->fam.k[mode].kind == kKindDiagTc);
  const int R = cell_R(h->cell);
  const int D = h->D, T = h->T, B = h->B, DP = h->DP;
  const void* xs = (h->cell == PN_CELL_EULER_TANH) ? (const void*)h->args_h->x : (const void*)h->xin;
  return encode_seq(&out[0], h->args_h->states, D, T, B, 32, L + 1, true) &&
         encode_seq(&out[1], h->buf1, D, T, B, 32, L + 1, true) &&
         encode_seq(&out[2], xs, R * D, T, B, padded_x ? R * DP + 4 : R * DP, L, false) &&
         encode_seq(&out[3], h->args_h->states, D, T, B, padded_x ? DP + 4 : DP, L, false) &&
         encode_seq(&out[4], h->buf1, D, T, B, padded_x ? DP + 4 : DP, L, false);
}

// Kernels that run before the loop: projection (tanh RNN, GRU) and init.
// The tensor-core GEMM for N output columns (the input projection's N = R*D).
template <int N>
void gemm_fn_of(const void** fn, size_t* smem) {
  *fn = (const void*)&wide_gemm_kernel<N>;
  *smem = (size_t)WideGemmCfg<N>::SMEM_BYTES;
}
bool gemm_for_width(int N, const void** fn, size_t* smem) {
  switch (N) {
    case 16: gemm_fn_of<16>(fn, smem); return true;
    case 32: gemm_fn_of<32>(fn, smem); return true;
    case 48: gemm_fn_of<48>(fn, smem); return true;
    case 64: gemm_fn_of<64>(fn, smem); return true;
    case 96: gemm_fn_of<96>(fn, smem); return true;
    case 128: gemm_fn_of<128>(fn, smem); return true;
    case 192: gemm_fn_of<192>(fn, smem); return true;
    case 256: gemm_fn_of<256>(fn, smem); return true;
    default: return false;
  }
}

struct PreLaunch {
  bool has_proj = false;
  dim3 proj_grid;
  int M = 0, N = 0, K = 0;
  dim3 init_grid{1, 1, 1};
  unsigned fin_grid = 1;
};

PreLaunch pre_launch(const pn_ctx* h) {
  PreLaunch p;
  p.has_proj = (h->cell != PN_CELL_EULER_TANH);
  p.M = h->B * h->T;
  p.N = cell_R(h->cell) * h->D;
  p.K = h->d_in;
  p.proj_grid = dim3((unsigned)((p.M + kProjTile - 1) / kProjTile), (unsigned)((p.N + kProjTile - 1) / kProjTile));
  const size_t n = (size_t)h->B * h->T * h->D;
  // init: about 8 CTAs per SM in all, whole sequences per grid row
  const unsigned gy = (unsigned)std::min(h->B, 65535);
  const unsigned gx = std::max(1u, std::min(grid_1d((size_t)h->T * h->D / 4 + 1, 256, 1u << 20), (148u * 8u) / gy));
  p.init_grid = dim3(gx, gy);
  p.fin_grid = grid_1d(n / 4 + 1, 256, 148u * 16u);
  return p;
}

// One launch of the tensor-core GEMM (wide_gemm_kernel<N>): the wide product Y = S W^T of an
// iteration, or the input projection u = x U^T + b.
struct GemmLaunch {
  const void* fn = nullptr;
  unsigned grid = 1;
  int nt = 256;
  size_t smem = 0;
  const CUtensorMap* maps = nullptr;
  float* y = nullptr;
  int rows = 0;
  int K = 0;
  const float* bias = nullptr;
  Ctrl* ctrl = nullptr;
  const Args* args = nullptr;
  void* kargs[7];
  void bind() {
    kargs[0] = (void*)&maps;
    kargs[1] = (void*)&y;
    kargs[2] = (void*)&rows;
    kargs[3] = (void*)&K;
    kargs[4] = (void*)&bias;
    kargs[5] = (void*)&ctrl;
    kargs[6] = (void*)&args;
  }
};

unsigned gemm_grid(const pn_ctx* h, int rows) {
  int nsm = 148;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, h->device);
  return (unsigned)std::max(1, std::min(nsm, (rows + 127) / 128));
}

// the wide product of `mode`'s iteration (ki.pre_fn)
void wide_launch(pn_ctx* h, const KInfo& ki, GemmLaunch& g) {
  g.fn = ki.pre_fn;
  g.nt = ki.pre_nt;
  g.smem = ki.pre_smem;
  g.maps = h->wmaps;
  g.y = h->ypre;
  g.rows = h->B * h->T;
  g.K = h->D;
  g.bias = nullptr;
  g.ctrl = h->ctrl;
  g.args = h->args;
  g.grid = gemm_grid(h, g.rows);
  g.bind();
}

// the input projection on the tensor cores (h->proj_gemm set at create)
void proj_launch(pn_ctx* h, GemmLaunch& g) {
  g.fn = h->proj_gemm;
  g.nt = WideGemmCfg<64>::NT;   // the same for every width
  g.smem = h->proj_gemm_smem;
  g.maps = h->pmaps;
  g.y = h->xin;
  g.rows = h->B * h->T;
  g.K = h->d_in;
  g.bias = h->proj_b;
  g.ctrl = h->ctrl;
  g.args = h->args;
  g.grid = gemm_grid(h, g.rows);
  g.bind();
}

pn_status build_graph(pn_ctx* h, int mode, bool adaptive = false) {
  if ((adaptive ? h->exec_ad[mode] : h->exec[mode])) return PN_OK;
  const PreLaunch pl = pre_launch(h);
  cudaGraph_t g = nullptr;
  PN_CUDA(h, cudaGraphCreate(&g, 0));
  cudaGraphNode_t prev = nullptr, node = nullptr;
  auto add_kernel = [&](cudaGraph_t graph, const void* fn, dim3 grid, dim3 block, size_t smem,
                        void** kargs, cudaGraphNode_t* dep, cudaGraphNode_t* out) -> cudaError_t {
    cudaKernelNodeParams kp{};
    kp.func = const_cast<void*>(fn);
    kp.gridDim = grid;
    kp.blockDim = block;
    kp.sharedMemBytes = (unsigned)smem;
    kp.kernelParams = kargs;
    kp.extra = nullptr;
    return cudaGraphAddKernelNode(out, graph, dep, dep ? 1 : 0, &kp);
  };
  cudaError_t e = cudaSuccess;
  // 1. input projection (FP32 kernel; the tensor-core one runs after init, below)
  const Args* a_d = h->args;
  GemmLaunch pg;
  if (pl.has_proj && !(h->proj_gemm && h->tc_opt)) {
    const float* w = h->proj_w;
    const float* bb = h->proj_b;
    float* o = h->xin;
    int M = pl.M, N = pl.N, K = pl.K;
    void* kargs[] = {(void*)&a_d, (void*)&w, (void*)&bb, (void*)&o, (void*)&M, (void*)&N, (void*)&K};
    e = add_kernel(g, (const void*)&proj_kernel, pl.proj_grid, dim3(256), 0, kargs, nullptr, &node);
    if (e != cudaSuccess) goto fail_graph;
    prev = node;
  }
  {
    // 2. init
    Ctrl* c = h->ctrl;
    int D = h->D, T = h->T, B = h->B;
    void* kargs[] = {(void*)&a_d, (void*)&c, (void*)&D, (void*)&T, (void*)&B};
    e = add_kernel(g, (const void*)&init_kernel, pl.init_grid, dim3(256), 0, kargs,
                   prev ? &prev : nullptr, &node);
    if (e != cudaSuccess) goto fail_graph;
    prev = node;
  }
  if (pl.has_proj && h->proj_gemm && h->tc_opt) {
    // 2b. input projection on the tensor cores (after init, which resets the error word it polls)
    proj_launch(h, pg);
    e = add_kernel(g, pg.fn, dim3(pg.grid), dim3(pg.nt), pg.smem, pg.kargs, &prev, &node);
    if (e != cudaSuccess) goto fail_graph;
    prev = node;
  }
  {
    // 3. WHILE (condition set to 0 by the iteration kernel's last CTA)
    cudaGraphConditionalHandle cond;
    e = cudaGraphConditionalHandleCreate(&cond, g, 1u, cudaGraphCondAssignDefault);
    if (e != cudaSuccess) goto fail_graph;
    cudaGraphNodeParams cp{};
    cp.type = cudaGraphNodeTypeConditional;
    cp.conditional.handle = cond;
    cp.conditional.type = cudaGraphCondTypeWhile;
    cp.conditional.size = 1;
    e = cudaGraphAddNode(&node, g, &prev, 1, &cp);
    if (e != cudaSuccess) goto fail_graph;
    cudaGraph_t body = cp.conditional.phGraph_out[0];
    // one iteration of mode m (its tensor-core product first, where it has one) into graph `gr`
    auto add_iteration = [&](cudaGraph_t gr, int m, const cudaGraphConditionalHandle* mc) -> cudaError_t {
      const KInfo& km = h->fam.k[m];
      IterParams P = make_params(h, m);
      P.cond = cond;
      if (mc)
        for (int q = 0; q < 4; ++q) P.mode_cond[q] = mc[q];
      void* kargs[] = {(void*)&P};
      cudaGraphNode_t knode, pnode;
      GemmLaunch wl;
      cudaGraphNode_t* dep = nullptr;
      cudaError_t err = cudaSuccess;
      if (km.pre_fn) {
        wide_launch(h, km, wl);
        err = add_kernel(gr, wl.fn, dim3(wl.grid), dim3(wl.nt), wl.smem, wl.kargs, nullptr, &pnode);
        if (err != cudaSuccess) return err;
        dep = &pnode;
      }
      err = add_kernel(gr, km.fn, dim3((unsigned)h->fam.grid[m]), dim3(km.nt), km.smem, kargs, dep, &knode);
      if (err != cudaSuccess || !km.coop) return err;
      if (h->fam.grid[m] > h->fam.resident[m]) return cudaErrorCooperativeLaunchTooLarge;
      cudaLaunchAttributeValue cv{};
      cv.cooperative = 1;
      return cudaGraphKernelNodeSetAttribute(knode, cudaLaunchAttributeCooperative, &cv);
    };
    if (!adaptive) {
      e = add_iteration(body, mode, nullptr);
      if (e != cudaSuccess) goto fail_graph;
    } else {
      // adaptive switching on the device: an IF node per mode, in the ladder's order, inside the
      // WHILE node; the starting mode's is on at every launch, and the last CTA of an iteration
      // turns on the one of the mode the next iteration runs in (a stronger mode is reached in the
      // same pass of the body, since its IF node comes later)
      cudaGraphConditionalHandle mc[4];
      for (int m = 0; m < 4 && e == cudaSuccess; ++m)
        e = cudaGraphConditionalHandleCreate(&mc[m], g, m == mode ? 1u : 0u, cudaGraphCondAssignDefault);
      if (e != cudaSuccess) goto fail_graph;
      cudaGraphNode_t bprev = nullptr;
      for (int m = 0; m < 4; ++m) {
        if (!h->fam.k[m].fn) continue;
        cudaGraphNodeParams ip{};
        ip.type = cudaGraphNodeTypeConditional;
        ip.conditional.handle = mc[m];
        ip.conditional.type = cudaGraphCondTypeIf;
        ip.conditional.size = 1;
        cudaGraphNode_t inode;
        e = cudaGraphAddNode(&inode, body, bprev ? &bprev : nullptr, bprev ? 1 : 0, &ip);
        if (e != cudaSuccess) goto fail_graph;
        e = add_iteration(ip.conditional.phGraph_out[0], m, mc);
        if (e != cudaSuccess) goto fail_graph;
        bprev = inode;
      }
    }
    prev = node;
  }
  {
    // 4. result copy (a narrow result in the caller's buffer first moves to the work buffer)
    const Ctrl* c = h->ctrl;
    float* b1 = h->buf1;
    size_t n = (size_t)h->B * h->T * h->D;
    for (int pass = (h->store_fmt != 0 ? 0 : 1); pass < 2; ++pass) {
      void* kargs[] = {(void*)&a_d, (void*)&c, (void*)&b1, (void*)&n, (void*)&pass};
      e = add_kernel(g, (const void*)&finish_kernel, dim3(pl.fin_grid), dim3(256), 0, kargs, &prev, &node);
      if (e != cudaSuccess) goto fail_graph;
      prev = node;
    }
  }
  e = cudaGraphInstantiate(adaptive ? &h->exec_ad[mode] : &h->exec[mode], g, 0);
  if (e != cudaSuccess) goto fail_graph;
  (adaptive ? h->graph_ad : h->graph)[mode] = g;
  return PN_OK;
fail_graph:
  cudaGraphDestroy(g);
  (adaptive ? h->exec_ad : h->exec)[mode] = nullptr;
  return fail(h, PN_ERR_CUDA, "building the CUDA graph for mode %d failed: %s", mode, cudaGetErrorString(e));
}

// The looping kernels' CTAs wait on one another (they meet at a grid barrier
// after every iteration; the channel-major kernel also starts each CTA with a
// static ticket, blockIdx.x, whose look-back may need any lower one), and so
// do those of the wide per-channel kernel (grid barriers between the phases of
// its scan), so all of their CTAs must be resident at once.  They are launched cooperatively:
// the runtime refuses a grid it cannot keep resident (another context's
// kernels, an MPS limit) instead of every wait running out its timeout.  The
// grid was sized from the occupancy query; the check below guards that sizing
// on the host.
pn_status launch_iter(pn_ctx* h, int mode, int persist = 0) {
  const KInfo& ki = h->fam.k[mode];
  IterParams P = make_params(h, mode);
  P.persist = persist;
  void* kargs[] = {(void*)&P};
  const unsigned grid = (unsigned)h->fam.grid[mode];
  if (ki.pre_fn) {   // the tensor-core product the iteration kernel reads
    GemmLaunch wl;
    wide_launch(h, ki, wl);
    PN_CUDA(h, cudaLaunchKernel(wl.fn, dim3(wl.grid), dim3(wl.nt), wl.kargs, wl.smem, h->stream));
  }
  if (!ki.loops && !ki.coop) {
    PN_CUDA(h, cudaLaunchKernel(ki.fn, dim3(grid), dim3(ki.nt), kargs, ki.smem, h->stream));
    return PN_OK;
  }
  if ((long long)grid > (long long)h->fam.resident[mode])
    return fail(h, PN_ERR_CUDA, "grid of %u CTAs exceeds the %d that can be resident", grid, h->fam.resident[mode]);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(ki.nt);
  cfg.dynamicSmemBytes = ki.smem;
  cfg.stream = h->stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  PN_CUDA(h, cudaLaunchKernelExC(&cfg, ki.fn, kargs));
  return PN_OK;
}

pn_status launch_pre(pn_ctx* h) {
  const PreLaunch pl = pre_launch(h);
  const Args* a_d = h->args;
  if (pl.has_proj && !(h->proj_gemm && h->tc_opt)) {
    const float* w = h->proj_w;
    const float* bb = h->proj_b;
    float* o = h->xin;
    int M = pl.M, N = pl.N, K = pl.K;
    void* kargs[] = {(void*)&a_d, (void*)&w, (void*)&bb, (void*)&o, (void*)&M, (void*)&N, (void*)&K};
    PN_CUDA(h, cudaLaunchKernel((const void*)&proj_kernel, pl.proj_grid, dim3(256), kargs, 0, h->stream));
  }
  Ctrl* c = h->ctrl;
  int D = h->D, T = h->T, B = h->B;
  void* kargs[] = {(void*)&a_d, (void*)&c, (void*)&D, (void*)&T, (void*)&B};
  PN_CUDA(h, cudaLaunchKernel((const void*)&init_kernel, pl.init_grid, dim3(256), kargs, 0, h->stream));
  if (pl.has_proj && h->proj_gemm && h->tc_opt) {
    GemmLaunch pg;
    proj_launch(h, pg);
    PN_CUDA(h, cudaLaunchKernel(pg.fn, dim3(pg.grid), dim3(pg.nt), pg.kargs, pg.smem, h->stream));
  }
  return PN_OK;
}

pn_status launch_finish(pn_ctx* h) {
  const PreLaunch pl = pre_launch(h);
  const Args* a_d = h->args;
  const Ctrl* c = h->ctrl;
  float* b1 = h->buf1;
  size_t n = (size_t)h->B * h->T * h->D;
  for (int pass = (h->store_fmt != 0 ? 0 : 1); pass < 2; ++pass) {
    void* kargs[] = {(void*)&a_d, (void*)&c, (void*)&b1, (void*)&n, (void*)&pass};
    PN_CUDA(h, cudaLaunchKernel((const void*)&finish_kernel, dim3(pl.fin_grid), dim3(256), kargs, 0, h->stream));
  }
  return PN_OK;
}

pn_status check_device_ptr(pn_ctx* h, const void* p, const char* name) {
  if (!p) return fail(h, PN_ERR_INVALID, "%s is NULL", name);
  if (((uintptr_t)p) & 15u) return fail(h, PN_ERR_INVALID, "%s must be 16-byte aligned", name);
  cudaPointerAttributes at{};
  cudaError_t e = cudaPointerGetAttributes(&at, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(h, PN_ERR_INVALID, "%s is not a CUDA pointer (%s)", name, cudaGetErrorString(e));
  }
  if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
    return fail(h, PN_ERR_INVALID, "%s must be device memory", name);
  if (at.type == cudaMemoryTypeDevice && at.device != h->device)
    return fail(h, PN_ERR_INVALID, "%s lives on device %d, the handle on device %d", name, at.device, h->device);
  return PN_OK;
}

pn_status validate_mode(pn_ctx* h, int mode, int max_iters, float tol) {
  if (mode < PN_JACOBI || mode > PN_NEWTON) return fail(h, PN_ERR_INVALID, "mode %d out of range", mode);
  if (!h->fam.k[mode].fn)
    return fail(h, PN_ERR_INVALID, "mode %d is not supported for D=%d (newton needs D <= %d)", mode, h->D,
                PN_MAX_D_NEWTON);
  if (max_iters < 0) return fail(h, PN_ERR_INVALID, "max_iters must be >= 0");
  if (!(tol >= 0.0f) || !std::isfinite(tol)) return fail(h, PN_ERR_INVALID, "tol must be finite and >= 0");
  return PN_OK;
}

// Prepares the look-back buffers for a launch of `mode`'s kernel.  Flags and
// tagged words carry the 30-bit launch epoch: clear them long before it
// wraps.  The tensor-core kernels read the aggregate and state buffers as
// tagged words, the others as plain floats: clear them when the format changes
// so no word of one format is ever read as the other.
pn_status prepare_lookback(pn_ctx* h, int mode) {
  const int kind = h->fam.k[mode].kind;
  const bool wrap = h->ctrl_h->epoch > (1u << 29);
  const bool format = (kind != h->last_kind) && (tagged_lookback(kind) || tagged_lookback(h->last_kind));
  if (wrap) {
    PN_CUDA(h, cudaMemsetAsync(h->flags, 0, h->nflags * sizeof(unsigned), h->stream));
    PN_CUDA(h, cudaMemsetAsync(&h->ctrl->epoch, 0, sizeof(unsigned), h->stream));
    h->ctrl_h->epoch = 0;
  }
  if (wrap || format) {
    PN_CUDA(h, cudaMemsetAsync(h->agg, 0, h->agg_floats * sizeof(float), h->stream));
    PN_CUDA(h, cudaMemsetAsync(h->pref, 0, h->pref_floats * sizeof(float), h->stream));
  }
  h->last_kind = kind;
  return PN_OK;
}

// Encodes and uploads the tensor maps when the mode runs a tensor-core kernel.
// The copy is ordered before the launches on the same stream; the pinned
// mirror is not touched again before the call's final synchronisation.
pn_status upload_tc_maps(pn_ctx* h, int mode) {
  if (h->proj_gemm && h->tc_opt && h->cell != PN_CELL_EULER_TANH) {   // x changes from call to call
    const long long rows = (long long)h->B * h->T;
    const int N = cell_R(h->cell) * h->D;
    if (!encode_2d_sw128(&h->pmaps_h[0], h->args_h->x, h->d_in, rows, 32, 128) ||
        !encode_2d_sw128(&h->pmaps_h[2], h->proj_hi, h->d_in, N, 32, N) ||
        !encode_2d_sw128(&h->pmaps_h[3], h->proj_lo, h->d_in, N, 32, N) ||
        (N % 32 == 0 && !encode_2d_sw128(&h->pmaps_h[4], h->xin, N, rows, 32, 128)))
      return fail(h, PN_ERR_CUDA, "encoding the input projection's tensor maps failed");
    h->pmaps_h[1] = h->pmaps_h[0];
    PN_CUDA(h, cudaMemcpyAsync(h->pmaps, h->pmaps_h, kProjMaps * sizeof(CUtensorMap), cudaMemcpyHostToDevice,
                               h->stream));
  }
  if (h->fam.k[mode].pre_fn) {
    if (!encode_wide_maps(h, h->wmaps_h, h->fam.k[mode].G, h->fam.k[mode].L))
      return fail(h, PN_ERR_CUDA, "encoding the wide product's tensor maps failed (D=%d, T=%d, B=%d)", h->D, h->T, h->B);
    PN_CUDA(h, cudaMemcpyAsync(h->wmaps, h->wmaps_h, kWideMaps * sizeof(CUtensorMap), cudaMemcpyHostToDevice,
                               h->stream));
    return PN_OK;
  }
  if (!tagged_lookback(h->fam.k[mode].kind)) return PN_OK;
  if (!encode_tc_maps(h, mode, h->tmaps_h + (size_t)mode * kTcMaps))
    return fail(h, PN_ERR_CUDA, "encoding the TMA tensor maps failed (D=%d, T=%d, B=%d)", h->D, h->T, h->B);
  PN_CUDA(h, cudaMemcpyAsync(h->tmaps + (size_t)mode * kTcMaps, h->tmaps_h + (size_t)mode * kTcMaps,
                             kTcMaps * sizeof(CUtensorMap), cudaMemcpyHostToDevice, h->stream));
  return PN_OK;
}

// One rung up the ladder of Jacobian approximations that the handle supports.
int stronger_mode(const pn_ctx* h, int mode) {
  int next = mode;
  if (mode == PN_JACOBI || mode == PN_PICARD) next = PN_QUASI;
  else if (mode == PN_QUASI) next = PN_NEWTON;
  return h->fam.k[next].fn ? next : mode;
}

// Adaptive switching (the page's §5.3: when the residual curve stalls, move to
// a more exact Jacobian approximation): a host loop, one launch per
// iteration.  Launch i measures r^(i) and applies update i in the current
// mode.  When r^(i) > stall * r^(i-1) (i >= 1) and a stronger mode exists,
// update i must use that mode: the control block's iteration index is set
// back to i and iteration i is launched again in the stronger mode (it reads
// the same s^(i) and overwrites s^(i+1) and r^(i)).
pn_status run_adaptive(pn_ctx* h, int mode) {
  pn_status st = launch_pre(h);
  if (st != PN_OK) return st;
  int cur = mode;
  float r_prev = 0.0f;
  // storage formats of iteration i's input and output, restored when iteration i runs again
  int fmt[2] = {h->store_fmt != 0, h->store_fmt != 0};
  for (int i = 0;; ++i) {
    float r = NAN;
    for (int attempt = 0; attempt < 2; ++attempt) {
      if (attempt == 1) PN_CUDA(h, cudaMemcpyAsync(&h->ctrl->fmt_in, fmt, sizeof fmt, cudaMemcpyHostToDevice, h->stream));
      if ((st = launch_iter(h, cur)) != PN_OK) return st;
      PN_CUDA(h, cudaMemcpyAsync(h->ctrl_h, h->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, h->stream));
      if (i < kHistCap) PN_CUDA(h, cudaMemcpyAsync(&r, h->hist + i, sizeof(float), cudaMemcpyDeviceToHost, h->stream));
      PN_CUDA(h, cudaStreamSynchronize(h->stream));
      if (h->ctrl_h->status != kRunning) return PN_OK;
      if (attempt == 1 || i == 0 || !(r > h->adapt_stall * r_prev)) break;
      const int next = stronger_mode(h, cur);
      if (next == cur) break;
      cur = next;
      if ((st = prepare_lookback(h, cur)) != PN_OK) return st;
      if ((st = upload_tc_maps(h, cur)) != PN_OK) return st;
      PN_CUDA(h, cudaMemcpyAsync(&h->ctrl->iter, &i, sizeof(int), cudaMemcpyHostToDevice, h->stream));
    }
    h->mode_hist.push_back(cur);
    r_prev = r;
    fmt[0] = h->ctrl_h->fmt_in;   // iteration i+1's formats, as the last launch left them
    fmt[1] = h->ctrl_h->fmt_out;
    if (i > h->args_h->max_iters + 2) return fail(h, PN_ERR_CUDA, "adaptive loop did not stop after max_iters launches");
  }
}

// The loop body shared by pn_eval and pn_eval_host: args already point at
// device buffers.
// The single-CTA Newton solve: projection, initial guess, iterations, stop rule and result copy.
pn_status launch_small(pn_ctx* h) {
  IterParams P = make_params(h, PN_NEWTON);
  const float* pw = h->proj_w;
  const float* pb = h->proj_b;
  void* kargs[] = {(void*)&P, (void*)&pw, (void*)&pb};
  PN_CUDA(h, cudaLaunchKernel(h->small_k.fn, dim3(1), dim3((unsigned)h->small_k.nt), kargs, h->small_k.smem,
                              h->stream));
  return PN_OK;
}

pn_status run_eval(pn_ctx* h, int mode, int* iters_out, float* resid_out) {
  pn_status st = prepare_lookback(h, mode);
  if (st != PN_OK) return st;
  const bool adaptive = h->adapt_stall >= 0.0f;
  const bool device_adaptive = adaptive && h->device_loop;   // the switching rule runs on the device
  h->args_h->use_cond = h->device_loop ? 1 : 0;
  h->args_h->newton_band = h->newton_band;
  h->args_h->damping = h->damping;
  h->args_h->store_fmt = h->store_fmt;
  h->args_h->store_until = h->store_until;
  h->args_h->adapt = device_adaptive ? 1 : 0;
  h->args_h->stall = h->adapt_stall;
  h->args_h->start_mode = mode;
  h->args_h->mode_ok = 0;
  for (int m = 0; m < 4; ++m)
    if (h->fam.k[m].fn) h->args_h->mode_ok |= 1 << m;
  PN_CUDA(h, cudaMemcpyAsync(h->args, h->args_h, sizeof(Args), cudaMemcpyHostToDevice, h->stream));
  if ((st = upload_tc_maps(h, mode)) != PN_OK) return st;
  if (device_adaptive) {   // the maps of every mode the ladder may reach
    for (int m = 0; m < 4; ++m)
      if (m != mode && h->fam.k[m].fn && (st = upload_tc_maps(h, m)) != PN_OK) return st;
  }
  h->mode_hist.clear();
  if (device_adaptive) {
    st = build_graph(h, mode, true);
    if (st != PN_OK) return st;
    PN_CUDA(h, cudaGraphLaunch(h->exec_ad[mode], h->stream));
  } else if (adaptive) {
    h->args_h->use_cond = 0;
    PN_CUDA(h, cudaMemcpyAsync(h->args, h->args_h, sizeof(Args), cudaMemcpyHostToDevice, h->stream));
    if ((st = run_adaptive(h, mode)) != PN_OK) return st;
    if ((st = launch_finish(h)) != PN_OK) return st;
  } else if (h->device_loop && mode == PN_NEWTON && h->small_k.fn) {
    // the whole solve in one launch of one CTA
    if ((st = launch_small(h)) != PN_OK) return st;
  } else if (h->device_loop && h->fam.k[mode].loops) {
    // the iteration kernel loops on the device: four plain launches, no graph needed
    if ((st = launch_pre(h)) != PN_OK) return st;
    if ((st = launch_iter(h, mode, 1)) != PN_OK) return st;
    if ((st = launch_finish(h)) != PN_OK) return st;
  } else if (h->device_loop) {
    st = build_graph(h, mode);
    if (st != PN_OK) return st;
    PN_CUDA(h, cudaGraphLaunch(h->exec[mode], h->stream));
  } else {
    st = launch_pre(h);
    if (st != PN_OK) return st;
    for (long it = 0;; ++it) {
      st = launch_iter(h, mode);
      if (st != PN_OK) return st;
      PN_CUDA(h, cudaMemcpyAsync(h->ctrl_h, h->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, h->stream));
      PN_CUDA(h, cudaStreamSynchronize(h->stream));
      if (h->ctrl_h->status != kRunning) break;
      if (it > (long)h->args_h->max_iters + 2)
        return fail(h, PN_ERR_CUDA, "host loop did not stop after max_iters launches");
    }
    st = launch_finish(h);
    if (st != PN_OK) return st;
  }
  PN_CUDA(h, cudaMemcpyAsync(h->ctrl_h, h->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, h->stream));
  PN_CUDA(h, cudaStreamSynchronize(h->stream));
  const Ctrl& c = *h->ctrl_h;
  if (device_adaptive) {
    // the modes of the kept updates, and the look-back format the last one left behind
    const int n = std::min(std::max(c.final_iter, 0), kHistCap);
    h->mode_hist.assign((size_t)n, 0);
    if (n > 0)
      PN_CUDA(h, cudaMemcpy(h->mode_hist.data(), h->mode_hist_d, (size_t)n * sizeof(int), cudaMemcpyDeviceToHost));
    if (c.cur_mode >= 0 && c.cur_mode < 4 && h->fam.k[c.cur_mode].fn) h->last_kind = h->fam.k[c.cur_mode].kind;
  }
  h->last_iters = c.final_iter;
  h->evals += 1;
  if (iters_out) *iters_out = c.final_iter;
  if (resid_out) *resid_out = c.final_resid;
  if (c.status == PN_ERR_TIMEOUT)
    return fail(h, PN_ERR_TIMEOUT, "a look-back wait gave up after %lld ns (tile ticket %d)",
                (long long)h->args_h->timeout_ns, c.timeout_ticket);
  if (c.status == PN_ERR_NONFINITE)
    return fail(h, PN_ERR_NONFINITE, "residual became non-finite at iteration %d", c.final_iter);
  if (c.status == kRunning) return fail(h, PN_ERR_CUDA, "the convergence loop did not finish");
  if (c.error)   // a bounded wait gave up after the stop rule had fired: the launch stalled
    return fail(h, PN_ERR_TIMEOUT, "a device wait gave up after the stop decision (%lld ns)",
                (long long)h->args_h->timeout_ns);
  h->err.clear();
  return (pn_status)c.status;
}

// Chooses the kernel of every mode for the handle's shape and options and
// records the tilings; grows the look-back buffer sizes to cover them.
pn_status select_kernels(pn_ctx* h) {
  const int D = h->D, T = h->T, B = h->B, DP = h->DP;
  for (int m = 0; m < 4; ++m) {
    // Damped Picard and damped GRU quasi-Newton run on the FP32 kernels: the row-major tensor-core
    // kernel releases s^(i)_t before its write-out, where damping needs it.
    // Narrow iterate storage runs on the plain FP32 kernels (element-wise loads and stores in the
    // storage format).
    const bool narrow = h->store_fmt != 0;
    // Newton: the tensor-core compositions take the one-gate cells at DP = 32, 64 unless a band is set
    const bool banded = h->newton_band >= 0 && h->newton_band < D - 1;
    const bool tc_m = (m == PN_NEWTON)
                          ? (h->tc_opt && h->cell != PN_CELL_GRU && (DP == 32 || DP == 64) && !banded)
                          : (h->use_tc && !narrow &&
                             !(h->damping != 1.0f && (m == PN_PICARD || (h->cell == PN_CELL_GRU && m == PN_QUASI))));
    KInfo ki = (m == PN_NEWTON && DP > PN_MAX_D_NEWTON) ? KInfo{nullptr, 0, 0, 0, 0, 0}
                                                         : lookup(h->cell, m, DP, h->use_tma && !narrow, tc_m);
    h->fam.k[m] = ki;
    if (!ki.fn) continue;
    h->fam.ngroups[m] = (m == PN_NEWTON) ? 1 : (D + ki.G - 1) / ki.G;
    if (h->fam.ngroups[m] > kMaxGroups)
      return fail(h, PN_ERR_INVALID, "D=%d needs %d channel groups (max %d)", D, h->fam.ngroups[m], kMaxGroups);
    // Set even below 48 KB: dynamic plus static shared memory above 48 KB needs the opt-in too
    // (dynamic 47.2 KB and 1 KB static leave no resident CTA without it).
    if (ki.smem > 0) {
      cudaError_t e = cudaFuncSetAttribute(ki.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ki.smem);
      if (e != cudaSuccess) return fail(h, PN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    if (ki.pre_fn && ki.pre_smem > 0) {
      cudaError_t e = cudaFuncSetAttribute(ki.pre_fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ki.pre_smem);
      if (e != cudaSuccess) return fail(h, PN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    int per_sm = 0, nsm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ki.fn, ki.nt, ki.smem) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess || per_sm < 1)
      return fail(h, PN_ERR_CUDA, "occupancy query failed for mode %d (D=%d)", m, D);
    // Kernels that take runs of chunks get one run per resident ticket-taker where the work allows
    // it: fewer tickets per sequence in flight, so fewer aggregates per look-back.
    const int chunks = (T + ki.L - 1) / ki.L;
    int run = 1;
    if (ki.tpc > 0) {
      const long long takers = (long long)per_sm * nsm * ki.tpc;
      run = (int)std::max<long long>(1, ((long long)chunks * B + takers - 1) / takers);
      if (h->run_opt > 0) run = std::min(h->run_opt, chunks);
    }
    h->fam.run[m] = run;
    h->fam.nchunks[m] = (chunks + run - 1) / run;
    h->fam.ntiles[m] = h->fam.ngroups[m] * B * h->fam.nchunks[m];
    const int ng = h->fam.ngroups[m];
    h->fam.resident[m] = per_sm * nsm;
    long long want = (long long)per_sm * nsm;
    want = std::max<long long>(ng, (want / ng) * ng);
    // kernels with several ticket-takers per CTA need only enough CTAs for the tickets
    const long long ctas_needed =
        ki.tpc > 0 ? ((long long)h->fam.ntiles[m] + ki.tpc - 1) / ki.tpc : (long long)h->fam.ntiles[m];
    h->fam.grid[m] = (int)std::max<long long>(1, std::min<long long>(want, ctas_needed));
    const size_t G = (size_t)ki.G;
    const size_t nt = (size_t)h->fam.ntiles[m];
    // the tensor-core kernels publish 64-bit tagged words: twice the floats
    const size_t wf = tagged_lookback(ki.kind) ? 2 : 1;
    const size_t aggf = nt * ((m == PN_NEWTON) ? G * (G + 1) : (ki.kind == kKindDiagPost ? 4 * G : 2 * G)) * wf;
    h->agg_floats = std::max(h->agg_floats, aggf);
    h->pref_floats = std::max(h->pref_floats, nt * G * wf);
    h->nflags = std::max(h->nflags, nt);
  }
  // Newton on a problem that fits in one SM's shared memory: the single-CTA solve
  h->small_k = KInfo{nullptr, 0, 0, 0, 0, 0};
  if (h->small_opt && DP <= 8 && h->fam.k[PN_NEWTON].fn) {
    const int dpp = DP <= 4 ? 4 : 8;
    const size_t bytes = small_smem_bytes(h->cell, dpp, B, T);
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device) == cudaSuccess &&
        bytes + 1024 <= (size_t)optin) {
      KInfo k = lookup_small(h->cell, dpp);
      // the attribute belongs to the function, not the handle: only ever raise it, so a handle
      // with a smaller problem never lowers the limit another handle's launches rely on
      cudaFuncAttributes fa{};
      if (k.fn && cudaFuncGetAttributes(&fa, k.fn) == cudaSuccess &&
          ((size_t)fa.maxDynamicSharedSizeBytes >= bytes ||
           cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess)) {
        k.smem = bytes;
        h->small_k = k;
      }
    }
    cudaGetLastError();
  }
  destroy_graphs(h);
  // a re-selection (an option changed the kernels or their tiling) may need larger look-back buffers
  // than create allocated: replace those (the stream has been synchronised), cleared like new ones.
  // If that fails, no mode has a kernel until a later re-selection succeeds.
  if (h->flags) {
    auto grow = [&](auto** buf, size_t need, size_t* cap, size_t elem) -> bool {
      if (need <= *cap) return true;
      void* nb = nullptr;
      if (cudaMalloc(&nb, need * elem) != cudaSuccess) return false;
      if (cudaMemset(nb, 0, need * elem) != cudaSuccess) {
        cudaFree(nb);
        return false;
      }
      cudaFree(*buf);
      *buf = static_cast<std::remove_reference_t<decltype(**buf)>*>(nb);
      *cap = need;
      return true;
    };
    if (!grow(&h->flags, h->nflags, &h->flags_cap, sizeof(unsigned)) ||
        !grow(&h->agg, h->agg_floats, &h->agg_cap, sizeof(float)) ||
        !grow(&h->pref, h->pref_floats, &h->pref_cap, sizeof(float))) {
      cudaGetLastError();
      for (int m = 0; m < 4; ++m) h->fam.k[m].fn = nullptr;
      return fail(h, PN_ERR_NOMEM, "growing the look-back buffers for the new tiling failed");
    }
  }
  return PN_OK;
}

}  // namespace

namespace pn {
// Sets the calling thread's handle-less error message (pn_last_error(NULL)).
void set_thread_error(const char* msg) { g_create_error = msg ? msg : ""; }

// Host stubs of the kernels around the convergence loop, for the other
// translation units of the library: 0 = projection, 1 = init, 2 = result copy.
const void* aux_kernel(int which) {
  switch (which) {
    case 0: return (const void*)&proj_kernel;
    case 1: return (const void*)&init_kernel;
    case 2: return (const void*)&finish_kernel;
    default: return nullptr;
  }
}
}  // namespace pn

extern "C" {

const char* pn_version(void) { return "libpn 0.1 (sm_100a)"; }

const char* pn_last_error(pn_handle h) {
  if (!h) return g_create_error.c_str();
  return h->err.c_str();
}

pn_status pn_create(pn_handle* out, pn_cell cell, int D, int d_in, int T, int B, const float* params,
                    size_t n_params, float eps, void* cuda_stream) {
  g_create_error.clear();
  if (!out) return fail(nullptr, PN_ERR_INVALID, "out is NULL");
  *out = nullptr;
  if (cell < PN_CELL_TANH_RNN || cell > PN_CELL_EULER_TANH) return fail(nullptr, PN_ERR_INVALID, "unknown cell %d", (int)cell);
  if (D < 1 || D > PN_MAX_D_DIAG) return fail(nullptr, PN_ERR_INVALID, "D=%d outside 1..%d", D, PN_MAX_D_DIAG);
  if (d_in < 1) return fail(nullptr, PN_ERR_INVALID, "d_in must be >= 1");
  if (cell == PN_CELL_EULER_TANH && d_in != D) return fail(nullptr, PN_ERR_INVALID, "the Euler cell needs d_in == D");
  if (T < 1 || B < 1) return fail(nullptr, PN_ERR_INVALID, "T and B must be >= 1");
  if ((long long)B * T > INT_MAX) return fail(nullptr, PN_ERR_INVALID, "B*T must fit in int");
  if (!params) return fail(nullptr, PN_ERR_INVALID, "params is NULL");
  if (!std::isfinite(eps)) return fail(nullptr, PN_ERR_INVALID, "eps must be finite");
  size_t need = 0;
  if (cell == PN_CELL_TANH_RNN) need = (size_t)D * D + (size_t)D * d_in + D;
  else if (cell == PN_CELL_GRU) need = 3 * (size_t)D * d_in + 3 * (size_t)D * D + 6 * (size_t)D;
  else need = (size_t)D * D;
  if (n_params != need) return fail(nullptr, PN_ERR_INVALID, "n_params=%zu, the cell needs %zu", n_params, need);

  pn_ctx* h = new pn_ctx();
  h->cell = cell;
  h->D = D;
  h->d_in = d_in;
  h->T = T;
  h->B = B;
  h->eps = eps;
  h->DP = padded_width(D);
  h->use_tma = (D % 4) == 0;
  h->tc_capable = (D == h->DP) && (D == 32 || (D == 64 && cell != PN_CELL_GRU));
  h->wide_capable = (D == h->DP) && (D == 128 || D == 256) && cell != PN_CELL_GRU;
  h->stream = (cudaStream_t)cuda_stream;
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return fail(nullptr, PN_ERR_CUDA, "no CUDA device");
  }
  const int R = cell_R(cell);
  const int DP = h->DP;
  const size_t BT = (size_t)B * T;

  // kernels and tilings; buffers are sized for both the tensor-core and the FP32 kernel sets
  {
    pn_status sk = PN_OK;
    for (int pass = 0; pass < 2 && sk == PN_OK; ++pass) {
      h->tc_opt = (pass == 1);
      h->use_tc = (pass == 0) ? false : (h->tc_capable || h->wide_capable);
      sk = select_kernels(h);
    }
    if (sk != PN_OK) {
      g_create_error = h->err;
      delete h;
      return sk;
    }
  }

  pn_status st = PN_OK;
#define PN_TRY(expr)           \
  do {                         \
    st = (expr);               \
    if (st != PN_OK) goto bad; \
  } while (0)
  {
    // weights, packed on the host
    const int Gd = lookup(cell, PN_QUASI, DP, h->use_tma, false).G;
    const int ng = (D + Gd - 1) / Gd;
    std::vector<float> wt((size_t)ng * DP * R * Gd, 0.0f);
    for (int g = 0; g < ng; ++g)
      for (int k = 0; k < D; ++k)
        for (int q = 0; q < R; ++q)
          for (int j = 0; j < Gd; ++j) {
            const int row = g * Gd + j;
            if (row < D) wt[(((size_t)g * DP + k) * R + q) * Gd + j] = w_block(h, params, q, row, k);
          }
    std::vector<float> wd((size_t)DP * R * DP + (size_t)R * DP * DP, 0.0f);
    for (int k = 0; k < D; ++k)
      for (int q = 0; q < R; ++q)
        for (int j = 0; j < D; ++j) wd[((size_t)k * R + q) * DP + j] = w_block(h, params, q, j, k);
    float* wr = wd.data() + (size_t)DP * R * DP;
    for (int q = 0; q < R; ++q)
      for (int i = 0; i < D; ++i)
        for (int k = 0; k < D; ++k) wr[((size_t)q * DP + i) * DP + k] = w_block(h, params, q, i, k);
    // tensor-core operand: rows n = q*DP + j of the R stacked blocks, K = DP inputs;
    // W (TF32-rounded) then W_lo = tf32(W - tf32(W)), each in the K-major core-matrix layout
    const int NN = R * DP;
    std::vector<float> wtc(2 * (size_t)NN * DP, 0.0f);
    for (int q = 0; q < R; ++q)
      for (int j = 0; j < D; ++j)
        for (int k = 0; k < D; ++k) {
          const float w = w_block(h, params, q, j, k);
          const float hi = tf32_round(w);
          const float lo = tf32_round(w - hi);
          const size_t off = kmajor_offset(q * DP + j, k, DP) / 4;
          wtc[off] = hi;
          wtc[(size_t)NN * DP + off] = lo;
        }
    // channel-major tensor-core operand (one-gate cells, D == DP): rows of the banded
    // buffer [Z(64-D); W_hi; Z(64-D); W_lo; Z(64-D)] (no zero rows for D = 64), K = DP,
    // K-major core-matrix layout; the kernel reads 64-row windows of it
    std::vector<float> wtct;
    if (h->tc_capable && cell != PN_CELL_GRU) {
      const int rows = 192 - DP;
      wtct.assign((size_t)rows * DP, 0.0f);
      for (int j = 0; j < D; ++j)
        for (int k = 0; k < D; ++k) {
          const float w = w_block(h, params, 0, j, k);
          const float hi = tf32_round(w);
          const float lo = tf32_round(w - hi);
          wtct[kmajor_offset((64 - DP) + j, k, DP) / 4] = hi;
          wtct[kmajor_offset((128 - DP) + j, k, DP) / 4] = lo;
        }
    }
    std::vector<float> wdg((size_t)R * DP, 0.0f);
    for (int q = 0; q < R; ++q)
      for (int j = 0; j < D; ++j) wdg[(size_t)q * DP + j] = w_block(h, params, q, j, j);
    std::vector<float> bhn(DP, 0.0f);
    std::vector<float> pw, pb;
    if (cell == PN_CELL_TANH_RNN) {
      pw.assign(params + (size_t)D * D, params + (size_t)D * D + (size_t)D * d_in);
      pb.assign(params + (size_t)D * D + (size_t)D * d_in, params + need);
    } else if (cell == PN_CELL_GRU) {
      const float* W_ih = params;
      const float* b_ih = params + 3 * (size_t)D * d_in + 3 * (size_t)D * D;
      const float* b_hh = b_ih + 3 * D;
      pw.assign(W_ih, W_ih + 3 * (size_t)D * d_in);
      pb.resize(3 * (size_t)D);
      for (int c = 0; c < D; ++c) {
        pb[c] = b_ih[c] + b_hh[c];               // r: b_ir + b_hr
        pb[D + c] = b_ih[D + c] + b_hh[D + c];   // z: b_iz + b_hz
        pb[2 * D + c] = b_ih[2 * D + c];         // n: b_in (b_hn stays inside r * (...))
        bhn[c] = b_hh[2 * D + c];
      }
    }
    PN_TRY(dalloc(h, &h->wt_diag, wt.size()));
    PN_TRY(dalloc(h, &h->wt_dense, wd.size()));
    PN_TRY(dalloc(h, &h->bhn, bhn.size()));
    PN_TRY(dalloc(h, &h->wt_tc, wtc.size()));
    PN_TRY(dalloc(h, &h->wdiag, wdg.size()));
    if (!wtct.empty()) {
      PN_TRY(dalloc(h, &h->wt_tct, wtct.size()));
      if (cudaMemcpy(h->wt_tct, wtct.data(), wtct.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess) {
        st = fail(h, PN_ERR_CUDA, "weight upload failed");
        goto bad;
      }
    }
    if (cudaMemcpy(h->wt_tc, wtc.data(), wtc.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(h->wdiag, wdg.data(), wdg.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(h->wt_diag, wt.data(), wt.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(h->wt_dense, wd.data(), wd.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(h->bhn, bhn.data(), bhn.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess) {
      st = fail(h, PN_ERR_CUDA, "weight upload failed");
      goto bad;
    }
    if (!pw.empty()) {
      PN_TRY(dalloc(h, &h->proj_w, pw.size()));
      PN_TRY(dalloc(h, &h->proj_b, pb.size()));
      PN_TRY(dalloc(h, &h->xin, BT * R * D));
      // the projection on the tensor cores where its shape allows: N = R*D a multiple of 16 up to
      // 256 and rows of x 16-byte aligned (d_in % 4 == 0)
      const void* gfn = nullptr;
      size_t gsmem = 0;
      if ((d_in % 4) == 0 && gemm_for_width(R * D, &gfn, &gsmem) &&
          cudaFuncSetAttribute(gfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem) == cudaSuccess) {
        const int N = R * D;
        std::vector<float> phi((size_t)N * d_in), plo((size_t)N * d_in);
        for (size_t e = 0; e < phi.size(); ++e) {
          phi[e] = tf32_round(pw[e]);
          plo[e] = tf32_round(pw[e] - phi[e]);
        }
        PN_TRY(dalloc(h, &h->proj_hi, phi.size()));
        PN_TRY(dalloc(h, &h->proj_lo, plo.size()));
        if (cudaMemcpy(h->proj_hi, phi.data(), phi.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
            cudaMemcpy(h->proj_lo, plo.data(), plo.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
            cudaMalloc((void**)&h->pmaps, kProjMaps * sizeof(CUtensorMap)) != cudaSuccess ||
            cudaMallocHost((void**)&h->pmaps_h, kProjMaps * sizeof(CUtensorMap)) != cudaSuccess) {
          st = fail(h, PN_ERR_NOMEM, "allocating the projection's tensor-core operands failed");
          goto bad;
        }
        h->proj_gemm = gfn;
        h->proj_gemm_smem = gsmem;
      } else {
        cudaGetLastError();
      }
      if (cudaMemcpy(h->proj_w, pw.data(), pw.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
          cudaMemcpy(h->proj_b, pb.data(), pb.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess) {
        st = fail(h, PN_ERR_CUDA, "weight upload failed");
        goto bad;
      }
    }
    PN_TRY(dalloc(h, &h->buf1, BT * D));
    if (h->wide_capable) {
      // the wide product's operands: W split into TF32 hi and lo parts (row-major, for the swizzled
      // tensor loads), its output Y, and the tensor maps
      std::vector<float> whi((size_t)D * D), wlo((size_t)D * D);
      for (int j = 0; j < D; ++j)
        for (int k = 0; k < D; ++k) {
          const float w = w_block(h, params, 0, j, k);
          whi[(size_t)j * D + k] = tf32_round(w);
          wlo[(size_t)j * D + k] = tf32_round(w - tf32_round(w));
        }
      PN_TRY(dalloc(h, &h->wt_hi, whi.size()));
      PN_TRY(dalloc(h, &h->wt_lo, wlo.size()));
      PN_TRY(dalloc(h, &h->ypre, BT * D));
      if (cudaMemcpy(h->wt_hi, whi.data(), whi.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
          cudaMemcpy(h->wt_lo, wlo.data(), wlo.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
          cudaMalloc((void**)&h->wmaps, kWideMaps * sizeof(CUtensorMap)) != cudaSuccess ||
          cudaMallocHost((void**)&h->wmaps_h, kWideMaps * sizeof(CUtensorMap)) != cudaSuccess) {
        st = fail(h, PN_ERR_NOMEM, "allocating the wide product's buffers failed");
        goto bad;
      }
    }
    PN_TRY(dalloc(h, &h->flags, h->nflags));
    PN_TRY(dalloc(h, &h->agg, h->agg_floats));
    PN_TRY(dalloc(h, &h->pref, h->pref_floats));
    h->flags_cap = h->nflags;
    h->agg_cap = h->agg_floats;
    h->pref_cap = h->pref_floats;
    PN_TRY(dalloc(h, &h->ctrl, 1));
    PN_TRY(dalloc(h, &h->args, 1));
    PN_TRY(dalloc(h, &h->hist, kHistCap));
    PN_TRY(dalloc(h, &h->mode_hist_d, kHistCap));
    if (cudaMemset(h->flags, 0, h->nflags * sizeof(unsigned)) != cudaSuccess ||
        cudaMemset(h->ctrl, 0, sizeof(Ctrl)) != cudaSuccess ||
        cudaMemset(h->hist, 0, kHistCap * sizeof(float)) != cudaSuccess) {
      st = fail(h, PN_ERR_CUDA, "memset failed");
      goto bad;
    }
    if (cudaMallocHost((void**)&h->args_h, sizeof(Args)) != cudaSuccess ||
        cudaMallocHost((void**)&h->ctrl_h, sizeof(Ctrl)) != cudaSuccess) {
      st = fail(h, PN_ERR_NOMEM, "pinned host allocation failed");
      goto bad;
    }
    memset(h->args_h, 0, sizeof(Args));
    memset(h->ctrl_h, 0, sizeof(Ctrl));
    if (h->tc_capable) {
      // the tensor-core kernels stage their tiles with TMA tensor maps; without
      // an encoder (or if the shape cannot be encoded) they are not used
      bool ok = cudaMalloc((void**)&h->tmaps, 4 * kTcMaps * sizeof(CUtensorMap)) == cudaSuccess &&
                cudaMallocHost((void**)&h->tmaps_h, 4 * kTcMaps * sizeof(CUtensorMap)) == cudaSuccess;
      if (ok) {
        h->args_h->states = h->buf1;   // probe encode with buffers of the same shapes
        h->args_h->x = (cell == PN_CELL_EULER_TANH) ? h->buf1 : nullptr;
        ok = encode_tc_maps(h, PN_QUASI, h->tmaps_h);
        h->args_h->states = nullptr;
        h->args_h->x = nullptr;
      }
      if (!ok) {
        cudaGetLastError();
        h->tc_capable = false;
        h->use_tc = false;
        PN_TRY(select_kernels(h));
      }
    }
    if (cudaDeviceSynchronize() != cudaSuccess) {
      st = fail(h, PN_ERR_CUDA, "device synchronisation after create failed");
      goto bad;
    }
  }
#undef PN_TRY
  *out = h;
  return PN_OK;
bad:
  g_create_error = h->err;
  free_all(h);
  delete h;
  return st;
}

pn_status pn_eval(pn_handle h, const float* x, const float* s0, pn_mode mode, int max_iters, float tol,
                  float* states, int* iters_out, float* resid_out) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  DeviceGuard dg(h->device);
  pn_status st = validate_mode(h, mode, max_iters, tol);
  if (st != PN_OK) return st;
  if ((st = check_device_ptr(h, x, "x")) != PN_OK) return st;
  if ((st = check_device_ptr(h, s0, "s0")) != PN_OK) return st;
  if ((st = check_device_ptr(h, states, "states")) != PN_OK) return st;
  Args& a = *h->args_h;
  a.x = x;
  a.s0 = s0;
  a.states = states;
  a.tol = tol;
  a.max_iters = max_iters;
  a.timeout_ns = h->timeout_ns;
  a.stall_ticket = h->stall_ticket;
  return run_eval(h, mode, iters_out, resid_out);
}

pn_status pn_eval_host(pn_handle h, const float* x_host, const float* s0_host, pn_mode mode, int max_iters,
                       float tol, float* states_host, int* iters_out, float* resid_out) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  DeviceGuard dg(h->device);
  pn_status st = validate_mode(h, mode, max_iters, tol);
  if (st != PN_OK) return st;
  if (!x_host || !s0_host || !states_host) return fail(h, PN_ERR_INVALID, "NULL host buffer");
  const size_t nx = (size_t)h->B * h->T * h->d_in;
  const size_t ns = (size_t)h->B * h->T * h->D;
  const size_t n0 = (size_t)h->B * h->D;
  if (!h->hx) {
    if ((st = dalloc(h, &h->hx, nx)) != PN_OK) return st;
    if ((st = dalloc(h, &h->hs0, n0)) != PN_OK) return st;
    if ((st = dalloc(h, &h->hst, ns)) != PN_OK) return st;
  }
  PN_CUDA(h, cudaMemcpyAsync(h->hx, x_host, nx * sizeof(float), cudaMemcpyHostToDevice, h->stream));
  PN_CUDA(h, cudaMemcpyAsync(h->hs0, s0_host, n0 * sizeof(float), cudaMemcpyHostToDevice, h->stream));
  Args& a = *h->args_h;
  a.x = h->hx;
  a.s0 = h->hs0;
  a.states = h->hst;
  a.tol = tol;
  a.max_iters = max_iters;
  a.timeout_ns = h->timeout_ns;
  a.stall_ticket = h->stall_ticket;
  st = run_eval(h, mode, iters_out, resid_out);
  if (st < 0 && st != PN_ERR_NONFINITE) return st;
  cudaError_t e = cudaMemcpyAsync(states_host, h->hst, ns * sizeof(float), cudaMemcpyDeviceToHost, h->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(h->stream);
  if (e != cudaSuccess) return fail(h, PN_ERR_CUDA, "copying states to the host failed: %s", cudaGetErrorString(e));
  return st;
}

pn_status pn_eval_host_many(pn_handle h, int n, const float* const* x_host, const float* const* s0_host,
                            pn_mode mode, int max_iters, float tol, float* const* states_host, int* iters_out,
                            float* resid_out) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  DeviceGuard dg(h->device);
  pn_status st = validate_mode(h, mode, max_iters, tol);
  if (st != PN_OK) return st;
  if (n < 0) return fail(h, PN_ERR_INVALID, "n = %d < 0", n);
  if (n == 0) return PN_OK;
  if (!x_host || !s0_host || !states_host) return fail(h, PN_ERR_INVALID, "NULL host buffer array");
  for (int k = 0; k < n; ++k)
    if (!x_host[k] || !s0_host[k] || !states_host[k]) return fail(h, PN_ERR_INVALID, "NULL host buffer (batch %d)", k);
  const size_t nx = (size_t)h->B * h->T * h->d_in;
  const size_t ns = (size_t)h->B * h->T * h->D;
  const size_t n0 = (size_t)h->B * h->D;
  if (!h->px[0]) {
    for (int q = 0; q < 2; ++q) {
      if ((st = dalloc(h, &h->px[q], nx)) != PN_OK) return st;
      if ((st = dalloc(h, &h->ps0[q], n0)) != PN_OK) return st;
      if ((st = dalloc(h, &h->pst[q], ns)) != PN_OK) return st;
      PN_CUDA(h, cudaEventCreateWithFlags(&h->ev_in[q], cudaEventDisableTiming));
      PN_CUDA(h, cudaEventCreateWithFlags(&h->ev_done[q], cudaEventDisableTiming));
      PN_CUDA(h, cudaEventCreateWithFlags(&h->ev_out[q], cudaEventDisableTiming));
    }
    PN_CUDA(h, cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking));
    PN_CUDA(h, cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking));
  }
  // batch k uses slot k & 1.  Its inputs go in on s_in once batch k-2's evaluation has read that
  // slot; it is evaluated on the handle's stream once they are in and batch k-2's states have
  // left the slot; its states go out on s_out once it is evaluated.
  auto copy_in = [&](int k) -> pn_status {
    const int q = k & 1;
    if (k >= 2) PN_CUDA(h, cudaStreamWaitEvent(h->s_in, h->ev_done[q], 0));
    PN_CUDA(h, cudaMemcpyAsync(h->px[q], x_host[k], nx * sizeof(float), cudaMemcpyHostToDevice, h->s_in));
    PN_CUDA(h, cudaMemcpyAsync(h->ps0[q], s0_host[k], n0 * sizeof(float), cudaMemcpyHostToDevice, h->s_in));
    PN_CUDA(h, cudaEventRecord(h->ev_in[q], h->s_in));
    return PN_OK;
  };
  pn_status result = PN_OK;
  if ((st = copy_in(0)) != PN_OK) return st;
  for (int k = 0; k < n; ++k) {
    const int q = k & 1;
    if (k + 1 < n && (st = copy_in(k + 1)) != PN_OK) return st;
    PN_CUDA(h, cudaStreamWaitEvent(h->stream, h->ev_in[q], 0));
    if (k >= 2) PN_CUDA(h, cudaStreamWaitEvent(h->stream, h->ev_out[q], 0));
    Args& a = *h->args_h;
    a.x = h->px[q];
    a.s0 = h->ps0[q];
    a.states = h->pst[q];
    a.tol = tol;
    a.max_iters = max_iters;
    a.timeout_ns = h->timeout_ns;
    a.stall_ticket = h->stall_ticket;
    int it = -1;
    float r = NAN;
    st = run_eval(h, mode, &it, &r);   // returns after the evaluation is complete
    if (iters_out) iters_out[k] = it;
    if (resid_out) resid_out[k] = r;
    if (st < 0 && st != PN_ERR_NONFINITE) {
      cudaStreamSynchronize(h->s_in);
      cudaStreamSynchronize(h->s_out);
      return st;
    }
    if (st != PN_OK && result == PN_OK) result = st;
    PN_CUDA(h, cudaEventRecord(h->ev_done[q], h->stream));
    PN_CUDA(h, cudaStreamWaitEvent(h->s_out, h->ev_done[q], 0));
    PN_CUDA(h, cudaMemcpyAsync(states_host[k], h->pst[q], ns * sizeof(float), cudaMemcpyDeviceToHost, h->s_out));
    PN_CUDA(h, cudaEventRecord(h->ev_out[q], h->s_out));
  }
  cudaError_t e = cudaStreamSynchronize(h->s_out);
  if (e == cudaSuccess) e = cudaStreamSynchronize(h->s_in);
  if (e != cudaSuccess) return fail(h, PN_ERR_CUDA, "copying states to the host failed: %s", cudaGetErrorString(e));
  return result;
}

pn_status pn_eval_windowed(pn_handle h, pn_handle tail, int T_total, const float* x, const float* s0,
                           pn_mode mode, int max_iters, float tol, float* states, int* iters_out,
                           float* resid_out, int* window_iters, int n_window_cap) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  DeviceGuard dg(h->device);
  pn_status st = validate_mode(h, mode, max_iters, tol);
  if (st != PN_OK) return st;
  if (T_total < 1) return fail(h, PN_ERR_INVALID, "T_total = %d < 1", T_total);
  if ((long long)h->B * T_total > INT_MAX) return fail(h, PN_ERR_INVALID, "B*T_total must fit in int");
  if (n_window_cap < 0 || (n_window_cap > 0 && !window_iters)) return fail(h, PN_ERR_INVALID, "bad window_iters array");
  const int W = h->T;
  const int rem = T_total % W;
  if (rem == 0 && tail) return fail(h, PN_ERR_INVALID, "tail must be NULL when the window length %d divides T_total", W);
  if (rem != 0) {
    if (!tail) return fail(h, PN_ERR_INVALID, "T_total %% %d = %d needs a tail handle", W, rem);
    if (tail == h || tail->T != rem || tail->cell != h->cell || tail->D != h->D || tail->d_in != h->d_in ||
        tail->B != h->B || tail->eps != h->eps || tail->device != h->device || tail->stream != h->stream)
      return fail(h, PN_ERR_INVALID, "tail handle must match (cell, D, d_in, B, eps, device, stream) with T = %d", rem);
    if ((st = validate_mode(tail, mode, max_iters, tol)) != PN_OK)
      return fail(h, st, "tail: %s", tail->err.c_str());
  }
  if ((st = check_device_ptr(h, x, "x")) != PN_OK) return st;
  if ((st = check_device_ptr(h, s0, "s0")) != PN_OK) return st;
  if ((st = check_device_ptr(h, states, "states")) != PN_OK) return st;
  const int B = h->B, D = h->D, d_in = h->d_in;
  if (!h->hx) {   // staging of one window, shared with pn_eval_host (the tail's windows are shorter)
    if ((st = dalloc(h, &h->hx, (size_t)B * W * d_in)) != PN_OK) return st;
    if ((st = dalloc(h, &h->hs0, (size_t)B * D)) != PN_OK) return st;
    if ((st = dalloc(h, &h->hst, (size_t)B * W * D)) != PN_OK) return st;
  }
  const size_t fsz = sizeof(float);
  const int nwin = (T_total + W - 1) / W;
  long long total = 0;
  float rmax = 0.0f;
  pn_status result = PN_OK;
  for (int w = 0; w < nwin; ++w) {
    const int t0 = w * W;
    const int L = std::min(W, T_total - t0);
    pn_ctx* hh = (L == W) ? h : tail;
    // x[:, t0:t0+L, :] -> staging [B][L][d_in]
    PN_CUDA(h, cudaMemcpy2DAsync(h->hx, (size_t)L * d_in * fsz, x + (size_t)t0 * d_in, (size_t)T_total * d_in * fsz,
                                 (size_t)L * d_in * fsz, (size_t)B, cudaMemcpyDeviceToDevice, h->stream));
    // the window's initial state: s0, or states[:, t0-1, :]
    if (w == 0)
      PN_CUDA(h, cudaMemcpyAsync(h->hs0, s0, (size_t)B * D * fsz, cudaMemcpyDeviceToDevice, h->stream));
    else
      PN_CUDA(h, cudaMemcpy2DAsync(h->hs0, (size_t)D * fsz, states + (size_t)(t0 - 1) * D, (size_t)T_total * D * fsz,
                                   (size_t)D * fsz, (size_t)B, cudaMemcpyDeviceToDevice, h->stream));
    Args& a = *hh->args_h;
    a.x = h->hx;
    a.s0 = h->hs0;
    a.states = h->hst;
    a.tol = tol;
    a.max_iters = max_iters;
    a.timeout_ns = hh->timeout_ns;
    a.stall_ticket = hh->stall_ticket;
    int it = -1;
    float r = NAN;
    st = run_eval(hh, mode, &it, &r);   // returns after the window is solved (stream synchronised)
    if (st < 0 && st != PN_ERR_NONFINITE) {
      if (hh != h) return fail(h, st, "window %d (tail): %s", w, tail->err.c_str());
      return st;
    }
    // staging [B][L][D] -> states[:, t0:t0+L, :]
    PN_CUDA(h, cudaMemcpy2DAsync(states + (size_t)t0 * D, (size_t)T_total * D * fsz, h->hst, (size_t)L * D * fsz,
                                 (size_t)L * D * fsz, (size_t)B, cudaMemcpyDeviceToDevice, h->stream));
    if (w < n_window_cap) window_iters[w] = it;
    total += it;
    if (r != r) rmax = r;                 // NaN sticks
    else if (rmax == rmax && r > rmax) rmax = r;
    if (st == PN_ERR_NONFINITE) {
      result = PN_ERR_NONFINITE;
      if (hh != h) fail(h, st, "window %d (tail): %s", w, tail->err.c_str());
      else fail(h, st, "window %d: %s", w, std::string(h->err).c_str());
      break;
    }
    if (st == PN_NOT_CONVERGED) result = PN_NOT_CONVERGED;
  }
  cudaError_t e = cudaStreamSynchronize(h->stream);
  if (e != cudaSuccess) return fail(h, PN_ERR_CUDA, "windowed solve: %s", cudaGetErrorString(e));
  if (iters_out) *iters_out = (int)std::min<long long>(total, INT_MAX);
  if (resid_out) *resid_out = rmax;
  if (result != PN_ERR_NONFINITE) h->err.clear();
  return result;
}

pn_status pn_get_residual_history(pn_handle h, float* out, int n, int* n_written) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  if (n < 0 || (n > 0 && !out)) return fail(h, PN_ERR_INVALID, "bad output buffer");
  DeviceGuard dg(h->device);
  int avail = h->last_iters < 0 ? 0 : std::min(h->last_iters + 1, kHistCap);
  int cnt = std::min(n, avail);
  if (cnt > 0) {
    PN_CUDA(h, cudaMemcpyAsync(out, h->hist, cnt * sizeof(float), cudaMemcpyDeviceToHost, h->stream));
    PN_CUDA(h, cudaStreamSynchronize(h->stream));
  }
  if (n_written) *n_written = cnt;
  return PN_OK;
}

pn_status pn_time_iterations(pn_handle h, pn_mode mode, int n_launches, float* avg_ms) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  if (n_launches < 1 || !avg_ms) return fail(h, PN_ERR_INVALID, "n_launches must be >= 1 and avg_ms non-NULL");
  DeviceGuard dg(h->device);
  pn_status st = validate_mode(h, mode, 0, 0.0f);
  if (st != PN_OK) return st;
  if (!h->args_h->states) return fail(h, PN_ERR_INVALID, "call pn_eval on this handle first");
  // Kernels that iterate on the device (the graph runs them as one launch per evaluation) are
  // timed the same way: one launch that runs n_launches iterations (a tolerance below zero never
  // stops it early, max_iters ends it), average = elapsed / n_launches.  The others: n_launches
  // launches that each re-evaluate the same iterate (r <= +inf stops after one iteration).
  const bool small = (mode == PN_NEWTON && h->small_k.fn && h->device_loop);
  if (small) {
    // the single-CTA solve: one launch of n_launches residual evaluations (n_launches - 1 updates)
    h->args_h->tol = -1.0f;
    h->args_h->max_iters = n_launches - 1;
    h->args_h->use_cond = 0;
    PN_CUDA(h, cudaMemcpyAsync(h->args, h->args_h, sizeof(Args), cudaMemcpyHostToDevice, h->stream));
    cudaEvent_t e0, e1;
    PN_CUDA(h, cudaEventCreate(&e0));
    PN_CUDA(h, cudaEventCreate(&e1));
    cudaError_t ce = cudaEventRecord(e0, h->stream);
    st = (ce == cudaSuccess) ? launch_small(h) : PN_OK;
    if (ce == cudaSuccess) ce = cudaEventRecord(e1, h->stream);
    if (ce == cudaSuccess) ce = cudaEventSynchronize(e1);
    float ms = 0.0f;
    if (ce == cudaSuccess) ce = cudaEventElapsedTime(&ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (st != PN_OK) return st;
    if (ce != cudaSuccess) return fail(h, PN_ERR_CUDA, "timing failed: %s", cudaGetErrorString(ce));
    PN_CUDA(h, cudaMemcpy(h->ctrl_h, h->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost));
    if (h->ctrl_h->final_iter != n_launches - 1)
      return fail(h, PN_ERR_CUDA, "timing run stopped at iteration %d, expected %d", h->ctrl_h->final_iter,
                  n_launches - 1);
    *avg_ms = ms / (float)n_launches;
    return PN_OK;
  }
  const bool looping = h->fam.k[mode].loops;
  if (looping) {
    PN_CUDA(h, cudaMemcpy(h->ctrl_h, h->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost));
    const long long last = (long long)h->ctrl_h->iter + n_launches - 1;
    if (last > INT_MAX) return fail(h, PN_ERR_INVALID, "n_launches too large");
    h->args_h->tol = -1.0f;
    h->args_h->max_iters = (int)last;
    const int running = kRunning, no_error = 0;
    PN_CUDA(h, cudaMemcpy(&h->ctrl->status, &running, sizeof running, cudaMemcpyHostToDevice));
    PN_CUDA(h, cudaMemcpy(&h->ctrl->error, &no_error, sizeof no_error, cudaMemcpyHostToDevice));
  } else {
    h->args_h->tol = INFINITY;
    h->args_h->max_iters = INT_MAX;
  }
  h->args_h->use_cond = 0;
  if ((st = prepare_lookback(h, mode)) != PN_OK) return st;
  PN_CUDA(h, cudaMemcpyAsync(h->args, h->args_h, sizeof(Args), cudaMemcpyHostToDevice, h->stream));
  if ((st = upload_tc_maps(h, mode)) != PN_OK) return st;
  cudaEvent_t e0, e1;
  PN_CUDA(h, cudaEventCreate(&e0));
  PN_CUDA(h, cudaEventCreate(&e1));
  st = PN_OK;
  cudaError_t ce = cudaEventRecord(e0, h->stream);
  if (looping) st = launch_iter(h, mode, 1);
  for (int i = 0; !looping && i < n_launches && ce == cudaSuccess && st == PN_OK; ++i) st = launch_iter(h, mode);
  if (ce == cudaSuccess) ce = cudaEventRecord(e1, h->stream);
  if (ce == cudaSuccess) ce = cudaEventSynchronize(e1);
  float ms = 0.0f;
  if (ce == cudaSuccess) ce = cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (st != PN_OK) return st;
  if (ce != cudaSuccess) return fail(h, PN_ERR_CUDA, "timing failed: %s", cudaGetErrorString(ce));
  PN_CUDA(h, cudaMemcpy(h->ctrl_h, h->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost));
  if (h->ctrl_h->error) return fail(h, PN_ERR_TIMEOUT, "a look-back wait gave up during timing");
  if (looping && h->ctrl_h->final_iter != (int)h->args_h->max_iters)
    return fail(h, PN_ERR_CUDA, "timing run stopped at iteration %d, expected %d", h->ctrl_h->final_iter,
                h->args_h->max_iters);
  *avg_ms = ms / (float)n_launches;
  return PN_OK;
}

pn_status pn_get_stats(pn_handle h, pn_stats* out) {
  if (!h || !out) return fail(h, PN_ERR_INVALID, "NULL argument");
  DeviceGuard dg(h->device);
  PN_CUDA(h, cudaStreamSynchronize(h->stream));
  PN_CUDA(h, cudaMemcpy(h->ctrl_h, h->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost));
  out->iteration_launches = (long long)h->ctrl_h->launches;
  out->iteration_ns = (long long)h->ctrl_h->kernel_ns;
  out->evals = h->evals;
  return PN_OK;
}

pn_status pn_reset_stats(pn_handle h) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  DeviceGuard dg(h->device);
  PN_CUDA(h, cudaStreamSynchronize(h->stream));
  unsigned long long z[2] = {0ull, 0ull};
  PN_CUDA(h, cudaMemcpy(&h->ctrl->kernel_ns, z, 2 * sizeof(unsigned long long), cudaMemcpyHostToDevice));
  h->evals = 0;
  return PN_OK;
}

pn_status pn_set_option(pn_handle h, pn_option opt, long long value) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  switch (opt) {
    case PN_OPT_WAIT_TIMEOUT_NS:
      if (value < 1000) return fail(h, PN_ERR_INVALID, "timeout must be >= 1000 ns");
      h->timeout_ns = value;
      return PN_OK;
    case PN_OPT_DEBUG_STALL_TICKET:
      if (value < -1 || value > INT_MAX) return fail(h, PN_ERR_INVALID, "bad ticket");
      h->stall_ticket = (int)value;
      return PN_OK;
    case PN_OPT_NEWTON_BAND: {
      if (value < -1 || value > INT_MAX) return fail(h, PN_ERR_INVALID, "band must be -1 or >= 0");
      const bool was = h->newton_band >= 0 && h->newton_band < h->D - 1;
      h->newton_band = (int)value;
      if (was != (h->newton_band >= 0 && h->newton_band < h->D - 1)) {   // Newton's kernel choice changes
        DeviceGuard dg(h->device);
        if (h->stream) cudaStreamSynchronize(h->stream);
        else cudaDeviceSynchronize();
        return select_kernels(h);
      }
      return PN_OK;
    }
    case PN_OPT_RUN_LENGTH: {
      if (value < 0 || value > INT_MAX) return fail(h, PN_ERR_INVALID, "run length must be >= 0");
      if ((int)value == h->run_opt) return PN_OK;
      h->run_opt = (int)value;
      DeviceGuard dg(h->device);
      if (h->stream) cudaStreamSynchronize(h->stream);
      else cudaDeviceSynchronize();
      return select_kernels(h);
    }
    case PN_OPT_SMALL_SOLVE: {
      if (value != 0 && value != 1) return fail(h, PN_ERR_INVALID, "small-solve option is 0 or 1");
      if ((int)value == h->small_opt) return PN_OK;
      h->small_opt = (int)value;
      DeviceGuard dg(h->device);
      if (h->stream) cudaStreamSynchronize(h->stream);
      else cudaDeviceSynchronize();
      return select_kernels(h);
    }
    case PN_OPT_DEVICE_LOOP:
      if (value != 0 && value != 1) return fail(h, PN_ERR_INVALID, "device loop option is 0 or 1");
      h->device_loop = (int)value;
      return PN_OK;
    case PN_OPT_TENSOR_CORES: {
      if (value != 0 && value != 1) return fail(h, PN_ERR_INVALID, "tensor-core option is 0 or 1");
      const bool want = (value == 1) && (h->tc_capable || h->wide_capable);
      if (want == h->use_tc && (value == 1) == h->tc_opt) return PN_OK;
      DeviceGuard dg(h->device);
      if (h->stream) cudaStreamSynchronize(h->stream);
      else cudaDeviceSynchronize();
      h->tc_opt = (value == 1);
      h->use_tc = want;
      return select_kernels(h);
    }
  }
  return fail(h, PN_ERR_INVALID, "unknown option %d", (int)opt);
}

pn_status pn_set_adaptive(pn_handle h, float stall) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  if (std::isnan(stall) || std::isinf(stall)) return fail(h, PN_ERR_INVALID, "stall ratio must be finite");
  h->adapt_stall = stall < 0.0f ? -1.0f : stall;
  return PN_OK;
}

pn_status pn_get_mode_history(pn_handle h, int* out, int n, int* n_written) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  if (n < 0 || (n > 0 && !out)) return fail(h, PN_ERR_INVALID, "bad output buffer");
  const int cnt = std::min(n, (int)h->mode_hist.size());
  for (int k = 0; k < cnt; ++k) out[k] = h->mode_hist[k];
  if (n_written) *n_written = cnt;
  return PN_OK;
}

pn_status pn_set_damping(pn_handle h, float lambda) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  if (!(lambda > 0.0f && lambda <= 1.0f)) return fail(h, PN_ERR_INVALID, "damping must be in (0, 1]");
  const bool was = h->damping != 1.0f;
  h->damping = lambda;
  if (was != (lambda != 1.0f) && h->use_tc) {   // the kernel choice of damped Picard / GRU quasi changes
    DeviceGuard dg(h->device);
    if (h->stream) cudaStreamSynchronize(h->stream);
    else cudaDeviceSynchronize();
    return select_kernels(h);
  }
  return PN_OK;
}

pn_status pn_set_storage(pn_handle h, int format, float store_until) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  if (format < PN_STORE_F32 || format > PN_STORE_F16) return fail(h, PN_ERR_INVALID, "unknown storage format %d", format);
  if (std::isnan(store_until)) return fail(h, PN_ERR_INVALID, "store_until must not be NaN");
  const bool changed = (format != 0) != (h->store_fmt != 0);
  h->store_fmt = format;
  h->store_until = store_until;
  if (changed) {   // the kernel choice and the result copy of the graphs change
    DeviceGuard dg(h->device);
    if (h->stream) cudaStreamSynchronize(h->stream);
    else cudaDeviceSynchronize();
    return select_kernels(h);
  }
  return PN_OK;   // the graphs read the format and the threshold from the per-call arguments
}

pn_status pn_set_stream(pn_handle h, void* cuda_stream) {
  if (!h) return fail(nullptr, PN_ERR_INVALID, "handle is NULL");
  h->stream = (cudaStream_t)cuda_stream;
  return PN_OK;
}

pn_status pn_activation(int which, const float* x, float* y, long long n, void* cuda_stream) {
  if (which != 0 && which != 1) return fail(nullptr, PN_ERR_INVALID, "which must be 0 (tanh) or 1 (sigmoid)");
  if (n < 0 || (n > 0 && (!x || !y))) return fail(nullptr, PN_ERR_INVALID, "bad arrays");
  if (n == 0) return PN_OK;
  cudaStream_t st = (cudaStream_t)cuda_stream;
  const unsigned grid = (unsigned)std::min<long long>((n + 255) / 256, 148LL * 32);
  void* kargs[] = {(void*)&which, (void*)&x, (void*)&y, (void*)&n};
  cudaError_t e = cudaLaunchKernel((const void*)&activation_kernel, dim3(grid), dim3(256), kargs, 0, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(nullptr, PN_ERR_CUDA, "activation kernel failed: %s", cudaGetErrorString(e));
  return PN_OK;
}

int pn_dim(pn_handle h, int which) {
  if (!h) return -1;
  switch (which) {
    case 0: return h->D;
    case 1: return h->d_in;
    case 2: return h->T;
    case 3: return h->B;
    case 4: return h->cell;
    case 5 + PN_JACOBI:
    case 5 + PN_PICARD:
    case 5 + PN_QUASI:
    case 5 + PN_NEWTON:
      if (which - 5 == PN_NEWTON && h->small_k.fn && h->device_loop && h->adapt_stall < 0.0f) return 2;
      return h->fam.k[which - 5].loops ? 1 : 0;
    default: return -1;
  }
}

void pn_destroy(pn_handle h) {
  if (!h) return;
  {
    DeviceGuard dg(h->device);
    if (h->stream) cudaStreamSynchronize(h->stream);
    else cudaDeviceSynchronize();
    free_all(h);
  }
  delete h;
}

}  // extern "C"

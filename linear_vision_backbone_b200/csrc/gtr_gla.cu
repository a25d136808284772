// gtr_gla.cu -- the C ABI of include/gtr_gla.h and the host side of every
// kernel launch.  Argument checks, the segment plan, workspace management and
// the stage sequence K2 (summary) -> K3 (boundary scan) -> K4 (output) of the
// chunkwise operator (GTR article, 方法详解 §4) live here; the kernels live in
// the included .cuh files, all in this one translation unit (the Spatial
// SwiGLU block is the library's other one, sswiglu.cu).
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "gtr_gla.h"
#include "common.cuh"
#include "gate_kernels.cuh"
#include "simt_kernels.cuh"
#include "scan_kernel.cuh"
#include "tc_kernels.cuh"
#include "tc128_kernels.cuh"
#include "gate_tc.cuh"
#include "mixer_proj.cuh"

namespace {

using namespace gtr;

std::atomic<int> g_path_setting{GTR_PATH_AUTO};
std::mutex g_mu;
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
void* g_user_ws[kMaxDevices];
size_t g_user_ws_bytes[kMaxDevices];
std::map<std::pair<int, void*>, std::pair<void*, size_t>> g_ws;   // (device, stream) -> buffer

bool valid_head_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool valid_chunk(int c) { return c == 16 || c == 32 || c == 64 || c == 128; }
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return GTR_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return GTR_ERR_UNSUPPORTED;
  return GTR_OK;
}

int sm_count(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

// Plan of one gtr_gla_fwd call: chunk length, segments (runs of consecutive
// chunks one block of K2/K4 walks through; segment s of nseg covers chunks
// [s nc / nseg, (s+1) nc / nseg)) and workspace layout.
struct Plan {
  int B, H, gh, gw, T, dk, dv, dir, chunk, dtype;
  int dev;
  int path;        // GTR_PATH_SIMT or GTR_PATH_TC
  int nc;          // chunks per sequence
  int nseg;        // segments per sequence
  int seg_chunks;  // chunks in the longest segment
  size_t offA;     // byte offset of the segment decay factors in the workspace
  size_t ws_bytes;
};

// Segment length for the multi-wave case: minimise (rounds of resident
// blocks) x (chunks per block); on ties take the longer segment, which moves
// fewer boundary states through memory.
int plan_segments(long long bh, int nc, long long slots) {
  int best = 1;
  long long best_cost = -1;
  const int mmax = nc < 65536 ? nc : 65536;
  for (int m = 1; m <= mmax; ++m) {
    const long long units = bh * ((nc + m - 1) / m);
    const long long cost = ((units + slots - 1) / slots) * m;
    if (best_cost < 0 || cost <= best_cost) { best_cost = cost; best = m; }
  }
  return best;
}

// Segments per sequence when every block fits in one wave of `per_sm` blocks
// per SM.  Block L = bh * nseg + seg is taken to share an SM with blocks
// L +- sms (the order in which a single wave fills the SMs); a block alone on
// its SM walks a chunk in time 1 and two co-resident blocks each take
// kPairCost (measured for the tensor-core output kernel: about 6.9 us against
// 4.0 us per chunk), so an SM holding blocks of a <= b chunks finishes at
// kPairCost a + (b - a).  Minimise the slowest SM; ties to fewer segments.
// Returns 0 when no split fits one wave.
int plan_nseg_one_wave(long long bh, int nc, int sms, int per_sm) {
  constexpr double kPairCost = 1.725;
  if (per_sm != 2 || bh <= 0 || sms <= 0) return 0;
  const long long slots = (long long)sms * per_sm;
  int best = 0;
  double best_cost = 0.0;
  for (int nseg = 1; nseg <= nc && bh * nseg <= slots; ++nseg) {
    const long long n = bh * nseg;
    double cost = 0.0;
    for (long long sm = 0; sm < sms && sm < n; ++sm) {
      const int s1 = (int)(sm % nseg);
      const int a = seg_first_chunk(s1 + 1, nc, nseg) - seg_first_chunk(s1, nc, nseg);
      double t = a;
      if (sm + sms < n) {
        const int s2 = (int)((sm + sms) % nseg);
        const int b = seg_first_chunk(s2 + 1, nc, nseg) - seg_first_chunk(s2, nc, nseg);
        const int lo = a < b ? a : b, hi = a < b ? b : a;
        t = kPairCost * lo + (hi - lo);
      }
      if (t > cost) cost = t;
    }
    if (best == 0 || cost < best_cost - 1e-9) { best = nseg; best_cost = cost; }
  }
  return best;
}

int check_gla_args(int B, int H, int gh, int gw, int dk, int dv, int dir, int chunk, int dtype) {
  if (B < 0 || H < 0 || gh < 0 || gw < 0) return GTR_ERR_INVALID_ARG;
  if (dir < 0 || dir > 4) return GTR_ERR_INVALID_ARG;
  if (dtype < 0 || dtype > 2) return GTR_ERR_INVALID_ARG;
  if (!valid_head_dim(dk) || !valid_head_dim(dv) || !valid_chunk(chunk)) return GTR_ERR_UNSUPPORTED;
  const long long T = (long long)gh * gw;
  if (T > 0x7fffffffLL) return GTR_ERR_INVALID_ARG;
  // every element offset must fit in 63 bits with room to spare
  const long long rows = (long long)B * T * H;
  if (B > 0 && H > 0 && T > 0 && rows / ((long long)B * H) != T) return GTR_ERR_INVALID_ARG;
  if (rows > (1LL << 46)) return GTR_ERR_INVALID_ARG;
  return GTR_OK;
}

bool tc_supported(int dk, int dv, int chunk, int dtype) {
  return tc_shape_supported(dk, dv, chunk, dtype) || tc128_shape_supported(dk, dv, chunk, dtype);
}

int choose_path(int dk, int dv, int chunk, int dtype) {
  const int setting = g_path_setting.load();
  if (setting == GTR_PATH_SIMT) return GTR_PATH_SIMT;
  if (setting == GTR_PATH_TC) return tc_supported(dk, dv, chunk, dtype) ? (int)GTR_PATH_TC : (int)GTR_ERR_UNSUPPORTED;
  return tc_supported(dk, dv, chunk, dtype) ? (int)GTR_PATH_TC : (int)GTR_PATH_SIMT;
}

int make_plan(Plan* p, int dev, int B, int H, int gh, int gw, int dk, int dv, int dir, int chunk,
              int dtype, int force_nseg) {
  p->B = B; p->H = H; p->gh = gh; p->gw = gw; p->T = gh * gw; p->dev = dev;
  p->dk = dk; p->dv = dv; p->dir = dir; p->chunk = chunk; p->dtype = dtype;
  const int path = choose_path(dk, dv, chunk, dtype);
  if (path < 0) return path;
  p->path = path;
  p->nc = (p->T + chunk - 1) / chunk;
  const long long bh = (long long)B * H;
  const int per_sm = path != GTR_PATH_TC ? 4
                     : dk == tc128::kD ? tc128_blocks_per_sm(dtype)
                                       : tc_blocks_per_sm(dk, dv);
  const long long slots = (long long)sm_count(dev) * per_sm;
  if (force_nseg > 0) {
    p->nseg = force_nseg < p->nc ? force_nseg : p->nc;
  } else {
    p->nseg = plan_nseg_one_wave(bh, p->nc, sm_count(dev), per_sm);
    if (p->nseg == 0) {
      const int m = plan_segments(bh, p->nc, slots);
      p->nseg = (p->nc + m - 1) / m;
    }
  }
  p->seg_chunks = (p->nc + p->nseg - 1) / p->nseg;
  const size_t nS = (size_t)bh * p->nseg * dk * dv * sizeof(float);
  p->offA = (nS + 255) & ~(size_t)255;
  p->ws_bytes = p->offA + (size_t)bh * p->nseg * dk * sizeof(float);
  return GTR_OK;
}

// Workspace of `bytes` for (device, stream): the registered caller buffer, or
// a cached library buffer grown with cudaMalloc outside stream capture.
int get_workspace(int dev, void* stream, size_t bytes, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_user_ws[dev]) {
    if (bytes > g_user_ws_bytes[dev]) return GTR_ERR_NO_MEMORY;
    *out = g_user_ws[dev];
    return GTR_OK;
  }
  auto key = std::make_pair(dev, stream);
  auto it = g_ws.find(key);
  if (it != g_ws.end() && it->second.second >= bytes) { *out = it->second.first; return GTR_OK; }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing((cudaStream_t)stream, &cs) != cudaSuccess) return GTR_ERR_CUDA;
  if (cs != cudaStreamCaptureStatusNone) return GTR_ERR_NO_MEMORY;
  if (it != g_ws.end()) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GTR_ERR_CUDA;
    cudaFree(it->second.first);
    g_ws.erase(it);
  }
  size_t want = bytes < ((size_t)1 << 20) ? ((size_t)1 << 20) : bytes + bytes / 4;
  void* p = nullptr;
  if (cudaMalloc(&p, want) != cudaSuccess) { (void)cudaGetLastError(); return GTR_ERR_NO_MEMORY; }
  g_ws[key] = std::make_pair(p, want);
  *out = p;
  return GTR_OK;
}

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
}



// cudaFuncSetAttribute once per kernel instance and device.
template <typename K>
int ensure_smem(K kern, size_t smem, bool* done, int dev) {
  if (done[dev]) return GTR_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return GTR_ERR_CUDA;
  done[dev] = true;
  return GTR_OK;
}

// ---- TMA tensor maps (encoded on the host through the driver entry point)
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load();
  if (!f) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && p) {
      f = (EncodeTiledFn)p;
      fn.store(f);
    } else {
      (void)cudaGetLastError();
    }
  }
  return f;
}
// 2-D row-major tensor [rows][cols] with the given row pitch, box box_cols x
// box_rows, 128-byte swizzle, out-of-range elements read as zero.
int tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, unsigned long long rows,
            unsigned long long cols, unsigned long long pitch_bytes, unsigned box_cols, unsigned box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return GTR_ERR_CUDA;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GTR_OK : GTR_ERR_CUDA;
}

// Tensor map of a [B, T, H, D] row-major tensor (element size es bytes,
// D = 64, or D = 16 with H = 1 for the rank-16 gate rows) for box loads of one
// chunk of one head: orientation 0 views it as (D, H, T, B), box (D, 1, 64,
// 1); orientation 1 as (D, H, gw, gh, B), box (D, 1, 1, 64, 1), a run of 64
// grid rows in one column.
int tmap_chunk(CUtensorMap* map, CUtensorMapDataType dt, int es, const void* base, const Plan& p, int orient,
               bool swizzle, int D_ = 64, int H_ = -1, int box_inner = 0) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return GTR_ERR_CUDA;
  const cuuint64_t D = (cuuint64_t)D_, es_ = (cuuint64_t)es;
  const cuuint64_t H = (cuuint64_t)(H_ < 0 ? p.H : H_);
  const cuuint64_t tok = H * D * es_;   // bytes per token
  CUresult r;
  if (orient == 0) {
    const cuuint64_t dims[4] = {D, H, (cuuint64_t)p.T, (cuuint64_t)p.B};
    const cuuint64_t strides[3] = {D * es_, tok, tok * (cuuint64_t)p.T};
    const cuuint32_t box[4] = {(cuuint32_t)(box_inner ? box_inner : D_), 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    r = enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[5] = {D, H, (cuuint64_t)p.gw, (cuuint64_t)p.gh, (cuuint64_t)p.B};
    const cuuint64_t strides[4] = {D * es_, tok, tok * (cuuint64_t)p.gw, tok * (cuuint64_t)p.T};
    const cuuint32_t box[5] = {(cuuint32_t)(box_inner ? box_inner : D_), 1, 1, 64, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    r = enc(map, dt, 5, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS ? GTR_OK : GTR_ERR_CUDA;
}
// Tensor maps of q (when given; the summary stage reads none), k, v, g, when
// every chunk of one head is one box: 16-byte aligned bases, and for the
// column orders (TB, BT) 64 | gh so that no chunk crosses a grid column.
// Returns false to gather with cp.async.
// With `low` (the gate's rank-16 rows) the g map is replaced by low's map and
// g may be null; `g_store` adds the store map of the g the summary kernel
// writes (32-column boxes, SWIZZLE_128B).
bool chunk_maps(const Plan& p, const void* q, const void* k, const void* v, const float* g, tc::Maps* maps,
                const float* low = nullptr, const float* g_store = nullptr) {
  for (const void* a : {q, k, v, (const void*)g, (const void*)low, (const void*)g_store})
    if (((uintptr_t)a & 15) != 0) return false;
  bool orient[2] = {false, false};
  for (int b = 0; b < (p.dir == kRotate ? (p.B < 4 ? p.B : 4) : 1); ++b) {
    const int d = p.dir == kRotate ? b : p.dir;
    orient[d == kTB || d == kBT] = true;
  }
  if (orient[1] && p.gh % 64 != 0) return false;
  if (p.T >= (1 << 30) || p.B >= (1 << 30)) return false;
  const CUtensorMapDataType dt = p.dtype == GTR_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  *maps = tc::Maps{};
  for (int o = 0; o < 2; ++o) {
    if (!orient[o]) continue;
    if ((q && tmap_chunk(&maps->t[o][tc::kMapQ], dt, 2, q, p, o, false)) ||
        tmap_chunk(&maps->t[o][tc::kMapK], dt, 2, k, p, o, false) ||
        tmap_chunk(&maps->t[o][tc::kMapV], dt, 2, v, p, o, true) ||
        (g && tmap_chunk(&maps->t[o][tc::kMapG], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, g, p, o, false)) ||
        (low && tmap_chunk(&maps->t[o][tc::kMapL], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, low, p, o, false,
                           tc::kLowRank, 1)) ||
        (g_store && tmap_chunk(&maps->t[o][tc::kMapGS], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, g_store, p, o, true,
                               64, -1, 32)))
      return false;
  }
  return true;
}

// ---- tensor-core gate: weight packing and the forward pass
int gate_pack_launch(int x_dtype, const float* w_down, const float* w_up, int dm, int HD, void* pack,
                     cudaStream_t st, int dev) {
  static bool done_h[kMaxDevices], done_b[kMaxDevices];
  if (x_dtype == GTR_F16) {
    if (int rc = ensure_smem(gate_tc::gate_pack_tc<__half>, gate_tc::Pack::kSmem, done_h, dev)) return rc;
    return launch_pdl(gate_tc::gate_pack_tc<__half>, dim3(1), dim3(gate_tc::kPackThreads),
                      gate_tc::Pack::kSmem, st, w_down, w_up, dm, HD, (uint8_t*)pack)
               ? GTR_ERR_CUDA
               : GTR_OK;
  }
  if (int rc = ensure_smem(gate_tc::gate_pack_tc<__nv_bfloat16>, gate_tc::Pack::kSmem, done_b, dev)) return rc;
  return launch_pdl(gate_tc::gate_pack_tc<__nv_bfloat16>, dim3(1), dim3(gate_tc::kPackThreads),
                    gate_tc::Pack::kSmem, st, w_down, w_up, dm, HD, (uint8_t*)pack)
             ? GTR_ERR_CUDA
             : GTR_OK;
}
int gate_fwd_packed_launch(int x_dtype, const void* x, const void* pack, const float* bias, float* g,
                           long long N, int dm, int HD, float tau, cudaStream_t st, int dev) {
  int tpc, spb, cols;
  long long blocks;
  gate_tc_grid(N, HD, sm_count(dev), &tpc, &spb, &blocks, &cols);
  CUtensorMap tmx, tmg;
  const CUtensorMapDataType xdt =
      x_dtype == GTR_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (int rc = tmap_2d(&tmx, xdt, x, (unsigned long long)N, (unsigned long long)dm,
                       (unsigned long long)dm * 2, 64, gate_tc::kM))
    return rc;
  if (int rc = tmap_2d(&tmg, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g, (unsigned long long)N,
                       (unsigned long long)HD, (unsigned long long)HD * 4, 32, (unsigned)tpc))
    return rc;
  const float inv_tau = 1.0f / tau;
  static bool done_h[kMaxDevices], done_b[kMaxDevices];
  if (x_dtype == GTR_F16) {
    if (int rc = ensure_smem(gate_tc::gate_fwd_tc<__half>, gate_tc::Layout::kSmem, done_h, dev)) return rc;
    return launch_pdl(gate_tc::gate_fwd_tc<__half>, dim3((unsigned)blocks, (unsigned)cols), dim3(gate_tc::kThreadsAll),
                      gate_tc::Layout::kSmem, st, tmx, tmg, (const uint8_t*)pack, bias, dm, HD, inv_tau, tpc, spb)
               ? GTR_ERR_CUDA
               : GTR_OK;
  }
  if (int rc = ensure_smem(gate_tc::gate_fwd_tc<__nv_bfloat16>, gate_tc::Layout::kSmem, done_b, dev)) return rc;
  return launch_pdl(gate_tc::gate_fwd_tc<__nv_bfloat16>, dim3((unsigned)blocks, (unsigned)cols), dim3(gate_tc::kThreadsAll),
                    gate_tc::Layout::kSmem, st, tmx, tmg, (const uint8_t*)pack, bias, dm, HD, inv_tau, tpc, spb)
             ? GTR_ERR_CUDA
             : GTR_OK;
}
// The gate's rank-16 rows low = x W_down [N, 16] fp32 (packed weights).
int gate_low_launch(int x_dtype, const void* x, const void* pack, float* low, long long N, int dm,
                    cudaStream_t st, int dev) {
  const int tpc = gate_tc_tile(N, sm_count(dev));
  const long long blocks = (N + tpc - 1) / tpc;
  CUtensorMap tmx;
  const CUtensorMapDataType xdt =
      x_dtype == GTR_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (int rc = tmap_2d(&tmx, xdt, x, (unsigned long long)N, (unsigned long long)dm,
                       (unsigned long long)dm * 2, 64, gate_tc::kM))
    return rc;
  static bool done_h[kMaxDevices], done_b[kMaxDevices];
  if (x_dtype == GTR_F16) {
    if (int rc = ensure_smem(gate_tc::gate_low_tc<__half>, gate_tc::LowLayout::kSmem, done_h, dev)) return rc;
    return launch_pdl(gate_tc::gate_low_tc<__half>, dim3((unsigned)blocks), dim3(gate_tc::kLowThreads),
                      gate_tc::LowLayout::kSmem, st, tmx, (const uint8_t*)pack, dm, low, N, tpc)
               ? GTR_ERR_CUDA
               : GTR_OK;
  }
  if (int rc = ensure_smem(gate_tc::gate_low_tc<__nv_bfloat16>, gate_tc::LowLayout::kSmem, done_b, dev)) return rc;
  return launch_pdl(gate_tc::gate_low_tc<__nv_bfloat16>, dim3((unsigned)blocks), dim3(gate_tc::kLowThreads),
                    gate_tc::LowLayout::kSmem, st, tmx, (const uint8_t*)pack, dm, low, N, tpc)
             ? GTR_ERR_CUDA
             : GTR_OK;
}
// Per-(device, stream) buffer for the packed weights gtr_gate_fwd makes each call.
std::map<std::pair<int, void*>, void*> g_pack_ws;
int pack_workspace(int dev, void* stream, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  auto key = std::make_pair(dev, stream);
  auto it = g_pack_ws.find(key);
  if (it != g_pack_ws.end()) { *out = it->second; return GTR_OK; }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing((cudaStream_t)stream, &cs) != cudaSuccess) return GTR_ERR_CUDA;
  if (cs != cudaStreamCaptureStatusNone) return GTR_ERR_NO_MEMORY;
  void* p = nullptr;
  if (cudaMalloc(&p, gate_tc::Pack::kBytes) != cudaSuccess) { (void)cudaGetLastError(); return GTR_ERR_NO_MEMORY; }
  g_pack_ws[key] = p;
  *out = p;
  return GTR_OK;
}

template <typename T, int ROWS>
int launch_simt_rows(const Plan& p, const void* q, const void* k, const void* v, const float* g,
                     const void* z, const float* w, void* out, float* wsS, float* wsA,
                     cudaStream_t st, int stage) {
  const dim3 grid(p.nseg, p.B * p.H);
  if (stage == 0) {
    // at most kSimtBatch * 4 * 128 floats = 32 KB: no opt-in needed
    const size_t smem = (size_t)simt_summary_smem_floats(p.dk, p.dv) * sizeof(float);
    auto kern = gla_summary_simt<T, ROWS>;
    kern<<<grid, kSimtThreads, smem, st>>>((const T*)k, (const T*)v, g, wsS, wsA, p.H, p.T, p.gh,
                                           p.gw, p.dk, p.dv, p.dir, p.chunk, p.nseg);
  } else {
    const size_t smem = (size_t)simt_output_smem_floats(p.dk, p.dv) * sizeof(float);
    auto kern = gla_output_simt<T, ROWS>;
    // opt in once to the largest footprint any (dk, dv) of this instance can need
    static bool done[kMaxDevices];
    if (int rc = ensure_smem(kern, simt_output_smem_floats(128, 128) * sizeof(float), done, p.dev))
      return rc;
    kern<<<grid, kSimtThreads, smem, st>>>((const T*)q, (const T*)k, (const T*)v, g, (const T*)z, w,
                                           wsS, (T*)out, p.H, p.T, p.gh, p.gw, p.dk, p.dv, p.dir,
                                           p.chunk, p.nseg);
  }
  return launch_status();
}

template <typename T>
int launch_simt(const Plan& p, const void* q, const void* k, const void* v, const float* g,
                const void* z, const float* w, void* out, float* wsS, float* wsA, cudaStream_t st,
                int stage) {
  switch ((p.dk * p.dv) / kSimtThreads) {
    case 1: return launch_simt_rows<T, 1>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    case 2: return launch_simt_rows<T, 2>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    case 4: return launch_simt_rows<T, 4>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    case 8: return launch_simt_rows<T, 8>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    case 16: return launch_simt_rows<T, 16>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    case 32: return launch_simt_rows<T, 32>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    case 64: return launch_simt_rows<T, 64>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    default: return GTR_ERR_UNSUPPORTED;
  }
}

// stage 0 = K2 summary, 1 = K4 output
int launch_stage(const Plan& p, const void* q, const void* k, const void* v, const float* g,
                 const void* z, const float* w, void* out, float* wsS, float* wsA, cudaStream_t st,
                 int stage) {
  if (p.path == GTR_PATH_TC && p.dk == tc128::kD) {
    const tc128::Params pp{q, k, v, g, z, w, wsS, wsA, out, p.H, p.T, p.gh, p.gw, p.dir, p.nc, p.nseg};
    return launch_tc128(p.dtype, stage, pp, p.B * p.H, st, p.dev) ? GTR_ERR_CUDA : GTR_OK;
  }
  if (p.path == GTR_PATH_TC) {
    tc::Maps maps;
    const bool boxes = chunk_maps(p, stage == 1 ? q : nullptr, k, v, g, &maps);
    return launch_tc(p.dtype, stage, q, k, v, g, z, w, out, wsS, wsA, p.B, p.H, p.T, p.gh, p.gw,
                     p.dk, p.dv, p.dir, p.chunk, p.nseg, boxes ? &maps : nullptr, st);
  }
  switch (p.dtype) {
    case GTR_F32: return launch_simt<float>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    case GTR_F16: return launch_simt<__half>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
    case GTR_BF16: return launch_simt<__nv_bfloat16>(p, q, k, v, g, z, w, out, wsS, wsA, st, stage);
  }
  return GTR_ERR_INVALID_ARG;
}

int launch_scan(const Plan& p, float* wsS, const float* wsA, int inclusive, cudaStream_t st) {
  const long long total = (long long)p.B * p.H * p.dk * p.dv;
  const long long groups = (total + 31) / 32;   // 32 elements per group
  auto go = [&](auto kern, int parts, int gpb) {
    const long long blocks = (groups + gpb - 1) / gpb;
    return launch_pdl(kern, dim3((unsigned)blocks), dim3(32 * parts * gpb), 0, st, wsS, wsA, total, p.nseg,
                      p.dk, p.dv, inclusive) == 0
               ? GTR_OK
               : GTR_ERR_CUDA;
  };
  // segments that fit one register window: one warp per group, four groups
  // per block; sixteen ranges per group only for very long scans (the wider
  // blocks keep fewer elements in flight: measured slower at 64 and 256
  // segments, faster at 1024)
  if (p.nseg <= kScanReg) return go(gla_state_scan<1, 4>, 1, 4);
  if (p.nseg >= 512) return go(gla_state_scan<kScanPartsWide, 1>, kScanPartsWide, 1);
  // ranges of up to 24 segments in one window (one load latency instead of four)
  if (p.nseg > kScanParts * kScanReg && p.nseg <= kScanParts * kScanRegLong)
    return go(gla_state_scan<kScanParts, 1, kScanRegLong>, kScanParts, 1);
  return go(gla_state_scan<kScanParts, 1>, kScanParts, 1);
}

// Record a caller event; inside stream capture it becomes an external event
// node, so a replayed graph records real timestamps.
int record(void* const* ev, int i, cudaStream_t st) {
  if (!ev || !ev[i]) return GTR_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return GTR_ERR_CUDA;
  const cudaError_t e = cs == cudaStreamCaptureStatusActive
                            ? cudaEventRecordWithFlags((cudaEvent_t)ev[i], st, cudaEventRecordExternal)
                            : cudaEventRecord((cudaEvent_t)ev[i], st);
  return e == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
}

int gla_fwd_impl(const void* q, const void* k, const void* v, const float* g, const void* z,
                 const float* w, void* out, int B, int H, int gh, int gw, int dk, int dv, int dir,
                 int chunk, int dtype, void* stream, void* const* ev) {
  int rc = check_gla_args(B, H, gh, gw, dk, dv, dir, chunk, dtype);
  if (rc) return rc;
  if (B == 0 || H == 0 || gh == 0 || gw == 0) return GTR_OK;
  if (!q || !k || !v || !g || !z || !out) return GTR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(z) ||
      !aligned16(out) || (w && !aligned16(w)))
    return GTR_ERR_ALIGNMENT;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  Plan p;
  if ((rc = make_plan(&p, dev, B, H, gh, gw, dk, dv, dir, chunk, dtype, 0))) return rc;
  void* ws = nullptr;
  if ((rc = get_workspace(dev, stream, p.ws_bytes, &ws))) return rc;
  float* wsS = (float*)ws;
  float* wsA = (float*)((char*)ws + p.offA);
  cudaStream_t st = (cudaStream_t)stream;
  if ((rc = record(ev, 0, st))) return rc;
  if ((rc = launch_stage(p, q, k, v, g, z, w, out, wsS, wsA, st, 0))) return rc;
  if ((rc = record(ev, 1, st))) return rc;
  if ((rc = launch_scan(p, wsS, wsA, 0, st))) return rc;
  if ((rc = record(ev, 2, st))) return rc;
  if ((rc = launch_stage(p, q, k, v, g, z, w, out, wsS, wsA, st, 1))) return rc;
  return record(ev, 3, st);
}

// Gate projection + GLA forward (gtr_gla_fwd_gated).  On the tensor-core path
// the gate is split at its rank-16 bottleneck: a short kernel writes low = x
// W_down ([N, 16] fp32, in the workspace), and the summary kernel forms g =
// logsigmoid(low W_up + b)/tau per chunk as it needs it, writing g_out for the
// output kernel; no separate pass over g runs.  Otherwise the gate kernel and
// gtr_gla_fwd run one after the other.  Events (profiling): ev[0] before the
// gate, ev[1] after it, ev[2] after the summary, ev[3] after the scan, ev[4]
// after the output kernel.
int gla_fwd_gated_impl(const void* x, int x_dtype, const void* packed, const float* bias, int d_model,
                       int rank, float tau, const void* q, const void* k, const void* v, const void* z,
                       const float* w, float* g_out, void* out, int B, int H, int gh, int gw, int dk, int dv,
                       int dir, int chunk, int dtype, void* stream, void* const* ev) {
  int rc = check_gla_args(B, H, gh, gw, dk, dv, dir, chunk, dtype);
  if (rc) return rc;
  if (x_dtype < 0 || x_dtype > 2 || d_model <= 0 || rank <= 0) return GTR_ERR_INVALID_ARG;
  if (!(tau > 0.0f) || !(tau < 3.0e38f)) return GTR_ERR_INVALID_ARG;
  const long long HD = (long long)H * dk;
  if (HD > 4096 || !gate_tc_supported(x_dtype, d_model, rank, (int)HD)) return GTR_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || gh == 0 || gw == 0) return GTR_OK;
  const long long N = (long long)B * gh * gw;
  if (N >= (1LL << 31)) return GTR_ERR_UNSUPPORTED;
  if (!x || !packed || !q || !k || !v || !z || !g_out || !out) return GTR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || (bias && !aligned16(bias)) || !aligned16(q) || !aligned16(k) ||
      !aligned16(v) || !aligned16(z) || !aligned16(g_out) || !aligned16(out) || (w && !aligned16(w)))
    return GTR_ERR_ALIGNMENT;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  Plan p;
  if ((rc = make_plan(&p, dev, B, H, gh, gw, dk, dv, dir, chunk, dtype, 0))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if ((rc = record(ev, 0, st))) return rc;
  if (p.path != GTR_PATH_TC || dk != tc::kD) {
    if ((rc = gate_fwd_packed_launch(x_dtype, x, packed, bias, g_out, N, d_model, (int)HD, tau, st, dev)))
      return rc;
    if ((rc = record(ev, 1, st))) return rc;
    void* ev4[4] = {nullptr, ev ? ev[2] : nullptr, ev ? ev[3] : nullptr, ev ? ev[4] : nullptr};
    return gla_fwd_impl(q, k, v, g_out, z, w, out, B, H, gh, gw, dk, dv, dir, chunk, dtype, stream, ev4);
  }
  const size_t offL = (p.ws_bytes + 255) & ~(size_t)255;
  void* ws = nullptr;
  if ((rc = get_workspace(dev, stream, offL + (size_t)N * tc::kLowRank * sizeof(float), &ws))) return rc;
  float* wsS = (float*)ws;
  float* wsA = (float*)((char*)ws + p.offA);
  float* low = (float*)((char*)ws + offL);
  if ((rc = gate_low_launch(x_dtype, x, packed, low, N, d_model, st, dev))) return rc;
  if ((rc = record(ev, 1, st))) return rc;
  tc::Maps maps;
  const bool boxes = chunk_maps(p, nullptr, k, v, nullptr, &maps, low, g_out);
  const uint8_t* pk = (const uint8_t*)packed;
  if (launch_tc_gated_sum(p.dtype, k, v, low, pk + gate_tc::Pack::kOffWu, gate_tc::Layout::kWu,
                          (const float*)(pk + gate_tc::Pack::kOffScale) + gate_tc::kRank, bias, 1.0f / tau,
                          g_out, wsS, wsA, B, H, p.T, gh, gw, dir, p.nseg, boxes ? &maps : nullptr, st))
    return GTR_ERR_CUDA;
  if ((rc = record(ev, 2, st))) return rc;
  if ((rc = launch_scan(p, wsS, wsA, 0, st))) return rc;
  if ((rc = record(ev, 3, st))) return rc;
  if ((rc = launch_stage(p, q, k, v, g_out, z, w, out, wsS, wsA, st, 1))) return rc;
  return record(ev, 4, st);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of gtr_gla_fwd.  Its scratch (the segment states of
// the summary and scan stages) is this file-scope device array instead of a
// cudaMalloc'ed workspace.  Every GPU that loads the library reserves it until
// the process exits.  Host code may not use the array's name as a device
// pointer (on the host it names a stand-in object), so its device address is
// looked up once per device with cudaGetSymbolAddress, with that device
// current, and passed to the kernels.
constexpr size_t kStaticScratchBytes = (size_t)8 << 20;   // 8 MiB per device
static __device__ __align__(256) unsigned char g_gtr_static_scratch[kStaticScratchBytes];
void* g_static_scratch_ptr[kMaxDevices];

int static_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_scratch_ptr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_gtr_static_scratch);
    if (e != cudaSuccess || !ptr) {
      (void)cudaGetLastError();
      // the array is placed on the device when the library's module first
      // loads there; on a full device that placement is what fails
      return e == cudaErrorMemoryAllocation ? GTR_ERR_NO_MEMORY : GTR_ERR_CUDA;
    }
    g_static_scratch_ptr[dev] = ptr;
  }
  *out = g_static_scratch_ptr[dev];
  return GTR_OK;
}

int gla_fwd_noalloc_impl(const void* q, const void* k, const void* v, const float* g, const void* z,
                         const float* w, void* out, int B, int H, int gh, int gw, int dk, int dv,
                         int dir, int chunk, int dtype, void* stream) {
  int rc = check_gla_args(B, H, gh, gw, dk, dv, dir, chunk, dtype);
  if (rc) return rc;
  if (B == 0 || H == 0 || gh == 0 || gw == 0) return GTR_OK;
  if (!q || !k || !v || !g || !z || !out) return GTR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(z) ||
      !aligned16(out) || (w && !aligned16(w)))
    return GTR_ERR_ALIGNMENT;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  Plan p;
  if ((rc = make_plan(&p, dev, B, H, gh, gw, dk, dv, dir, chunk, dtype, 0))) return rc;
  if (p.ws_bytes > kStaticScratchBytes) {
    // fewer, longer segments until the boundary states fit the static scratch
    const size_t per_seg = (size_t)B * H * ((size_t)dk * dv + dk) * sizeof(float);
    const size_t max_nseg = (kStaticScratchBytes - 256) / per_seg;
    if (max_nseg < 1) return GTR_ERR_NO_MEMORY;
    const int nseg = (int)(max_nseg < (size_t)p.nc ? max_nseg : (size_t)p.nc);
    if ((rc = make_plan(&p, dev, B, H, gh, gw, dk, dv, dir, chunk, dtype, nseg))) return rc;
    if (p.ws_bytes > kStaticScratchBytes) return GTR_ERR_NO_MEMORY;
  }
  void* ws = nullptr;
  if ((rc = static_scratch(dev, &ws))) return rc;
  float* wsS = (float*)ws;
  float* wsA = (float*)((char*)ws + p.offA);
  cudaStream_t st = (cudaStream_t)stream;
  if ((rc = launch_stage(p, q, k, v, g, z, w, out, wsS, wsA, st, 0))) return rc;
  if ((rc = launch_scan(p, wsS, wsA, 0, st))) return rc;
  return launch_stage(p, q, k, v, g, z, w, out, wsS, wsA, st, 1);
}

}  // namespace

// The projections' GEMM: its host side (tensor maps, tile width, launch),
// after the helpers above that it uses.
#include "gemm_host.cuh"

extern "C" {

int gtr_abi_version(void) { return GTR_ABI_VERSION; }

const char* gtr_status_string(int status) {
  switch (status) {
    case GTR_OK: return "ok";
    case GTR_ERR_INVALID_ARG: return "invalid argument";
    case GTR_ERR_UNSUPPORTED: return "unsupported shape or option";
    case GTR_ERR_ALIGNMENT: return "tensor pointer not 16-byte aligned";
    case GTR_ERR_NO_MEMORY: return "workspace unavailable";
    case GTR_ERR_CUDA: return "CUDA runtime or launch error";
    case GTR_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

gtr_status_t gtr_gate_fwd(const void* x, int x_dtype, const float* w_down, const float* w_up,
                          const float* bias, float* g_out, int B, int T, int d_model, int rank,
                          int H, int dk, float tau, void* stream) {
  if (B < 0 || T < 0 || H < 0 || dk < 0 || d_model <= 0 || rank <= 0) return GTR_ERR_INVALID_ARG;
  if (x_dtype < 0 || x_dtype > 2) return GTR_ERR_INVALID_ARG;
  if (!(tau > 0.0f) || !(tau < 3.0e38f)) return GTR_ERR_INVALID_ARG;
  if (rank > kGateMaxRank || d_model > 4096 || (long long)H * dk > 4096) return GTR_ERR_UNSUPPORTED;
  const long long N = (long long)B * T;
  if (N == 0 || H == 0 || dk == 0) return GTR_OK;
  if (N > (1LL << 40)) return GTR_ERR_INVALID_ARG;
  if (!x || !w_down || !w_up || !g_out) return GTR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(g_out) || !aligned16(w_down) || !aligned16(w_up) ||
      (bias && !aligned16(bias)))
    return GTR_ERR_ALIGNMENT;
  const int HD = H * dk;
  cudaStream_t st = (cudaStream_t)stream;
  if (gate_tc_supported(x_dtype, d_model, rank, HD) && N < (1LL << 31)) {
    // tensor-core kernels: pack the weights into this stream's buffer, then
    // the forward pass (about one tile of tokens per SM)
    int dev;
    if (int rc = current_device(&dev)) return (gtr_status_t)rc;
    void* pack = nullptr;
    if (int rc = pack_workspace(dev, stream, &pack)) return (gtr_status_t)rc;
    if (int rc = gate_pack_launch(x_dtype, w_down, w_up, d_model, HD, pack, st, dev)) return (gtr_status_t)rc;
    return (gtr_status_t)gate_fwd_packed_launch(x_dtype, x, pack, bias, g_out, N, d_model, HD, tau, st, dev);
  }
  if (rank <= 16 && HD % 4 == 0 && HD <= kGate2MaxHD && (!bias || aligned16(bias))) {
    // register-tiled kernel: one block per 64 tokens
    const long long blocks = (N + kGate2Tok - 1) / kGate2Tok;
    if (blocks > 0x7fffffffLL) return GTR_ERR_INVALID_ARG;
    const size_t smem = gate_tiled_smem(HD);
    int dev;
    if (int rc = current_device(&dev)) return (gtr_status_t)rc;
    const float inv_tau = 1.0f / tau;
    switch (x_dtype) {
      case GTR_F32: {
        static bool done[kMaxDevices];
        if (int rc = ensure_smem(gate_proj_tiled<float>, gate_tiled_smem(kGate2MaxHD), done, dev))
          return (gtr_status_t)rc;
        gate_proj_tiled<float><<<(unsigned)blocks, kGate2Threads, smem, st>>>(
            (const float*)x, w_down, w_up, bias, g_out, N, d_model, rank, HD, inv_tau);
        break;
      }
      case GTR_F16: {
        static bool done[kMaxDevices];
        if (int rc = ensure_smem(gate_proj_tiled<__half>, gate_tiled_smem(kGate2MaxHD), done, dev))
          return (gtr_status_t)rc;
        gate_proj_tiled<__half><<<(unsigned)blocks, kGate2Threads, smem, st>>>(
            (const __half*)x, w_down, w_up, bias, g_out, N, d_model, rank, HD, inv_tau);
        break;
      }
      default: {
        static bool done[kMaxDevices];
        if (int rc = ensure_smem(gate_proj_tiled<__nv_bfloat16>, gate_tiled_smem(kGate2MaxHD), done, dev))
          return (gtr_status_t)rc;
        gate_proj_tiled<__nv_bfloat16><<<(unsigned)blocks, kGate2Threads, smem, st>>>(
            (const __nv_bfloat16*)x, w_down, w_up, bias, g_out, N, d_model, rank, HD, inv_tau);
        break;
      }
    }
    return (gtr_status_t)launch_status();
  }
  const long long blocks = (N + kGateTok - 1) / kGateTok;
  if (blocks > 0x7fffffffLL) return GTR_ERR_INVALID_ARG;
  switch (x_dtype) {
    case GTR_F32:
      gate_proj_kernel<float><<<(unsigned)blocks, kGateThreads, 0, st>>>(
          (const float*)x, w_down, w_up, bias, g_out, N, d_model, rank, HD, tau);
      break;
    case GTR_F16:
      gate_proj_kernel<__half><<<(unsigned)blocks, kGateThreads, 0, st>>>(
          (const __half*)x, w_down, w_up, bias, g_out, N, d_model, rank, HD, tau);
      break;
    default:
      gate_proj_kernel<__nv_bfloat16><<<(unsigned)blocks, kGateThreads, 0, st>>>(
          (const __nv_bfloat16*)x, w_down, w_up, bias, g_out, N, d_model, rank, HD, tau);
      break;
  }
  return (gtr_status_t)launch_status();
}

size_t gtr_gate_packed_bytes(void) { return (size_t)gate_tc::Pack::kBytes; }

gtr_status_t gtr_gate_pack(const float* w_down, const float* w_up, int x_dtype, int d_model, int rank,
                           int H, int dk, void* packed, size_t packed_bytes, void* stream) {
  if (H <= 0 || dk <= 0 || d_model <= 0 || rank <= 0) return GTR_ERR_INVALID_ARG;
  if (x_dtype < 0 || x_dtype > 2) return GTR_ERR_INVALID_ARG;
  const long long HD = (long long)H * dk;
  if (HD > 4096 || !gate_tc_supported(x_dtype, d_model, rank, (int)HD)) return GTR_ERR_UNSUPPORTED;
  if (!w_down || !w_up || !packed) return GTR_ERR_INVALID_ARG;
  if (packed_bytes < (size_t)gate_tc::Pack::kBytes) return GTR_ERR_NO_MEMORY;
  if (!aligned16(w_down) || !aligned16(w_up) || !aligned16(packed)) return GTR_ERR_ALIGNMENT;
  int dev;
  if (int rc = current_device(&dev)) return (gtr_status_t)rc;
  return (gtr_status_t)gate_pack_launch(x_dtype, w_down, w_up, d_model, (int)HD, packed,
                                        (cudaStream_t)stream, dev);
}

gtr_status_t gtr_gate_fwd_packed(const void* x, int x_dtype, const void* packed, const float* bias,
                                 float* g_out, int B, int T, int d_model, int rank, int H, int dk,
                                 float tau, void* stream) {
  if (B < 0 || T < 0 || H <= 0 || dk <= 0 || d_model <= 0 || rank <= 0) return GTR_ERR_INVALID_ARG;
  if (x_dtype < 0 || x_dtype > 2) return GTR_ERR_INVALID_ARG;
  if (!(tau > 0.0f) || !(tau < 3.0e38f)) return GTR_ERR_INVALID_ARG;
  const long long HD = (long long)H * dk;
  if (HD > 4096 || !gate_tc_supported(x_dtype, d_model, rank, (int)HD)) return GTR_ERR_UNSUPPORTED;
  const long long N = (long long)B * T;
  if (N == 0) return GTR_OK;
  if (N >= (1LL << 31)) return GTR_ERR_UNSUPPORTED;
  if (!x || !packed || !g_out) return GTR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(g_out) || (bias && !aligned16(bias)))
    return GTR_ERR_ALIGNMENT;
  int dev;
  if (int rc = current_device(&dev)) return (gtr_status_t)rc;
  return (gtr_status_t)gate_fwd_packed_launch(x_dtype, x, packed, bias, g_out, N, d_model, (int)HD, tau,
                                              (cudaStream_t)stream, dev);
}

gtr_status_t gtr_gla_fwd(const void* q, const void* k, const void* v, const float* g,
                         const void* outgate, const float* rms_w, void* out, int B, int H,
                         int grid_h, int grid_w, int dk, int dv, int dir, int chunk, int dtype,
                         void* stream) {
  return (gtr_status_t)gla_fwd_impl(q, k, v, g, outgate, rms_w, out, B, H, grid_h, grid_w, dk, dv,
                                    dir, chunk, dtype, stream, nullptr);
}

gtr_status_t gtr_gla_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                 const void* outgate, const float* rms_w, void* out, int B, int H,
                                 int grid_h, int grid_w, int dk, int dv, int dir, int chunk,
                                 int dtype, void* stream) {
  return (gtr_status_t)gla_fwd_noalloc_impl(q, k, v, g, outgate, rms_w, out, B, H, grid_h, grid_w,
                                            dk, dv, dir, chunk, dtype, stream);
}

gtr_status_t gtr_gla_fwd_timed(const void* q, const void* k, const void* v, const float* g,
                               const void* outgate, const float* rms_w, void* out, int B, int H,
                               int grid_h, int grid_w, int dk, int dv, int dir, int chunk,
                               int dtype, void* stream, void* const* ev) {
  return (gtr_status_t)gla_fwd_impl(q, k, v, g, outgate, rms_w, out, B, H, grid_h, grid_w, dk, dv,
                                    dir, chunk, dtype, stream, ev);
}

gtr_status_t gtr_gla_fwd_gated(const void* x, int x_dtype, const void* packed, const float* bias,
                               int d_model, int rank, float tau, const void* q, const void* k,
                               const void* v, const void* outgate, const float* rms_w, float* g_out,
                               void* out, int B, int H, int grid_h, int grid_w, int dk, int dv, int dir,
                               int chunk, int dtype, void* stream) {
  return (gtr_status_t)gla_fwd_gated_impl(x, x_dtype, packed, bias, d_model, rank, tau, q, k, v, outgate,
                                          rms_w, g_out, out, B, H, grid_h, grid_w, dk, dv, dir, chunk,
                                          dtype, stream, nullptr);
}

gtr_status_t gtr_gla_fwd_gated_timed(const void* x, int x_dtype, const void* packed, const float* bias,
                                     int d_model, int rank, float tau, const void* q, const void* k,
                                     const void* v, const void* outgate, const float* rms_w, float* g_out,
                                     void* out, int B, int H, int grid_h, int grid_w, int dk, int dv,
                                     int dir, int chunk, int dtype, void* stream, void* const* ev) {
  return (gtr_status_t)gla_fwd_gated_impl(x, x_dtype, packed, bias, d_model, rank, tau, q, k, v, outgate,
                                          rms_w, g_out, out, B, H, grid_h, grid_w, dk, dv, dir, chunk,
                                          dtype, stream, ev);
}

gtr_status_t gtr_mixer_in_proj(const void* x, const void* w_in, void* q, void* k, void* v, void* z, int B, int T,
                               int d_model, int H, int dk, int dv, int dtype, void* stream) {
  if (B < 0 || T < 0 || H < 0 || dk < 0 || dv < 0 || d_model < 0) return GTR_ERR_INVALID_ARG;
  if (dtype < 0 || dtype > 2) return GTR_ERR_INVALID_ARG;
  const long long N = (long long)B * T, n_q = (long long)H * dk, n_v = (long long)H * dv;
  if (N == 0 || n_q + n_v == 0 || d_model == 0) return GTR_OK;
  if (dtype == GTR_F32) return GTR_ERR_UNSUPPORTED;
  if (N >= (1LL << 31) || 2 * (n_q + n_v) >= (1LL << 31)) return GTR_ERR_INVALID_ARG;
  if (!x || !w_in || !q || !k || !v || !z) return GTR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_in) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(z))
    return GTR_ERR_ALIGNMENT;
  int dev;
  if (int rc = current_device(&dev)) return (gtr_status_t)rc;
  const int ldw = (int)(2 * (n_q + n_v));
  const char* W = (const char*)w_in;
  cudaStream_t st = (cudaStream_t)stream;
  {
    // our tensor-core GEMM: the four column blocks as one launch with four
    // outputs when they are equally wide whole tiles, else one launch each
    void* outs4[4] = {q, k, v, z};
    int rc = gtr::gemm_tc(dtype, x, d_model, W, ldw, outs4, 4, (int)n_q, (int)n_q, (int)N, ldw, d_model, st);
    if (n_q != n_v || rc == GTR_ERR_UNSUPPORTED) {
      const long long off[4] = {0, n_q, 2 * n_q, 2 * n_q + n_v};
      const long long width[4] = {n_q, n_q, n_v, n_v};
      rc = GTR_OK;
      for (int i = 0; i < 4 && rc == GTR_OK; ++i) {
        if (width[i] == 0) continue;
        void* o1[1] = {outs4[i]};
        rc = gtr::gemm_tc(dtype, x, d_model, W + off[i] * 2, ldw, o1, 1, (int)width[i], (int)width[i], (int)N,
                          (int)width[i], d_model, st);
      }
    }
    if (rc != GTR_ERR_UNSUPPORTED) return (gtr_status_t)rc;
  }
  // shapes the tensor maps cannot address: cuBLAS
  const cudaDataType dt = dtype == GTR_F16 ? CUDA_R_16F : CUDA_R_16BF;
  // column blocks of W: q | k | v | z.  Four equal blocks whose outputs lie
  // equally spaced in memory go out as one strided-batched product.
  const long long gap = (const char*)k - (const char*)q;
  if (n_q == n_v && gap > 0 && gap % 2 == 0 && (const char*)v - (const char*)k == gap &&
      (const char*)z - (const char*)v == gap && gap >= N * n_q * 2)
    return (gtr_status_t)blas_gemm_rowmajor(dev, st, dt, x, d_model, W, ldw, q, (int)n_q, (int)N, d_model,
                                            (int)n_q, 4, n_q, gap / 2);
  const long long off[4] = {0, n_q, 2 * n_q, 2 * n_q + n_v};
  const long long width[4] = {n_q, n_q, n_v, n_v};
  void* outs[4] = {q, k, v, z};
  for (int i = 0; i < 4; ++i) {
    if (width[i] == 0) continue;
    if (int rc = blas_gemm_rowmajor(dev, st, dt, x, d_model, W + off[i] * 2, ldw, outs[i], (int)width[i], (int)N,
                                    d_model, (int)width[i]))
      return (gtr_status_t)rc;
  }
  return GTR_OK;
}

gtr_status_t gtr_mixer_out_proj(const void* y, const void* w_out, void* out, long long N, int d_in, int d_out,
                                int dtype, void* stream) {
  if (N < 0 || d_in < 0 || d_out < 0) return GTR_ERR_INVALID_ARG;
  if (dtype < 0 || dtype > 2) return GTR_ERR_INVALID_ARG;
  if (N == 0 || d_in == 0 || d_out == 0) return GTR_OK;
  if (dtype == GTR_F32) return GTR_ERR_UNSUPPORTED;
  if (N >= (1LL << 31)) return GTR_ERR_INVALID_ARG;
  if (!y || !w_out || !out) return GTR_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(w_out) || !aligned16(out)) return GTR_ERR_ALIGNMENT;
  int dev;
  if (int rc = current_device(&dev)) return (gtr_status_t)rc;
  void* o1[1] = {out};
  const int rc = gtr::gemm_tc(dtype, y, d_in, w_out, d_out, o1, 1, d_out, d_out, (int)N, d_out, d_in,
                              (cudaStream_t)stream);
  if (rc != GTR_ERR_UNSUPPORTED) return (gtr_status_t)rc;
  // shapes the tensor maps cannot address: cuBLAS
  const cudaDataType dt = dtype == GTR_F16 ? CUDA_R_16F : CUDA_R_16BF;
  return (gtr_status_t)blas_gemm_rowmajor(dev, (cudaStream_t)stream, dt, y, d_in, w_out, d_out, out, d_out, (int)N,
                                          d_in, d_out);
}

gtr_status_t gtr_gla_chunk_states(const void* k, const void* v, const float* g, float* states,
                                  int B, int H, int grid_h, int grid_w, int dk, int dv, int dir,
                                  int chunk, int dtype, void* stream) {
  int rc = check_gla_args(B, H, grid_h, grid_w, dk, dv, dir, chunk, dtype);
  if (rc) return (gtr_status_t)rc;
  if (B == 0 || H == 0 || grid_h == 0 || grid_w == 0) return GTR_OK;
  if (!k || !v || !g || !states) return GTR_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(states)) return GTR_ERR_ALIGNMENT;
  int dev;
  if ((rc = current_device(&dev))) return (gtr_status_t)rc;
  Plan p;
  // one chunk per segment: the scan then gives the state after every chunk
  if ((rc = make_plan(&p, dev, B, H, grid_h, grid_w, dk, dv, dir, chunk, dtype, 0x7fffffff)))
    return (gtr_status_t)rc;
  void* ws = nullptr;
  const size_t lbytes = (size_t)B * H * p.nseg * dk * sizeof(float);
  if ((rc = get_workspace(dev, stream, lbytes, &ws))) return (gtr_status_t)rc;
  cudaStream_t st = (cudaStream_t)stream;
  if ((rc = launch_stage(p, nullptr, k, v, g, nullptr, nullptr, nullptr, states, (float*)ws, st, 0)))
    return (gtr_status_t)rc;
  return (gtr_status_t)launch_scan(p, states, (const float*)ws, 1, st);
}

size_t gtr_gla_workspace_bytes(int B, int H, int grid_h, int grid_w, int dk, int dv, int chunk,
                               int dtype) {
  if (check_gla_args(B, H, grid_h, grid_w, dk, dv, 0, chunk, dtype)) return (size_t)-1;
  if (B == 0 || H == 0 || grid_h == 0 || grid_w == 0) return 0;
  int dev;
  if (current_device(&dev)) return (size_t)-1;
  Plan p;
  if (make_plan(&p, dev, B, H, grid_h, grid_w, dk, dv, 0, chunk, dtype, 0)) return (size_t)-1;
  return p.ws_bytes;
}

int gtr_gla_segment_chunks(int B, int H, int grid_h, int grid_w, int dk, int dv, int chunk,
                           int dtype) {
  int rc = check_gla_args(B, H, grid_h, grid_w, dk, dv, 0, chunk, dtype);
  if (rc) return rc;
  if (B == 0 || H == 0 || grid_h == 0 || grid_w == 0) return 0;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  Plan p;
  if ((rc = make_plan(&p, dev, B, H, grid_h, grid_w, dk, dv, 0, chunk, dtype, 0))) return rc;
  return p.seg_chunks;
}

int gtr_gla_segment_count(int B, int H, int grid_h, int grid_w, int dk, int dv, int chunk, int dtype) {
  int rc = check_gla_args(B, H, grid_h, grid_w, dk, dv, 0, chunk, dtype);
  if (rc) return rc;
  if (B == 0 || H == 0 || grid_h == 0 || grid_w == 0) return 0;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  Plan p;
  if ((rc = make_plan(&p, dev, B, H, grid_h, grid_w, dk, dv, 0, chunk, dtype, 0))) return rc;
  return p.nseg;
}

gtr_status_t gtr_gla_set_workspace(void* ptr, size_t bytes) {
  int dev;
  int rc = current_device(&dev);
  if (rc) return (gtr_status_t)rc;
  if (ptr && ((uintptr_t)ptr & 255u)) return GTR_ERR_ALIGNMENT;
  std::lock_guard<std::mutex> lk(g_mu);
  g_user_ws[dev] = ptr;
  g_user_ws_bytes[dev] = ptr ? bytes : 0;
  return GTR_OK;
}

gtr_status_t gtr_gla_set_path(int path) {
  if (path < GTR_PATH_AUTO || path > GTR_PATH_TC) return GTR_ERR_INVALID_ARG;
  g_path_setting.store(path);
  return GTR_OK;
}

int gtr_gla_path_for(int B, int H, int grid_h, int grid_w, int dk, int dv, int chunk, int dtype) {
  int rc = check_gla_args(B, H, grid_h, grid_w, dk, dv, 0, chunk, dtype);
  if (rc) return rc;
  return choose_path(dk, dv, chunk, dtype);
}

gtr_status_t gtr_last_device_status(void* stream, unsigned long long* counters) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GTR_ERR_CUDA;
  unsigned int st = 0;
  unsigned long long ex = 0;
  const unsigned int zero = 0;
  const unsigned long long zero64 = 0;
  if (cudaMemcpyFromSymbol(&st, g_gtr_status, sizeof(st)) != cudaSuccess) return GTR_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&ex, g_gtr_exact_chunks, sizeof(ex)) != cudaSuccess) return GTR_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_gtr_status, &zero, sizeof(zero)) != cudaSuccess) return GTR_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_gtr_exact_chunks, &zero64, sizeof(zero64)) != cudaSuccess) return GTR_ERR_CUDA;
  if (counters) { counters[0] = st; counters[1] = ex; }
  return st ? GTR_ERR_DEVICE_CHECK : GTR_OK;
}

}  // extern "C"

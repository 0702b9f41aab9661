// api.cu -- host side of the libssmscan C ABI: argument checks, work planning
// and kernel dispatch.  Every entry point is declared in include/ssmscan.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdio>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "../../include/ssmscan.h"
#include "scan_bwd.cuh"
#include "scan_fwd.cuh"
#include "scan_step.cuh"
#include "ssd_fwd.cuh"

namespace {

using namespace ssm;

constexpr int kMaxDevices = 64;

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int device_sm_count() {
  // per-device cache; concurrent first calls store the same value
  static std::atomic<int> counts[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = counts[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    counts[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per
// (kernel, device).  The cache is keyed by the kernel's address: every
// kernel template instance has the same function type.
cudaError_t set_smem(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) done.insert({kernel, dev});
  return e;
}

size_t elem_size(ssm_dtype_t t) { return t == SSM_BF16 ? 2 : 4; }

thread_local char g_last_error[256] = "";

// Maps a CUDA result to a status, remembering the message of a failure.
ssm_status_t cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return SSM_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorString(e),
           cudaGetErrorName(e));
  return SSM_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Mamba-1 selective scan
// ---------------------------------------------------------------------------
struct ScanPlan {
  ScanParams p;
  bool vec;
  size_t ws_bytes;
};

// check_ptrs = false skips the null-pointer checks (workspace-size queries
// look only at sizes, types and layout).
ssm_status_t plan_scan(const ssm_scan_args_t* a, ScanPlan* out, bool check_ptrs = true) {
  if (a == nullptr) return SSM_ERR_INVALID_ARG;
  if (a->batch < 0 || a->dim < 0 || a->seqlen < 0) return SSM_ERR_INVALID_ARG;
  if (a->dtype != SSM_F32 && a->dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
  if (a->dstate < 1 || a->dstate > fwd::kMaxN) return SSM_ERR_UNSUPPORTED;
  if (a->batch > 65535) return SSM_ERR_UNSUPPORTED;
  const int64_t L = a->seqlen;
  const size_t es = elem_size(a->dtype);
  const bool any_work = a->batch > 0 && a->dim > 0;
  if (any_work && check_ptrs) {
    if (a->A == nullptr) return SSM_ERR_INVALID_ARG;
    if (L > 0 && (a->u == nullptr || a->delta == nullptr || a->B == nullptr ||
                  a->C == nullptr || a->y == nullptr))
      return SSM_ERR_INVALID_ARG;
  }
  const void* tensors[] = {a->u, a->delta, a->B, a->C, a->z, a->y};
  for (const void* t : tensors)
    if (t != nullptr && !aligned(t, es)) return SSM_ERR_ALIGNMENT;
  const void* f32s[] = {a->A, a->D, a->delta_bias, a->h0, a->h_last};
  for (const void* t : f32s)
    if (t != nullptr && !aligned(t, 4)) return SSM_ERR_ALIGNMENT;

  ScanParams& p = out->p;
  p.batch = a->batch;
  p.dim = a->dim;
  p.dstate = a->dstate;
  p.seqlen = L;
  p.u = a->u;
  p.delta = a->delta;
  p.z = a->z;
  p.y = a->y;
  p.B = a->B;
  p.C = a->C;
  auto pick = [](int64_t s, int64_t def) { return s == 0 ? def : s; };
  if (a->ngroups < 0) return SSM_ERR_INVALID_ARG;
  const int64_t G = a->ngroups > 1 ? a->ngroups : 1;
  if (G > 1 && (a->dim % G != 0 || (a->dim / G) % fwd::kCH != 0)) return SSM_ERR_UNSUPPORTED;
  p.group_ch = G > 1 ? a->dim / G : (a->dim > 0 ? a->dim : 1);
  const int64_t xb = a->dim * L, xd = L, bcb = G * a->dstate * L, bcn = L;
  p.B_sg = G > 1 ? pick(a->B_group_stride, a->dstate * L) : 0;
  p.C_sg = G > 1 ? pick(a->C_group_stride, a->dstate * L) : 0;
  p.u_sb = pick(a->u_stride[0], xb);
  p.u_sd = pick(a->u_stride[1], xd);
  p.dl_sb = pick(a->delta_stride[0], xb);
  p.dl_sd = pick(a->delta_stride[1], xd);
  p.z_sb = pick(a->z_stride[0], xb);
  p.z_sd = pick(a->z_stride[1], xd);
  p.y_sb = pick(a->y_stride[0], xb);
  p.y_sd = pick(a->y_stride[1], xd);
  p.B_sb = pick(a->B_stride[0], bcb);
  p.B_sn = pick(a->B_stride[1], bcn);
  p.C_sb = pick(a->C_stride[0], bcb);
  p.C_sn = pick(a->C_stride[1], bcn);
  const int64_t strides[] = {p.u_sb, p.u_sd, p.dl_sb, p.dl_sd, p.z_sb, p.z_sd, p.y_sb,
                             p.y_sd, p.B_sb, p.B_sn, p.C_sb, p.C_sn, p.B_sg, p.C_sg};
  for (int64_t s : strides)
    if (s < 0) return SSM_ERR_INVALID_ARG;
  p.A = a->A;
  p.D = a->D;
  p.bias = a->delta_bias;
  p.softplus = a->delta_softplus ? 1 : 0;
  p.h0 = a->h0;
  p.h_last = a->h_last;

  // 16-byte rows take the cp.async path.
  bool vec = true;
  for (const void* t : tensors)
    if (t != nullptr && !aligned(t, 16)) vec = false;
  const int64_t need = 16 / static_cast<int64_t>(es);
  for (int64_t s : strides)
    if (s % need != 0) vec = false;
  out->vec = vec;

  // L-segments: split the sequence when the channels alone leave the GPU idle.
  const int64_t ctas = ((a->dim + fwd::kCH - 1) / fwd::kCH) * a->batch;
  const int64_t sms = device_sm_count();
  const int64_t target = sms * 8;
  int64_t nseg = 1;
  if (any_work && L > 0 && ctas > 0 && ctas < 2 * sms) {
    const int64_t max_seg = (L + fwd::kTL - 1) / fwd::kTL;
    nseg = (target + ctas - 1) / ctas;
    if (nseg > max_seg) nseg = max_seg;
    if (nseg > 65535) nseg = 65535;
  }
  int64_t seg_len = L;
  if (nseg > 1) {
    seg_len = (L + nseg - 1) / nseg;
    seg_len = (seg_len + fwd::kTL - 1) / fwd::kTL * fwd::kTL;
    nseg = (L + seg_len - 1) / seg_len;
  }
  if (seg_len <= 0) seg_len = 1;
  p.nseg = nseg;
  p.seg_len = seg_len;
  out->ws_bytes = nseg > 1 ? static_cast<size_t>(nseg - 1) * a->batch * a->dim *
                                 (fwd::kMaxN + 1) * sizeof(float)
                           : 0;
  return SSM_OK;
}

template <typename T, int MODE, bool HAS_Z, bool VEC, bool CONV, bool VARLEN>
ssm_status_t launch_fwd(const ScanParams& p, cudaStream_t stream) {
  auto kernel = fwd::scan_fwd_kernel<T, MODE, HAS_Z, VEC, CONV, VARLEN>;
  const size_t smem = sizeof(fwd::Smem<T, CONV, fwd::packed_bc<T, MODE, HAS_Z>()>);
  ssm_status_t st = cuda_status(set_smem(reinterpret_cast<const void*>(kernel), smem),
                                "scan_fwd: shared-memory opt-in");
  if (st != SSM_OK) return st;
  const dim3 grid(static_cast<unsigned>((p.dim + fwd::kCH - 1) / fwd::kCH),
                  static_cast<unsigned>(p.batch),
                  static_cast<unsigned>(MODE == fwd::kAgg ? p.nseg - 1 : p.nseg));
  kernel<<<grid, fwd::kThreads, smem, stream>>>(p);
  return cuda_status(cudaGetLastError(), MODE == fwd::kAgg ? "scan_fwd: aggregate pass launch"
                                                           : "scan_fwd: scan pass launch");
}

template <typename T, bool VEC, bool CONV, bool VARLEN = false>
ssm_status_t run_fwd(const ScanParams& p, cudaStream_t stream) {
  ssm_status_t st = SSM_OK;
  if (p.nseg > 1) {
    st = launch_fwd<T, fwd::kAgg, false, VEC, CONV, VARLEN>(p, stream);
    if (st != SSM_OK) return st;
    const int64_t total = p.batch * p.dim * fwd::kMaxN;
    const int threads = 256;
    fwd::scan_carry_kernel<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0,
                             stream>>>(p);
    st = cuda_status(cudaGetLastError(), "scan_fwd: carry launch");
    if (st != SSM_OK) return st;
  }
  return p.z != nullptr ? launch_fwd<T, fwd::kFull, true, VEC, CONV, VARLEN>(p, stream)
                        : launch_fwd<T, fwd::kFull, false, VEC, CONV, VARLEN>(p, stream);
}

// ---------------------------------------------------------------------------
// decode step
// ---------------------------------------------------------------------------
template <typename T, bool HAS_Z, bool VEC4>
ssm_status_t launch_step(const StepParams& p, cudaStream_t stream) {
  const int64_t threads = p.batch * p.dim * step::kNG;
  const int64_t blocks = (threads + step::kThreads - 1) / step::kThreads;
  if (blocks > INT_MAX) return SSM_ERR_UNSUPPORTED;
  step::scan_step_kernel<T, HAS_Z, VEC4>
      <<<static_cast<unsigned>(blocks), step::kThreads, 0, stream>>>(p);
  return cuda_status(cudaGetLastError(), "scan_step: launch");
}

template <typename T>
ssm_status_t run_step(const StepParams& p, bool vec4, cudaStream_t stream) {
  if (p.z != nullptr)
    return vec4 ? launch_step<T, true, true>(p, stream) : launch_step<T, true, false>(p, stream);
  return vec4 ? launch_step<T, false, true>(p, stream) : launch_step<T, false, false>(p, stream);
}

// ---------------------------------------------------------------------------
// Mamba-2 chunked scan
// ---------------------------------------------------------------------------
constexpr size_t kSsdStatusBytes = 256;  // status word at the start of the workspace

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// A bf16 tensor map with 128-byte swizzle and zero fill: dims[0] is the
// contiguous dimension, strides (bytes) are those of dims[1..rank-1].
bool encode_bf16_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    if (i + 1 < rank) st[i] = strides[i];
  }
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
            const_cast<void*>(base), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The operand maps of the chunked scan (boxes of 64 elements along the
// contiguous dimension and one chunk of steps, or 64 rows of the state).
ssm_status_t make_ssd_maps(const SsdParams& p, SsdMaps* m) {
  const uint64_t B = p.batch, L = p.seqlen, H = p.nheads, P = ssd::kP, N = ssd::kN;
  const uint32_t Q = static_cast<uint32_t>(p.chunk);
  const uint64_t xd[3] = {H * P, L, B}, xs[2] = {H * P * 2, L * H * P * 2};
  const uint32_t xb[3] = {64, Q, 1};
  const uint64_t bd[3] = {N, L, B}, bs[2] = {N * 2, L * N * 2};
  const uint32_t bb[3] = {64, Q, 1};
  const uint64_t sd[2] = {N, B * H * static_cast<uint64_t>(p.nchunks) * P}, ss[1] = {N * 2};
  const uint32_t sb[2] = {64, 64};
  const bool ok = encode_bf16_map(&m->x, p.x, 3, xd, xs, xb) &&
                  encode_bf16_map(&m->B, p.B, 3, bd, bs, bb) &&
                  encode_bf16_map(&m->C, p.C, 3, bd, bs, bb) &&
                  encode_bf16_map(&m->sprev, p.sprev, 2, sd, ss, sb);
  if (!ok) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "ssd: tensor-map encoding failed (driver entry point unavailable or "
                  "operand layout rejected)");
    return SSM_ERR_CUDA;
  }
  return SSM_OK;
}

ssm_status_t plan_ssd(const ssm_ssd_args_t* a, SsdParams* p, size_t* ws_bytes, bool check_ptrs) {
  if (a == nullptr) return SSM_ERR_INVALID_ARG;
  if (a->batch < 0 || a->seqlen < 0 || a->nheads < 0 || a->headdim < 0 || a->dstate < 0)
    return SSM_ERR_INVALID_ARG;
  if (a->dtype != SSM_F32 && a->dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
  if (a->dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if (a->dstate != ssd::kN || a->headdim != ssd::kP) return SSM_ERR_UNSUPPORTED;
  if (a->chunk != 128 && a->chunk != 256) return SSM_ERR_UNSUPPORTED;
  if (a->batch > 65535 || a->nheads > 65535) return SSM_ERR_UNSUPPORTED;
  const bool any = a->batch > 0 && a->nheads > 0;
  if (any && check_ptrs) {
    if (a->A == nullptr) return SSM_ERR_INVALID_ARG;
    if (a->seqlen > 0 && (a->x == nullptr || a->delta == nullptr || a->B == nullptr ||
                          a->C == nullptr || a->y == nullptr))
      return SSM_ERR_INVALID_ARG;
  }
  const void* vec[] = {a->x, a->B, a->C, a->y, a->z};
  for (const void* t : vec)
    if (t != nullptr && !aligned(t, 16)) return SSM_ERR_ALIGNMENT;
  if (a->delta != nullptr && !aligned(a->delta, 2)) return SSM_ERR_ALIGNMENT;
  const void* f32s[] = {a->A, a->D, a->delta_bias, a->h0, a->h_last};
  for (const void* t : f32s)
    if (t != nullptr && !aligned(t, 4)) return SSM_ERR_ALIGNMENT;
  p->batch = a->batch;
  p->seqlen = a->seqlen;
  p->nheads = a->nheads;
  p->headdim = a->headdim;
  p->dstate = a->dstate;
  p->chunk = a->chunk;
  p->nchunks = (a->seqlen + a->chunk - 1) / a->chunk;
  if (p->nchunks > 2147483647) return SSM_ERR_UNSUPPORTED;
  // TMA coordinates are 32-bit: steps, and rows of the carried states.
  if (a->seqlen > INT32_MAX ||
      static_cast<double>(a->batch) * a->nheads * p->nchunks * ssd::kP > INT32_MAX)
    return SSM_ERR_UNSUPPORTED;
  p->x = static_cast<const __nv_bfloat16*>(a->x);
  p->delta = static_cast<const __nv_bfloat16*>(a->delta);
  p->A = a->A;
  p->B = static_cast<const __nv_bfloat16*>(a->B);
  p->C = static_cast<const __nv_bfloat16*>(a->C);
  p->D = a->D;
  p->bias = a->delta_bias;
  p->softplus = a->delta_softplus ? 1 : 0;
  p->z = static_cast<const __nv_bfloat16*>(a->z);
  p->h0 = a->h0;
  p->y = static_cast<__nv_bfloat16*>(a->y);
  p->h_last = a->h_last;
  const size_t states = static_cast<size_t>(a->batch) * a->nheads * p->nchunks * ssd::kN * ssd::kP;
  const size_t cums = (static_cast<size_t>(a->batch) * a->nheads * p->nchunks * sizeof(float) + 255) /
                      256 * 256;
  const size_t steps = static_cast<size_t>(a->batch) * a->nheads * p->nchunks * 2 * a->chunk;
  *ws_bytes = kSsdStatusBytes + states * sizeof(float) + cums + states * sizeof(__nv_bfloat16) +
              steps * sizeof(float);
  // Heads per block: the chunk-state and scan kernels run one block per SM;
  // choose the group that minimises (rounds of blocks) x (heads per block + the
  // shared C B^T product, worth about 1.5 heads).
  const int64_t sms = device_sm_count();
  int64_t best = 1;
  double best_cost = 1e300;
  for (int64_t g = 1; g <= a->nheads && g <= ssd::kMaxGroup; ++g) {
    const int64_t groups = (a->nheads + g - 1) / g;
    if (g > 1 && (a->nheads + g - 2) / (g - 1) == groups) continue;  // same split, more heads
    const int64_t blocks = a->batch * p->nchunks * groups;
    const int64_t rounds = blocks == 0 ? 0 : (blocks + sms - 1) / sms;
    const double cost = static_cast<double>(rounds) * (static_cast<double>(g) + 1.5);
    if (cost < best_cost) {
      best_cost = cost;
      best = g;
    }
  }
  p->hgroup = best;
  return SSM_OK;
}

template <int Q>
ssm_status_t run_ssd(const SsdParams& p, const SsdMaps& maps, cudaStream_t stream) {
  ssm_status_t st = SSM_OK;
  const unsigned groups = static_cast<unsigned>((p.nheads + p.hgroup - 1) / p.hgroup);
  const dim3 grid(groups, static_cast<unsigned>(p.nchunks), static_cast<unsigned>(p.batch));
  if (p.nchunks > 0) {
    auto chunk_state = ssd::ssd_chunk_state_kernel<Q>;
    const size_t smem = sizeof(ssd::ChunkStateSmem<Q>) + 1024;
    st = cuda_status(set_smem(reinterpret_cast<const void*>(chunk_state), smem), "ssd: opt-in");
    if (st != SSM_OK) return st;
    chunk_state<<<grid, ssd::kThreads, smem, stream>>>(p, maps);
    st = cuda_status(cudaGetLastError(), "ssd: chunk-state launch");
    if (st != SSM_OK) return st;
  }
  const int64_t elems = p.batch * p.nheads * ssd::kP * ssd::kN;
  ssd::ssd_pass_kernel<<<static_cast<unsigned>((elems + 255) / 256), 256, 0, stream>>>(p);
  st = cuda_status(cudaGetLastError(), "ssd: state pass launch");
  if (st != SSM_OK || p.nchunks == 0) return st;
  const size_t smem_scan = sizeof(ssd::ScanSmem<Q>) + 1024;
  if (p.z != nullptr) {
    auto scan = ssd::ssd_scan_kernel<Q, true>;
    st = cuda_status(set_smem(reinterpret_cast<const void*>(scan), smem_scan), "ssd: opt-in");
    if (st != SSM_OK) return st;
    scan<<<grid, ssd::kScanThreads, smem_scan, stream>>>(p, maps);
  } else {
    auto scan = ssd::ssd_scan_kernel<Q, false>;
    st = cuda_status(set_smem(reinterpret_cast<const void*>(scan), smem_scan), "ssd: opt-in");
    if (st != SSM_OK) return st;
    scan<<<grid, ssd::kScanThreads, smem_scan, stream>>>(p, maps);
  }
  return cuda_status(cudaGetLastError(), "ssd: chunk scan launch");
}

// ---------------------------------------------------------------------------
// Static scratch for ssm_scan_fwd_noalloc.  In host code the name below is a
// host-side stand-in, not a device address: the address kernels must use is
// looked up with cudaGetSymbolAddress, once per device.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = SSM_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

cudaError_t noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* ptrs[kMaxDevices] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return cudaSuccess;
}

// ---- host-resident scan: batch slices pipelined through device staging ------

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

struct HostPlan {
  int64_t sb = 1, nslices = 0;
  size_t es = 0, x_bytes = 0, bc_bytes = 0, h_bytes = 0;  // one full slice of u / B / h
  size_t off_A = 0, off_D = 0, off_bias = 0, off_ws = 0, ws_bytes = 0, off_slot = 0;
  // within a slot
  size_t off_u = 0, off_dl = 0, off_z = 0, off_B = 0, off_C = 0, off_y = 0, off_h0 = 0, off_h = 0;
  size_t slot_bytes = 0, total = 0;
};

ssm_status_t plan_host(const ssm_scan_args_t* a, int64_t sb, HostPlan* hp) {
  if (a == nullptr || sb < 1) return SSM_ERR_INVALID_ARG;
  const int64_t* strides[] = {a->u_stride, a->delta_stride, a->z_stride,
                              a->y_stride, a->B_stride, a->C_stride};
  for (const int64_t* st : strides)
    if (st[0] != 0 || st[1] != 0) return SSM_ERR_UNSUPPORTED;
  if (a->B_group_stride != 0 || a->C_group_stride != 0) return SSM_ERR_UNSUPPORTED;
  ScanPlan whole;
  ssm_status_t st = plan_scan(a, &whole);  // sizes, flags and the host pointers
  if (st != SSM_OK) return st;
  hp->sb = sb < a->batch ? sb : (a->batch > 0 ? a->batch : 1);
  hp->nslices = (a->batch + hp->sb - 1) / hp->sb;
  // scratch of the scan of a full slice and of the last (possibly smaller) one
  size_t ws = 0;
  for (int64_t nb : {hp->sb, a->batch - (hp->nslices - 1) * hp->sb}) {
    if (nb <= 0) continue;
    ssm_scan_args_t sa = *a;
    sa.batch = nb;
    ScanPlan sp;
    st = plan_scan(&sa, &sp, false);
    if (st != SSM_OK) return st;
    if (sp.ws_bytes > ws) ws = sp.ws_bytes;
  }
  const size_t es = elem_size(a->dtype);
  const size_t D = static_cast<size_t>(a->dim), N = static_cast<size_t>(a->dstate);
  const size_t NB = N * static_cast<size_t>(a->ngroups > 1 ? a->ngroups : 1);  // B/C rows per batch
  const size_t L = static_cast<size_t>(a->seqlen), S = static_cast<size_t>(hp->sb);
  hp->es = es;
  hp->x_bytes = S * D * L * es;
  hp->bc_bytes = S * NB * L * es;
  hp->h_bytes = S * D * N * sizeof(float);
  size_t o = 0;
  hp->off_A = o;    o += round256(D * N * sizeof(float));
  hp->off_D = o;    o += a->D ? round256(D * sizeof(float)) : 0;
  hp->off_bias = o; o += a->delta_bias ? round256(D * sizeof(float)) : 0;
  hp->off_ws = o;   o += round256(ws);
  hp->ws_bytes = ws;
  hp->off_slot = o;
  size_t q = 0;
  hp->off_u = q;  q += round256(hp->x_bytes);
  hp->off_dl = q; q += round256(hp->x_bytes);
  hp->off_z = q;  q += a->z ? round256(hp->x_bytes) : 0;
  hp->off_B = q;  q += round256(hp->bc_bytes);
  hp->off_C = q;  q += round256(hp->bc_bytes);
  hp->off_y = q;  q += round256(hp->x_bytes);
  hp->off_h0 = q; q += a->h0 ? round256(hp->h_bytes) : 0;
  hp->off_h = q;  q += a->h_last ? round256(hp->h_bytes) : 0;
  hp->slot_bytes = q;
  hp->total = o + 2 * q;
  return SSM_OK;
}

// Two copy streams per device (host-to-device, device-to-host), created on
// first use and kept for the life of the process.
ssm_status_t copy_streams(cudaStream_t* in, cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t streams[kMaxDevices][2] = {};
  int dev = 0;
  ssm_status_t st = cuda_status(cudaGetDevice(&dev), "scan_fwd_host: current device");
  if (st != SSM_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return SSM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < 2; ++i) {
    if (streams[dev][i] == nullptr) {
      st = cuda_status(cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking),
                       "scan_fwd_host: copy stream");
      if (st != SSM_OK) return st;
    }
  }
  *in = streams[dev][0];
  *out = streams[dev][1];
  return SSM_OK;
}

// The queued work of one ssm_scan_fwd_host call (see include/ssmscan.h).
ssm_status_t run_host(const ssm_scan_args_t* a, const HostPlan& hp, unsigned char* stg,
                      cudaStream_t stream) {
  cudaStream_t sin = nullptr, sout = nullptr;
  ssm_status_t st = copy_streams(&sin, &sout);
  if (st != SSM_OK) return st;
  // start, then per slot: inputs in, scan done, outputs out
  cudaEvent_t ev[7] = {};
  for (cudaEvent_t& e : ev) {
    st = cuda_status(cudaEventCreateWithFlags(&e, cudaEventDisableTiming), "scan_fwd_host: event");
    if (st != SSM_OK) break;
  }
  cudaEvent_t ev_start = ev[0], *in_done = ev + 1, *comp_done = ev + 3, *out_done = ev + 5;
  auto chk = [&](cudaError_t e, const char* what) {
    if (st == SSM_OK) st = cuda_status(e, what);
    return st == SSM_OK;
  };
  auto h2d = [&](void* dst, const void* src, size_t n) {
    return n == 0 || chk(cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, sin),
                         "scan_fwd_host: copy to device");
  };
  auto d2h = [&](void* dst, const void* src, size_t n) {
    return n == 0 || chk(cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, sout),
                         "scan_fwd_host: copy to host");
  };
  const size_t D = static_cast<size_t>(a->dim), N = static_cast<size_t>(a->dstate);
  const size_t NB = N * static_cast<size_t>(a->ngroups > 1 ? a->ngroups : 1);  // B/C rows per batch
  const size_t L = static_cast<size_t>(a->seqlen), es = hp.es;
  if (st == SSM_OK && chk(cudaEventRecord(ev_start, stream), "scan_fwd_host: record") &&
      chk(cudaStreamWaitEvent(sin, ev_start, 0), "scan_fwd_host: wait") &&
      chk(cudaStreamWaitEvent(sout, ev_start, 0), "scan_fwd_host: wait") &&
      h2d(stg + hp.off_A, a->A, D * N * sizeof(float)) &&
      (a->D == nullptr || h2d(stg + hp.off_D, a->D, D * sizeof(float))) &&
      (a->delta_bias == nullptr || h2d(stg + hp.off_bias, a->delta_bias, D * sizeof(float)))) {
    for (int64_t s = 0; s < hp.nslices && st == SSM_OK; ++s) {
      const int k = static_cast<int>(s & 1);
      unsigned char* slot = stg + hp.off_slot + k * hp.slot_bytes;
      const int64_t b0 = s * hp.sb;
      const int64_t nb = a->batch - b0 < hp.sb ? a->batch - b0 : hp.sb;
      const size_t xo = static_cast<size_t>(b0) * D * L * es, xn = static_cast<size_t>(nb) * D * L * es;
      const size_t bo = static_cast<size_t>(b0) * NB * L * es, bn = static_cast<size_t>(nb) * NB * L * es;
      const size_t ho = static_cast<size_t>(b0) * D * N * sizeof(float);
      const size_t hn = static_cast<size_t>(nb) * D * N * sizeof(float);
      auto in = [](const void* base, size_t off) {
        return static_cast<const unsigned char*>(base) + off;
      };
      // slot k's inputs were last read by the scan of slice s - 2
      if (s >= 2 && !chk(cudaStreamWaitEvent(sin, comp_done[k], 0), "scan_fwd_host: wait")) break;
      if (!(h2d(slot + hp.off_u, in(a->u, xo), xn) && h2d(slot + hp.off_dl, in(a->delta, xo), xn) &&
            (a->z == nullptr || h2d(slot + hp.off_z, in(a->z, xo), xn)) &&
            h2d(slot + hp.off_B, in(a->B, bo), bn) && h2d(slot + hp.off_C, in(a->C, bo), bn) &&
            (a->h0 == nullptr || h2d(slot + hp.off_h0, in(a->h0, ho), hn)) &&
            chk(cudaEventRecord(in_done[k], sin), "scan_fwd_host: record") &&
            chk(cudaStreamWaitEvent(stream, in_done[k], 0), "scan_fwd_host: wait")))
        break;
      // slot k's outputs of slice s - 2 must have left before the scan rewrites them
      if (s >= 2 && !chk(cudaStreamWaitEvent(stream, out_done[k], 0), "scan_fwd_host: wait")) break;
      ssm_scan_args_t sa = *a;
      sa.batch = nb;
      sa.u = slot + hp.off_u;
      sa.delta = slot + hp.off_dl;
      sa.z = a->z ? slot + hp.off_z : nullptr;
      sa.B = slot + hp.off_B;
      sa.C = slot + hp.off_C;
      sa.y = slot + hp.off_y;
      sa.h0 = a->h0 ? reinterpret_cast<const float*>(slot + hp.off_h0) : nullptr;
      sa.h_last = a->h_last ? reinterpret_cast<float*>(slot + hp.off_h) : nullptr;
      sa.A = reinterpret_cast<const float*>(stg + hp.off_A);
      sa.D = a->D ? reinterpret_cast<const float*>(stg + hp.off_D) : nullptr;
      sa.delta_bias = a->delta_bias ? reinterpret_cast<const float*>(stg + hp.off_bias) : nullptr;
      st = ssm_scan_fwd(&sa, hp.ws_bytes ? stg + hp.off_ws : nullptr, hp.ws_bytes,
                        reinterpret_cast<ssm_stream_t>(stream));
      if (st != SSM_OK) break;
      if (!(chk(cudaEventRecord(comp_done[k], stream), "scan_fwd_host: record") &&
            chk(cudaStreamWaitEvent(sout, comp_done[k], 0), "scan_fwd_host: wait") &&
            d2h(static_cast<unsigned char*>(a->y) + xo, slot + hp.off_y, xn) &&
            (a->h_last == nullptr ||
             d2h(reinterpret_cast<unsigned char*>(a->h_last) + ho, slot + hp.off_h, hn)) &&
            chk(cudaEventRecord(out_done[k], sout), "scan_fwd_host: record")))
        break;
    }
    // the caller's stream finishes when every copy back has landed
    for (int k = 0; k < 2 && k < hp.nslices && st == SSM_OK; ++k)
      chk(cudaStreamWaitEvent(stream, out_done[k], 0), "scan_fwd_host: wait");
  }
  for (cudaEvent_t e : ev)
    if (e != nullptr) cudaEventDestroy(e);  // released once the queued work has used them
  return st;
}

// ssm_scan_fwd, with the convolution stage in front when `conv` is given,
// or over a packed variable-length batch when `cu_seqlens` is.
ssm_status_t scan_fwd_impl(const ssm_scan_args_t* args, const ssm_conv_args_t* conv,
                           void* workspace, size_t workspace_bytes, ssm_stream_t stream_,
                           const int32_t* cu_seqlens = nullptr, int64_t nseq = 0) {
  ScanPlan plan;
  ssm_status_t st = plan_scan(args, &plan);
  if (st != SSM_OK) return st;
  ScanParams& p = plan.p;
  p.conv_width = 0;
  p.conv_w = p.conv_b = p.conv_prev = nullptr;
  p.cu_seqlens = cu_seqlens;
  p.nseq = nseq;
  if (conv != nullptr) {
    if (conv->width < 1 || conv->width > fwd::kMaxConv) return SSM_ERR_UNSUPPORTED;
    if (p.batch > 0 && p.dim > 0 && conv->weight == nullptr) return SSM_ERR_INVALID_ARG;
    const void* f32s[] = {conv->weight, conv->bias, conv->x_prev};
    for (const void* t : f32s)
      if (t != nullptr && !aligned(t, 4)) return SSM_ERR_ALIGNMENT;
    p.conv_width = static_cast<int>(conv->width);
    p.conv_w = conv->weight;
    p.conv_b = conv->bias;
    p.conv_prev = conv->width > 1 ? conv->x_prev : nullptr;
  }
  if (p.batch == 0 || p.dim == 0) return SSM_OK;
  if (plan.ws_bytes > 0) {
    if (workspace == nullptr || workspace_bytes < plan.ws_bytes) return SSM_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return SSM_ERR_ALIGNMENT;
    float* ws = static_cast<float*>(workspace);
    const int64_t slots = (p.nseg - 1) * p.batch * p.dim;
    p.carry_h = ws;
    p.carry_dt = ws + slots * fwd::kMaxN;
  } else {
    p.carry_h = nullptr;
    p.carry_dt = nullptr;
  }
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const bool bf16 = args->dtype == SSM_BF16;
  if (cu_seqlens != nullptr) {
    if (bf16)
      return plan.vec ? run_fwd<__nv_bfloat16, true, false, true>(p, stream)
                      : run_fwd<__nv_bfloat16, false, false, true>(p, stream);
    return plan.vec ? run_fwd<float, true, false, true>(p, stream)
                    : run_fwd<float, false, false, true>(p, stream);
  }
  if (conv != nullptr) {
    if (bf16)
      return plan.vec ? run_fwd<__nv_bfloat16, true, true>(p, stream)
                      : run_fwd<__nv_bfloat16, false, true>(p, stream);
    return plan.vec ? run_fwd<float, true, true>(p, stream) : run_fwd<float, false, true>(p, stream);
  }
  if (bf16)
    return plan.vec ? run_fwd<__nv_bfloat16, true, false>(p, stream)
                    : run_fwd<__nv_bfloat16, false, false>(p, stream);
  return plan.vec ? run_fwd<float, true, false>(p, stream) : run_fwd<float, false, false>(p, stream);
}

// ---- gradients -------------------------------------------------------------------------
ssm_status_t plan_bwd(const ssm_scan_args_t* a, BwdParams* p, size_t* ws_bytes, bool check_ptrs) {
  ScanPlan plan;
  ssm_status_t st = plan_scan(a, &plan, false);  // y and h_last play no part here
  if (st != SSM_OK) return st;
  if (check_ptrs && a->batch > 0 && a->dim > 0) {
    if (a->A == nullptr) return SSM_ERR_INVALID_ARG;
    if (a->seqlen > 0 && (a->u == nullptr || a->delta == nullptr || a->B == nullptr ||
                          a->C == nullptr))
      return SSM_ERR_INVALID_ARG;
  }
  const int64_t* strides[] = {a->u_stride, a->delta_stride, a->z_stride,
                              a->y_stride, a->B_stride, a->C_stride};
  for (const int64_t* s : strides)
    if (s[0] != 0 || s[1] != 0) return SSM_ERR_UNSUPPORTED;
  if (a->ngroups > 1) return SSM_ERR_UNSUPPORTED;
  p->batch = a->batch;
  p->dim = a->dim;
  p->dstate = a->dstate;
  p->seqlen = a->seqlen;
  p->u = a->u;
  p->delta = a->delta;
  p->z = a->z;
  p->B = a->B;
  p->C = a->C;
  p->A = a->A;
  p->D = a->D;
  p->bias = a->delta_bias;
  p->softplus = a->delta_softplus ? 1 : 0;
  p->h0 = a->h0;
  p->nblk = (a->seqlen + bwd::kBlk - 1) / bwd::kBlk;
  p->nchb = (a->dim + bwd::kCh - 1) / bwd::kCh;
  const size_t ckpt = static_cast<size_t>(a->batch) * a->dim * bwd::kStates * p->nblk;
  const size_t part = 2 * static_cast<size_t>(p->nchb) * a->batch * a->dstate * a->seqlen;
  *ws_bytes = (ckpt + part) * sizeof(float);
  return SSM_OK;
}

}  // namespace

extern "C" {

size_t ssm_scan_bwd_workspace_size(const ssm_scan_args_t* args) {
  BwdParams p;
  size_t ws = 0;
  if (plan_bwd(args, &p, &ws, false) != SSM_OK) return static_cast<size_t>(-1);
  return ws;
}

ssm_status_t ssm_scan_bwd(const ssm_scan_args_t* args, const float* dy, const ssm_scan_grads_t* g,
                          void* workspace, size_t workspace_bytes, ssm_stream_t stream_) {
  if (g == nullptr) return SSM_ERR_INVALID_ARG;
  BwdParams p;
  size_t ws = 0;
  ssm_status_t st = plan_bwd(args, &p, &ws, true);
  if (st != SSM_OK) return st;
  if (p.batch == 0 || p.dim == 0) return SSM_OK;
  if (dy == nullptr && p.seqlen > 0) return SSM_ERR_INVALID_ARG;
  if (g->dA == nullptr || g->dB == nullptr || g->dC == nullptr) return SSM_ERR_INVALID_ARG;
  const void* f32s[] = {dy, g->du, g->ddelta, g->dz, g->dA, g->dB, g->dC, g->dD, g->ddelta_bias,
                        g->dh0};
  for (const void* t : f32s)
    if (t != nullptr && !aligned(t, 4)) return SSM_ERR_ALIGNMENT;
  if (ws > 0 && (workspace == nullptr || workspace_bytes < ws)) return SSM_ERR_WORKSPACE;
  if (workspace != nullptr && !aligned(workspace, 16)) return SSM_ERR_ALIGNMENT;
  p.dy = dy;
  p.du = g->du;
  p.ddelta = g->ddelta;
  p.dz = args->z ? g->dz : nullptr;
  p.dA = g->dA;
  p.dB = g->dB;
  p.dC = g->dC;
  p.dD = args->D ? g->dD : nullptr;
  p.dbias = args->delta_bias ? g->ddelta_bias : nullptr;
  p.dh0 = args->h0 ? g->dh0 : nullptr;
  p.ckpt = static_cast<float*>(workspace);
  p.part = p.ckpt + static_cast<size_t>(p.batch) * p.dim * bwd::kStates * p.nblk;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  // the accumulated gradients start from zero (dB and dC are written whole)
  const size_t bnl = static_cast<size_t>(p.batch) * p.dstate * p.seqlen;
  st = cuda_status(cudaMemsetAsync(p.dA, 0, static_cast<size_t>(p.dim) * p.dstate * sizeof(float),
                                   stream), "scan_bwd: zero dA");
  if (st == SSM_OK && p.dD)
    st = cuda_status(cudaMemsetAsync(p.dD, 0, p.dim * sizeof(float), stream), "scan_bwd: zero dD");
  if (st == SSM_OK && p.dbias)
    st = cuda_status(cudaMemsetAsync(p.dbias, 0, p.dim * sizeof(float), stream),
                     "scan_bwd: zero bias gradient");
  if (st != SSM_OK) return st;
  const dim3 grid(static_cast<unsigned>((p.dim + bwd::kCh - 1) / bwd::kCh),
                  static_cast<unsigned>(p.batch));
  if (args->dtype == SSM_BF16) {
    const size_t smem = sizeof(bwd::Smem<__nv_bfloat16>);
    auto kernel = bwd::scan_bwd_kernel<__nv_bfloat16>;
    st = cuda_status(set_smem(reinterpret_cast<const void*>(kernel), smem), "scan_bwd: opt-in");
    if (st != SSM_OK) return st;
    kernel<<<grid, bwd::kThreads, smem, stream>>>(p);
  } else {
    const size_t smem = sizeof(bwd::Smem<float>);
    auto kernel = bwd::scan_bwd_kernel<float>;
    st = cuda_status(set_smem(reinterpret_cast<const void*>(kernel), smem), "scan_bwd: opt-in");
    if (st != SSM_OK) return st;
    kernel<<<grid, bwd::kThreads, smem, stream>>>(p);
  }
  st = cuda_status(cudaGetLastError(), "scan_bwd: launch");
  if (st != SSM_OK || bnl == 0) return st;
  bwd::scan_bwd_reduce_bc<<<static_cast<unsigned>((bnl + 255) / 256), 256, 0, stream>>>(p);
  return cuda_status(cudaGetLastError(), "scan_bwd: dB / dC reduction launch");
}


size_t ssm_scan_fwd_workspace_size(const ssm_scan_args_t* args) {
  ScanPlan plan;
  if (plan_scan(args, &plan, false) != SSM_OK) return static_cast<size_t>(-1);
  return plan.ws_bytes;
}

ssm_status_t ssm_scan_fwd(const ssm_scan_args_t* args, void* workspace, size_t workspace_bytes,
                          ssm_stream_t stream_) {
  return scan_fwd_impl(args, nullptr, workspace, workspace_bytes, stream_);
}

ssm_status_t ssm_scan_fwd_conv(const ssm_scan_args_t* args, const ssm_conv_args_t* conv,
                               void* workspace, size_t workspace_bytes, ssm_stream_t stream) {
  if (conv == nullptr) return SSM_ERR_INVALID_ARG;
  return scan_fwd_impl(args, conv, workspace, workspace_bytes, stream);
}

ssm_status_t ssm_scan_fwd_varlen(const ssm_scan_args_t* args, const int32_t* cu_seqlens,
                                 int64_t nseq, void* workspace, size_t workspace_bytes,
                                 ssm_stream_t stream) {
  if (args == nullptr || cu_seqlens == nullptr || nseq < 1) return SSM_ERR_INVALID_ARG;
  if (args->batch != 1 || args->h0 != nullptr || args->seqlen > INT32_MAX)
    return SSM_ERR_UNSUPPORTED;
  if (!aligned(cu_seqlens, 4)) return SSM_ERR_ALIGNMENT;
  return scan_fwd_impl(args, nullptr, workspace, workspace_bytes, stream, cu_seqlens, nseq);
}

size_t ssm_scan_fwd_host_staging_size(const ssm_scan_args_t* args, int64_t slice_batch) {
  HostPlan hp;
  if (plan_host(args, slice_batch, &hp) != SSM_OK) return static_cast<size_t>(-1);
  return hp.total;
}

ssm_status_t ssm_scan_fwd_host(const ssm_scan_args_t* args, int64_t slice_batch, void* staging,
                               size_t staging_bytes, ssm_stream_t stream) {
  HostPlan hp;
  ssm_status_t st = plan_host(args, slice_batch, &hp);
  if (st != SSM_OK) return st;
  if (args->batch == 0 || args->dim == 0) return SSM_OK;
  if (staging == nullptr || staging_bytes < hp.total) return SSM_ERR_WORKSPACE;
  if (!aligned(staging, 256)) return SSM_ERR_ALIGNMENT;
  return run_host(args, hp, static_cast<unsigned char*>(staging),
                  reinterpret_cast<cudaStream_t>(stream));
}

ssm_status_t ssm_scan_fwd_noalloc(const ssm_scan_args_t* args, ssm_stream_t stream) {
  ScanPlan plan;
  ssm_status_t st = plan_scan(args, &plan);
  if (st != SSM_OK) return st;
  if (plan.ws_bytes > kNoAllocScratchBytes) {
    snprintf(g_last_error, sizeof(g_last_error),
             "ssm_scan_fwd_noalloc: needs %zu bytes of scratch, the static scratch holds %zu",
             plan.ws_bytes, kNoAllocScratchBytes);
    return SSM_ERR_WORKSPACE;
  }
  if (plan.p.batch == 0 || plan.p.dim == 0) return SSM_OK;
  void* ws = nullptr;
  if (plan.ws_bytes > 0) {
    st = cuda_status(noalloc_scratch(&ws), "ssm_scan_fwd_noalloc: scratch address lookup");
    if (st != SSM_OK) return st;
  }
  return ssm_scan_fwd(args, ws, plan.ws_bytes, stream);
}

ssm_status_t ssm_scan_step(const ssm_step_args_t* a, ssm_stream_t stream_) {
  if (a == nullptr) return SSM_ERR_INVALID_ARG;
  if (a->batch < 0 || a->dim < 0) return SSM_ERR_INVALID_ARG;
  if (a->dtype != SSM_F32 && a->dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
  if (a->dstate < 1 || a->dstate > step::kNG * step::kNPT) return SSM_ERR_UNSUPPORTED;
  if (a->batch == 0 || a->dim == 0) return SSM_OK;
  if (a->u == nullptr || a->delta == nullptr || a->B == nullptr || a->C == nullptr ||
      a->A == nullptr || a->state == nullptr || a->y == nullptr)
    return SSM_ERR_INVALID_ARG;
  const size_t es = elem_size(a->dtype);
  const void* tensors[] = {a->u, a->delta, a->z, a->B, a->C, a->y};
  for (const void* t : tensors)
    if (t != nullptr && !aligned(t, es)) return SSM_ERR_ALIGNMENT;
  const void* f32s[] = {a->A, a->D, a->delta_bias, a->state};
  for (const void* t : f32s)
    if (t != nullptr && !aligned(t, 4)) return SSM_ERR_ALIGNMENT;
  StepParams p;
  p.batch = a->batch;
  p.dim = a->dim;
  p.dstate = a->dstate;
  p.u = a->u;
  p.delta = a->delta;
  p.z = a->z;
  p.B = a->B;
  p.C = a->C;
  p.A = a->A;
  p.D = a->D;
  p.bias = a->delta_bias;
  p.softplus = a->delta_softplus ? 1 : 0;
  p.state = a->state;
  p.y = a->y;
  const bool vec4 = a->dstate == 16 && aligned(a->state, 16);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  return a->dtype == SSM_BF16 ? run_step<__nv_bfloat16>(p, vec4, stream)
                              : run_step<float>(p, vec4, stream);
}

size_t ssm_scan_fwd_chunked_workspace_size(const ssm_ssd_args_t* args) {
  SsdParams p;
  size_t ws = 0;
  if (plan_ssd(args, &p, &ws, false) != SSM_OK) return static_cast<size_t>(-1);
  return ws;
}

ssm_status_t ssm_scan_fwd_chunked(const ssm_ssd_args_t* args, void* workspace,
                                  size_t workspace_bytes, ssm_stream_t stream_) {
  SsdParams p;
  size_t ws = 0;
  ssm_status_t st = plan_ssd(args, &p, &ws, true);
  if (st != SSM_OK) return st;
  if (p.batch == 0 || p.nheads == 0) return SSM_OK;
  if (workspace == nullptr || workspace_bytes < ws) return SSM_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return SSM_ERR_ALIGNMENT;
  unsigned char* w = static_cast<unsigned char*>(workspace);
  const size_t states = static_cast<size_t>(p.batch) * p.nheads * p.nchunks * ssd::kN * ssd::kP;
  const size_t cums = (static_cast<size_t>(p.batch) * p.nheads * p.nchunks * sizeof(float) + 255) /
                      256 * 256;
  p.status = reinterpret_cast<int*>(w);
  p.sloc = reinterpret_cast<float*>(w + kSsdStatusBytes);
  p.cum_end = reinterpret_cast<float*>(w + kSsdStatusBytes + states * sizeof(float));
  p.sprev = reinterpret_cast<__nv_bfloat16*>(w + kSsdStatusBytes + states * sizeof(float) + cums);
  p.dtc = reinterpret_cast<float*>(w + kSsdStatusBytes + states * sizeof(float) + cums +
                                   states * sizeof(__nv_bfloat16));
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  st = cuda_status(cudaMemsetAsync(p.status, 0, sizeof(int), stream), "ssd: status reset");
  if (st != SSM_OK) return st;
  SsdMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (p.nchunks > 0) {
    st = make_ssd_maps(p, &maps);
    if (st != SSM_OK) return st;
  }
  return p.chunk == 256 ? run_ssd<256>(p, maps, stream) : run_ssd<128>(p, maps, stream);
}

const char* ssm_status_string(ssm_status_t s) {
  switch (s) {
    case SSM_OK: return "ok";
    case SSM_ERR_INVALID_ARG: return "invalid argument";
    case SSM_ERR_UNSUPPORTED: return "unsupported size or option";
    case SSM_ERR_ALIGNMENT: return "misaligned pointer or stride";
    case SSM_ERR_CUDA: return "CUDA error";
    case SSM_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int ssm_version(void) { return 100; }

const char* ssm_last_error_string(void) { return g_last_error; }

}  // extern "C"

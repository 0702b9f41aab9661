// ssd_fwd.cuh -- the Mamba-2 scalar-decay (SSD) scan as a chunked scan on the
// sm_100a tensor cores.
//
// Page "Mamba状态空间模型的硬件感知推理优化", section 4: with a scalar decay
// a_t per step, h_t = a_t h_{t-1} + b_t x_t has the closed form
// h_t = cumprod_t h_0 + sum_k (cumprod_t / cumprod_k) b_k x_k; the same
// section's "parallel-serial hybrid" evaluates it in chunks: parallel inside
// a chunk, serial between chunks.  Section 6.2: the cumulative decay is taken
// in log space, exp(cumsum(log a)).  Per batch b and head h, with
// dt'_t = softplus(delta + bias_h) and cum_t = sum_{j <= t in chunk} dt'_j A_h:
//
//   intra-chunk:  Y_t = sum_{k <= t} (C_t . B_k) exp(cum_t - cum_k) dt'_k x_k
//   chunk state:  S_loc = sum_k exp(cum_end - cum_k) dt'_k x_k B_k^T     (P x N)
//   carried in:   Z_t = C_t S_prev^T,   y_t = Y_t + exp(cum_t) Z_t + D_h x_t
//   state pass:   S_next = exp(cum_end) S_prev + S_loc
//
// The dense contractions run as tcgen05 MMAs (bf16 operands in 128-byte-
// swizzled shared memory, fp32 accumulators in tensor memory).  Three kernels:
//  * ssd_chunk_state_kernel, one block per (b, chunk, head group): loads the B
//    chunk once, computes dt' and cum of every head of the group in one pass
//    (one warp-shuffle scan per head, one block barrier for all of them) and
//    stores them for the chunk scan, then per head stages x with cp.async, scales it in place by
//    exp(cum_end - cum_k) dt'_k and runs S_loc^T = B^T (scaled x); two tensor-
//    memory accumulators alternate so the next head's MMA overlaps the
//    previous read-out.  S_loc goes to the workspace ([p][n], fp32).
//  * ssd_pass_kernel, one thread per (b, h, p, n): walks the chunks in order,
//    writes the state entering each chunk (bf16: it is only used as an MMA
//    operand) and the final state.
//  * ssd_scan_kernel, one block per (b, chunk, head group), the chunk in row
//    blocks of 128 steps: G = C B^T once per group in tensor memory; per head
//    the stored dt' and cum arrive with the head's x and S_prev (cp.async, one
//    head ahead);
//    the causal decay mask times dt'_k is applied per row in registers into a
//    bf16 operand (blocks above the diagonal skipped; the block below it
//    factorised as exp(cum_t - cum_r) exp(cum_r - cum_k) with both factors
//    <= 1), then Y = M x and Z = C S_prev^T by MMA and the epilogue
//    y = Y + exp(cum_t) Z + D x (optional silu(z) gate).
#pragma once
#include <cuda.h>  // CUtensorMap

#include "common.cuh"
#include "tc.cuh"

namespace ssm {

struct SsdParams {
  int64_t batch, seqlen, nheads, headdim, dstate, chunk, nchunks;
  int64_t hgroup;  // heads per block in the chunk-state and scan kernels
  const __nv_bfloat16* x;
  const __nv_bfloat16* delta;
  const float* A;
  const __nv_bfloat16* B;
  const __nv_bfloat16* C;
  const float* D;
  const float* bias;
  int softplus;
  const __nv_bfloat16* z;
  const float* h0;
  __nv_bfloat16* y;
  float* h_last;
  float* sloc;           // (batch, nheads, nchunks, headdim, dstate) fp32: chunk-local states
  float* cum_end;        // (batch, nheads, nchunks): log decay over each chunk
  __nv_bfloat16* sprev;  // (batch, nheads, nchunks, headdim, dstate) bf16: state entering each chunk
  float* dtc;            // (batch, nheads, nchunks, 2, chunk) fp32: dt', then cum, of every step
  int* status;           // bit 0: a tensor-core completion wait timed out
};

// TMA descriptors of the operands (all bf16, 128-byte swizzle, 64-element
// boxes along the contiguous dimension, zero fill outside the tensor).
struct SsdMaps {
  CUtensorMap x;      // (headdim * nheads, seqlen, batch), box (64, chunk, 1)
  CUtensorMap B;      // (dstate, seqlen, batch), box (64, chunk, 1)
  CUtensorMap C;      // same as B
  CUtensorMap sprev;  // (dstate, batch * nheads * nchunks * headdim), box (64, 64)
};

namespace ssd {

constexpr int kThreads = 256;       // chunk-state kernel: 8 warps
// Chunk scan: 16 compute warps (warps w, w + 4, w + 8, w + 12 share TMEM
// lanes 32 (w % 4) .. + 31) and one producer warp whose first thread issues
// every TMA load and MMA, so no compute warp waits behind MMA issue.
constexpr int kScanCompute = 512;
constexpr int kScanThreads = kScanCompute + 32;
constexpr int kN = 128;   // dstate
constexpr int kP = 64;    // headdim
constexpr uint32_t kWaitPolls = 1u << 22;

// The head group's dt rows for one chunk: dl[t * kMaxGroup + j] = delta[b, t0 + t, hg0 + j].
constexpr int kMaxGroup = 24;
template <int Q>
__device__ __forceinline__ void stage_delta(const SsdParams& p, int64_t b, int64_t t0, int len,
                                            int64_t hg0, int nh, __nv_bfloat16* dl) {
  for (int i = threadIdx.x; i < Q * nh; i += kThreads) {
    const int t = i / nh, j = i % nh;
    dl[t * kMaxGroup + j] =
        t < len ? p.delta[(b * p.seqlen + t0 + t) * p.nheads + hg0 + j] : __float2bfloat16(0.f);
  }
}

// dt' and the in-chunk cumulative log decay cum of every head of the group,
// for every step of the chunk: dtp[j * Q + t], cum[j * Q + t] (steps past the
// end get dt' = 0, so they neither decay nor feed the state).  One step per
// thread; one warp-shuffle scan per head, then a single block barrier before
// the warp offsets are added.  wtot holds (kThreads / 32) x kMaxGroup floats.
template <int Q>
__device__ __forceinline__ void group_decays(const SsdParams& p, int64_t hg0, int nh, int len,
                                             const __nv_bfloat16* dl, float* dtp, float* cum,
                                             float* wtot) {
  static_assert(Q <= kThreads, "one step per thread");
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  for (int j = 0; j < nh; ++j) {
    float s = 0.f;
    if (t < len) {
      s = __bfloat162float(dl[t * kMaxGroup + j]) + (p.bias ? __ldg(p.bias + hg0 + j) : 0.f);
      if (p.softplus) s = softplus_f(s);
    }
    float a = s * __ldg(p.A + hg0 + j);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float n = __shfl_up_sync(0xffffffffu, a, o);
      if (lane >= o) a += n;
    }
    if (t < Q) {
      dtp[j * Q + t] = s;
      cum[j * Q + t] = a;
    }
    if (lane == 31) wtot[warp * kMaxGroup + j] = a;
  }
  __syncthreads();
  if (t < Q) {
    for (int j = 0; j < nh; ++j) {
      float off = 0.f;
      for (int w = 0; w < warp; ++w) off += wtot[w * kMaxGroup + j];
      cum[j * Q + t] += off;
    }
  }
  __syncthreads();
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// chunk-local states: one block per (b, chunk, head group)
// ---------------------------------------------------------------------------
template <int Q>
struct ChunkStateSmem {
  unsigned char bt[Q * kN * 2];      // B chunk: MN-major A operand of B^T (rows = time)
  unsigned char xw[2][Q * kP * 2];   // scaled x per head: MN-major B operand (rows = time)
  __nv_bfloat16 dl[Q * kMaxGroup];   // the group's delta rows
  float dtp[kMaxGroup * Q];          // dt' per (head of the group, step)
  float cum[kMaxGroup * Q];          // in-chunk cumulative log decay, same layout
  float wtot[(kThreads / 32) * kMaxGroup];
  uint64_t mbar[2];
  uint64_t lbar[3];  // TMA completion: B chunk, x buffer 0, x buffer 1
  uint32_t tmem;
};

template <int Q>
__global__ void __launch_bounds__(kThreads)
    ssd_chunk_state_kernel(const SsdParams p, const __grid_constant__ SsdMaps maps) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ChunkStateSmem<Q>& sm = *reinterpret_cast<ChunkStateSmem<Q>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t hg0 = static_cast<int64_t>(blockIdx.x) * p.hgroup;
  const int64_t c = blockIdx.y, b = blockIdx.z;
  const int64_t L = p.seqlen, H = p.nheads;
  const int nh = static_cast<int>(imin64(p.hgroup, H - hg0));
  const int64_t t0 = c * Q;
  const int len = static_cast<int>(imin64(Q, L - t0));

  // TMA loads: thread 0 issues them; issued[i] / waited[i] count the phases
  // of lbar[i] (only thread 0's counts are used, to drain copies still in
  // flight after a timed-out wait).
  uint32_t issued[3] = {0u, 0u, 0u}, waited[3] = {0u, 0u, 0u};
  bool ok = true;
  auto stage_x = [&](int hj) {  // thread 0
    uint64_t* bar = &sm.lbar[1 + (hj & 1)];
    tc::mbar_arrive_expect_tx(bar, Q * kP * 2);
    tc::tma_load_3d(sm.xw[hj & 1], &maps.x, static_cast<int32_t>((hg0 + hj) * kP),
                    static_cast<int32_t>(t0), static_cast<int32_t>(b), bar);
    ++issued[1 + (hj & 1)];
  };
  auto lwait = [&](int i) {
    if (ok && !tc::mbar_wait(&sm.lbar[i], waited[i] & 1u, kWaitPolls)) ok = false;
    if (ok) ++waited[i];
  };
  if (warp == 0) tc::tmem_alloc(&sm.tmem, 128);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar[0], 1);
    tc::mbar_init(&sm.mbar[1], 1);
    for (int i = 0; i < 3; ++i) tc::mbar_init(&sm.lbar[i], 1);
    tc::mbar_fence_init();
    tc::mbar_arrive_expect_tx(&sm.lbar[0], Q * kN * 2);
    for (int hf = 0; hf < kN / 64; ++hf)
      tc::tma_load_3d(sm.bt + hf * Q * 128, &maps.B, 64 * hf, static_cast<int32_t>(t0),
                      static_cast<int32_t>(b), &sm.lbar[0]);
    ++issued[0];
    stage_x(0);
  }
  stage_delta<Q>(p, b, t0, len, hg0, nh, sm.dl);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  group_decays<Q>(p, hg0, nh, len, sm.dl, sm.dtp, sm.cum, sm.wtot);
  // dt' and cum of every head, for the chunk scan; cum_end for the state pass
  for (int i = tid; i < nh * Q; i += kThreads) {
    const int j = i / Q, t = i % Q;
    float* dst = p.dtc + ((b * H + hg0 + j) * p.nchunks + c) * (2 * Q);
    dst[t] = sm.dtp[j * Q + t];
    dst[Q + t] = sm.cum[j * Q + t];
  }
  for (int j = tid; j < nh; j += kThreads)
    p.cum_end[(b * H + hg0 + j) * p.nchunks + c] = sm.cum[j * Q + Q - 1];
  const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
  uint32_t ph[2] = {0u, 0u};
  if (tid == 0) lwait(0);  // the B chunk, read only by the MMAs

  auto drain = [&](int hj) {  // read out head hj's accumulator, store S_loc [p][n]
    const int bj = hj & 1;
    if (ok && !tc::mbar_wait(&sm.mbar[bj], ph[bj], kWaitPolls)) ok = false;
    ph[bj] ^= 1;
    tc::fence_after_sync();
    // warp w: state rows n = 32 (w % 4) + lane, headdim columns 32 (w / 4) ..+31
    const int n = 32 * (warp & 3) + (tid & 31);
    const int pc = 32 * (warp >> 2);
    float* dst = p.sloc + (((b * H + hg0 + hj) * p.nchunks + c) * kP + pc) * kN + n;
    float v[32];
    tc::tmem_ld32(tmem + lane_off + 64 * bj + pc, v);
#pragma unroll
    for (int q = 0; q < 32; ++q) dst[q * kN] = v[q];
  };

  for (int hi = 0; hi < nh; ++hi) {
    const int bi = hi & 1;
    // Next head's x into the other buffer as soon as the MMA that last read it
    // (head hi - 1) has completed; drain(hi - 1) waits on the same phase later.
    if (tid == 0 && ok && hi + 1 < nh) {
      if (hi >= 1 && !tc::mbar_wait(&sm.mbar[bi ^ 1], ph[bi ^ 1], kWaitPolls)) ok = false;
      if (ok) stage_x(hi + 1);
    }
    const float* cumh = sm.cum + hi * Q;
    const float* dtph = sm.dtp + hi * Q;
    const float cend = cumh[Q - 1];
    lwait(1 + bi);  // x of this head has landed
    // scale x rows in place: w_t = exp(cum_end - cum_t) dt'_t
    for (int i = tid; i < Q * (kP / 8); i += kThreads) {
      const int t = i / (kP / 8);
      const int p8 = (i % (kP / 8)) * 8;
      uint4* ptr = reinterpret_cast<uint4*>(sm.xw[bi] + tc::sw128_offset(t, p8));
      const float w = ex2_approx((cend - cumh[t]) * kLog2e) * dtph[t];
      uint4 v = *ptr;
      uint32_t* vw = &v.x;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        vw[j] = pack_bf16(__uint_as_float(vw[j] << 16) * w, __uint_as_float(vw[j] & 0xffff0000u) * w);
      *ptr = v;
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0 && ok) {
      constexpr uint32_t idesc = tc::make_idesc_bf16(128, kP, 1, 1);
      const uint32_t a0 = tc::smem_u32(sm.bt), x0 = tc::smem_u32(sm.xw[bi]);
#pragma unroll 4
      for (int ks = 0; ks < Q / 16; ++ks)
        tc::mma_bf16(tmem + 64 * bi, tc::make_sdesc(a0 + ks * 2048, Q * 128, 1024),
                     tc::make_sdesc(x0 + ks * 2048, Q * 128, 1024), idesc, ks > 0);
      tc::mma_commit(&sm.mbar[bi]);
    }
    if (hi >= 1) drain(hi - 1);
  }
  if (nh > 0) drain(nh - 1);
  if (!ok && tid == 0) {
    atomicOr(p.status, 1);
    for (int i = 0; i < 3; ++i)  // copies still in flight land before the block exits
      for (; waited[i] < issued[i]; ++waited[i]) tc::mbar_wait(&sm.lbar[i], waited[i] & 1u, kWaitPolls);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------------------
// state pass: one thread per (b, h, p, n), sequential over chunks
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) ssd_pass_kernel(const SsdParams p) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int64_t per = static_cast<int64_t>(kP) * kN;
  if (idx >= p.batch * p.nheads * per) return;
  const int64_t bh = idx / per, e = idx % per;  // e = p * N + n
  float s = p.h0 ? p.h0[idx] : 0.f;             // h0 is (b, h, p, n): same order
  constexpr int kAhead = 8;                      // loads issued ahead of the dependent chain
  int64_t c = 0;
  for (; c + kAhead <= p.nchunks; c += kAhead) {
    float sl[kAhead], ce[kAhead];
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      sl[j] = p.sloc[(bh * p.nchunks + c + j) * per + e];
      ce[j] = p.cum_end[bh * p.nchunks + c + j];
    }
#pragma unroll
    for (int j = 0; j < kAhead; ++j) {
      p.sprev[(bh * p.nchunks + c + j) * per + e] = __float2bfloat16_rn(s);
      s = fmaf(ex2_approx(ce[j] * kLog2e), s, sl[j]);
    }
  }
  for (; c < p.nchunks; ++c) {
    const int64_t off = (bh * p.nchunks + c) * per + e;
    p.sprev[off] = __float2bfloat16_rn(s);
    s = fmaf(ex2_approx(p.cum_end[bh * p.nchunks + c] * kLog2e), s, p.sloc[off]);
  }
  if (p.h_last) p.h_last[idx] = s;
}

// ---------------------------------------------------------------------------
// chunk scan: one block per (b, chunk, head group)
// ---------------------------------------------------------------------------
template <int Q>
struct ScanSmem {
  unsigned char c[Q * kN * 2];    // C chunk: K-major A operand (rows = time)
  unsigned char bk[Q * kN * 2];   // B chunk: K-major B operand of G; then the odd heads' x / S_prev
  unsigned char x0[Q * kP * 2];   // even heads' x: MN-major B operand (rows = time)
  unsigned char sp0[kP * kN * 2]; // even heads' S_prev [p][n]: K-major B operand (rows = p)
  unsigned char m[128 * 128 * 2]; // masked decays, K-major A operand: two 64-key halves
  float dc[2][2 * Q];             // per head (two buffers): dt'[Q], then cum[Q]
  float vk[128];                  // exp(cum_r - cum_k) dt'_k below the diagonal block
  float hD[kMaxGroup];
  uint64_t mbar[2];
  uint64_t lbar[3];  // TMA completion: C and B chunks, head buffers 0 and 1
  uint32_t tmem;
};

template <int Q, bool HAS_Z>
__global__ void __launch_bounds__(kScanThreads, 1)
    ssd_scan_kernel(const SsdParams p, const __grid_constant__ SsdMaps maps) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ScanSmem<Q>& sm = *reinterpret_cast<ScanSmem<Q>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool producer = tid >= kScanCompute;      // the producer warp
  const bool issuer = tid == kScanCompute;        // its thread that issues TMA and MMA
  const int64_t hg0 = static_cast<int64_t>(blockIdx.x) * p.hgroup;
  const int64_t c = blockIdx.y, b = blockIdx.z;
  const int64_t L = p.seqlen, H = p.nheads;
  const int nh = static_cast<int>(imin64(p.hgroup, H - hg0));
  const int64_t t0 = c * Q;
  const int len = static_cast<int>(imin64(Q, L - t0));
  constexpr uint32_t kColG1 = 0;    // rows 128..255 against keys 0..255 (Q = 256)
  constexpr uint32_t kColG0 = Q == 256 ? 256 : 0;  // rows 0..127 against keys 0..127
  constexpr uint32_t kColY = 384, kColZ = 448;
  unsigned char* xbuf[2] = {sm.x0, sm.bk};
  unsigned char* spbuf[2] = {sm.sp0, sm.bk + Q * kP * 2};
  // TMA loads: the issuer thread issues them; issued[i] / waited[i] count the
  // phases of lbar[i] (its counts drain copies still in flight after a
  // timed-out wait).
  uint32_t issued[3] = {0u, 0u, 0u}, waited[3] = {0u, 0u, 0u};
  bool ok = true;
  auto stage_head = [&](int hj) {  // issuer: x, S_prev, dt' and cum of head hg0 + hj
    const int64_t h = hg0 + hj;
    uint64_t* bar = &sm.lbar[1 + (hj & 1)];
    tc::mbar_arrive_expect_tx(bar, Q * kP * 2 + kP * kN * 2 + 2 * Q * 4);
    tc::tma_load_3d(xbuf[hj & 1], &maps.x, static_cast<int32_t>(h * kP), static_cast<int32_t>(t0),
                    static_cast<int32_t>(b), bar);
    const int32_t row = static_cast<int32_t>(((b * H + h) * p.nchunks + c) * kP);
    for (int hf = 0; hf < kN / 64; ++hf)
      tc::tma_load_2d(spbuf[hj & 1] + hf * kP * 128, &maps.sprev, 64 * hf, row, bar);
    tc::bulk_load(sm.dc[hj & 1], p.dtc + ((b * H + h) * p.nchunks + c) * (2 * Q), 2 * Q * 4, bar);
    ++issued[1 + (hj & 1)];
  };
  auto lwait = [&](int i) {
    if (ok && !tc::mbar_wait(&sm.lbar[i], waited[i] & 1u, kWaitPolls)) ok = false;
    if (ok) ++waited[i];
  };

  if (warp == 0) tc::tmem_alloc(&sm.tmem, 512);
  if (issuer) {
    tc::mbar_init(&sm.mbar[0], 1);
    tc::mbar_init(&sm.mbar[1], 1);
    for (int i = 0; i < 3; ++i) tc::mbar_init(&sm.lbar[i], 1);
    tc::mbar_fence_init();
    tc::mbar_arrive_expect_tx(&sm.lbar[0], 2 * Q * kN * 2);
    for (int hf = 0; hf < kN / 64; ++hf) {
      tc::tma_load_3d(sm.c + hf * Q * 128, &maps.C, 64 * hf, static_cast<int32_t>(t0),
                      static_cast<int32_t>(b), &sm.lbar[0]);
      tc::tma_load_3d(sm.bk + hf * Q * 128, &maps.B, 64 * hf, static_cast<int32_t>(t0),
                      static_cast<int32_t>(b), &sm.lbar[0]);
    }
    ++issued[0];
    stage_head(0);
  }
  for (int j = tid; j < nh; j += kScanThreads) sm.hD[j] = p.D ? p.D[hg0 + j] : 0.f;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  const int quarter = warp & 3;         // TMEM lanes 32 quarter ..+31 = rows of the row block
  const int cq = warp >> 2;             // which 16 of each 64 columns this warp handles
  const int rl = 32 * quarter + (tid & 31);  // this thread's row within the row block
  const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
  uint32_t ph[2] = {0u, 0u};
  auto wait_bar = [&](int i) {
    if (ok && !tc::mbar_wait(&sm.mbar[i], ph[i], kWaitPolls)) ok = false;
    ph[i] ^= 1;
    tc::fence_after_sync();
  };

  // G = C B^T for the chunk, shared by every head of the group.
  if (issuer) lwait(0);  // C and B chunks landed (read only by the MMAs)
  if (issuer && ok) {
    const uint32_t ca = tc::smem_u32(sm.c), bb = tc::smem_u32(sm.bk);
#pragma unroll
    for (int ks = 0; ks < kN / 16; ++ks) {
      const uint32_t ko = (ks / 4) * (Q * 128) + (ks % 4) * 32;
      tc::mma_bf16(tmem + kColG0, tc::make_sdesc(ca + ko, 16, 1024), tc::make_sdesc(bb + ko, 16, 1024),
                   tc::make_idesc_bf16(128, 128, 0, 0), ks > 0);
      if (Q == 256)
        tc::mma_bf16(tmem + kColG1, tc::make_sdesc(ca + 128 * 128 + ko, 16, 1024),
                     tc::make_sdesc(bb + ko, 16, 1024), tc::make_idesc_bf16(128, 256, 0, 0), ks > 0);
    }
    tc::mma_commit(&sm.mbar[0]);
  }
  wait_bar(0);  // the B chunk's region is free from here on (the producer warp
                // waits on no MMA after this one: the barriers order it)

  for (int hi = 0; hi < nh; ++hi) {
    const int64_t h = hg0 + hi;
    const int bi = hi & 1;
    // into the other buffers: their last readers finished before the barrier
    // that ended the previous head
    if (issuer && ok && hi + 1 < nh) stage_head(hi + 1);
    lwait(1 + bi);  // this head's operands landed
    const float* dtph = sm.dc[bi];
    const float* cumh = sm.dc[bi] + Q;
    // Factor below the diagonal block (reference step r = 127).  Row block 1
    // reads it only after row block 0's barriers.
    if (Q == 256) {
      const float cr = cumh[127];
      for (int k = tid; k < 128; k += kScanThreads)
        sm.vk[k] = ex2_approx((cr - cumh[k]) * kLog2e) * dtph[k];
    }
    const uint32_t xb = tc::smem_u32(xbuf[bi]);
    const uint32_t spb = tc::smem_u32(spbuf[bi]);
    const float Dh = sm.hD[hi];

    for (int i = 0; i < Q / 128; ++i) {
      const int tr = 128 * i + rl;  // this thread's row (step) in the chunk
      const float cum_t = cumh[tr];
      const uint32_t gcol = i == 0 ? kColG0 : kColG1;
      // Z_i = C_i S_prev^T (K = states)
      if (issuer && ok) {
        const uint32_t ca = tc::smem_u32(sm.c) + i * 128 * 128;
        for (int ks = 0; ks < kN / 16; ++ks) {
          tc::mma_bf16(tmem + kColZ, tc::make_sdesc(ca + (ks / 4) * (Q * 128) + (ks % 4) * 32, 16, 1024),
                       tc::make_sdesc(spb + (ks / 4) * (kP * 128) + (ks % 4) * 32, 16, 1024),
                       tc::make_idesc_bf16(128, kP, 0, 0), ks > 0);
        }
      }
      // Y_i = sum over key blocks of (masked decays) x, 64 keys per step.  Each
      // warp handles 16 keys of a block; the next block's G slab is loaded from
      // tensor memory while the current one is turned into decays.
      const int nkb = 2 * (i + 1);  // 64-key blocks reaching this row block
      auto slab_active = [&](int kb) {  // warp-uniform: skip slabs above the diagonal
        return kb < 2 * i || (64 * kb + 16 * cq - 128 * i) <= 32 * quarter + 31;
      };
      uint32_t gA[16], gB[16];  // double buffer of G slabs (named, so they stay in registers)
      if (!producer && slab_active(0)) tc::tmem_ld16_issue(tmem + lane_off + gcol + 16 * cq, gA);
      auto key_block = [&](int kb, const uint32_t (&cur_raw)[16], uint32_t (&next_raw)[16]) {
        const int mb = kb & 1;  // shared-memory half of m used by this key block
        const int kbase = 64 * kb;
        if (!producer) {
        const bool active = slab_active(kb);
        tc::tmem_wait();
        uint32_t cur[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) cur[j] = cur_raw[j];
        if (kb + 1 < nkb && slab_active(kb + 1))
          tc::tmem_ld16_issue(tmem + lane_off + gcol + 64 * (kb + 1) + 16 * cq, next_raw);
        if (kb >= 2) wait_bar(mb);  // the MMA that read this half two steps ago is done
        const bool below = i == 1 && kb < 2;          // keys 0..127 of rows 128..255
        const int cb = 16 * cq;
        const int k0 = kbase + cb;
        uint32_t packed[8];
        if (active) {
          if (below) {
            const float urow = ex2_approx((cum_t - cumh[127]) * kLog2e);
            float vv[16];
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<float4*>(&vv[j]) = *reinterpret_cast<const float4*>(&sm.vk[k0 + j]);
#pragma unroll
            for (int j = 0; j < 16; j += 2)
              packed[j / 2] = pack_bf16(__uint_as_float(cur[j]) * urow * vv[j],
                                        __uint_as_float(cur[j + 1]) * urow * vv[j + 1]);
          } else {
            float ck[16], dk[16];
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              *reinterpret_cast<float4*>(&ck[j]) = *reinterpret_cast<const float4*>(&cumh[k0 + j]);
              *reinterpret_cast<float4*>(&dk[j]) = *reinterpret_cast<const float4*>(&dtph[k0 + j]);
            }
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const int k = k0 + j;
              const float e0 = k <= tr ? ex2_approx((cum_t - ck[j]) * kLog2e) * dk[j] * __uint_as_float(cur[j]) : 0.f;
              const float e1 = k + 1 <= tr ? ex2_approx((cum_t - ck[j + 1]) * kLog2e) * dk[j + 1] * __uint_as_float(cur[j + 1]) : 0.f;
              packed[j / 2] = pack_bf16(e0, e1);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) packed[j] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          *reinterpret_cast<uint4*>(sm.m + mb * (128 * 128) + tc::sw128_offset(rl, cb + 8 * q)) =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
        tc::fence_proxy_async_smem();
        }
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (issuer && ok) {
          const uint32_t ma = tc::smem_u32(sm.m) + mb * (128 * 128);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            tc::mma_bf16(tmem + kColY, tc::make_sdesc(ma + ks * 32, 16, 1024),
                         tc::make_sdesc(xb + (kbase + 16 * ks) * 128, Q * 128, 1024),
                         tc::make_idesc_bf16(128, kP, 0, 1), kb > 0 || ks > 0);
          tc::mma_commit(&sm.mbar[mb]);
        }
      };
#pragma unroll 1
      for (int kb = 0; kb < nkb; kb += 2) {  // nkb is even
        key_block(kb, gA, gB);
        key_block(kb + 1, gB, gA);
      }
      // both halves' last MMAs (this row block's Y and Z) complete
      if (!producer) {
        wait_bar(0);
        wait_bar(1);
      }

      // epilogue: y = Y + exp(cum_t) Z + D x (then the gate), row tr.  The
      // tensor-memory loads are warp-collective: every lane runs them.
      const bool row_ok = tr < len;
      const float ec = ex2_approx(cum_t * kLog2e);
      const int64_t row = ((b * L + t0 + (row_ok ? tr : 0)) * H + h) * kP;
      if (!producer) {
        const int cb = 16 * cq;
        uint32_t yr[16], zr16[16];
        tc::tmem_ld16_issue(tmem + lane_off + kColY + cb, yr);
        tc::tmem_ld16_issue(tmem + lane_off + kColZ + cb, zr16);
        tc::tmem_wait();
        if (row_ok) {
#pragma unroll
          for (int q = 0; q < 16; q += 8) {
            const uint4 xr = *reinterpret_cast<const uint4*>(xbuf[bi] + tc::sw128_offset(tr, cb + q));
            const uint32_t* xw = &xr.x;
            uint4 zr = make_uint4(0, 0, 0, 0);
            if (HAS_Z) zr = *reinterpret_cast<const uint4*>(p.z + row + cb + q);
            const uint32_t* zw = &zr.x;
            uint4 o;
            uint32_t* ow = &o.x;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float v0 = __uint_as_float(yr[q + 2 * j]) + ec * __uint_as_float(zr16[q + 2 * j]) +
                         Dh * __uint_as_float(xw[j] << 16);
              float v1 = __uint_as_float(yr[q + 2 * j + 1]) + ec * __uint_as_float(zr16[q + 2 * j + 1]) +
                         Dh * __uint_as_float(xw[j] & 0xffff0000u);
              if (HAS_Z) {
                v0 *= silu_f(__uint_as_float(zw[j] << 16));
                v1 *= silu_f(__uint_as_float(zw[j] & 0xffff0000u));
              }
              ow[j] = pack_bf16(v0, v1);
            }
            *reinterpret_cast<uint4*>(p.y + row + cb + q) = o;
          }
        }
      }
      tc::fence_before_sync();
      __syncthreads();  // Y / Z / m are rewritten by the next row block or head
      tc::fence_after_sync();
    }
  }
  if (!ok) atomicOr(p.status, 1);
  if (!ok && issuer) {
    for (int i = 0; i < 3; ++i)  // copies still in flight land before the block exits
      for (; waited[i] < issued[i]; ++waited[i]) tc::mbar_wait(&sm.lbar[i], waited[i] & 1u, kWaitPolls);
  }
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace ssd
}  // namespace ssm

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
//    chunk once, then per head stages x with cp.async, scales it in place by
//    exp(cum_end - cum_k) dt'_k and runs S_loc^T = B^T (scaled x); two tensor-
//    memory accumulators alternate so the next head's MMA overlaps the
//    previous read-out.  S_loc goes to the workspace ([p][n], fp32).
//  * ssd_pass_kernel, one thread per (b, h, p, n): walks the chunks in order,
//    writes the state entering each chunk (bf16: it is only used as an MMA
//    operand) and the final state.
//  * ssd_scan_kernel, one block per (b, chunk, head group), the chunk in row
//    blocks of 128 steps: G = C B^T once per group in tensor memory; per head
//    the causal decay mask times dt'_k is applied per row in registers into a
//    bf16 operand (blocks above the diagonal skipped; the block below it
//    factorised as exp(cum_t - cum_r) exp(cum_r - cum_k) with both factors
//    <= 1), then Y = M x and Z = C S_prev^T by MMA and the epilogue
//    y = Y + exp(cum_t) Z + D x (optional silu(z) gate).
#pragma once
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
  int* status;           // bit 0: a tensor-core completion wait timed out
};

namespace ssd {

constexpr int kThreads = 256;  // 8 warps: warps w and w + 4 share TMEM lanes 32 (w % 4)..+31
constexpr int kN = 128;   // dstate
constexpr int kP = 64;    // headdim
constexpr uint32_t kWaitPolls = 1u << 22;

// Block-wide inclusive prefix sum over Q values v[t] in shared memory
// (ceil(Q / kThreads) consecutive values per thread).
template <int Q>
__device__ __forceinline__ void block_cumsum(float* v, float* warp_tot) {
  constexpr int kPer = (Q + kThreads - 1) / kThreads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float loc[kPer];
  float run = 0.f;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int t = tid * kPer + j;
    run += t < Q ? v[t] : 0.f;
    loc[j] = run;
  }
  float incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  float off = incl - run;
  for (int w = 0; w < warp; ++w) off += warp_tot[w];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int t = tid * kPer + j;
    if (t < Q) v[t] = loc[j] + off;
  }
  __syncthreads();
}

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

// dt' and cum for head hg0 + j of the chunk (steps past the end get dt' = 0,
// so they neither decay nor feed the state).
template <int Q>
__device__ __forceinline__ void chunk_decays(const SsdParams& p, float Ah, float bias, int j,
                                             int len, const __nv_bfloat16* dl, float* dtp,
                                             float* cum, float* wtot) {
  for (int i = threadIdx.x; i < Q; i += kThreads) {
    float s = 0.f;
    if (i < len) {
      s = __bfloat162float(dl[i * kMaxGroup + j]) + bias;
      if (p.softplus) s = softplus_f(s);
    }
    dtp[i] = s;
    cum[i] = s * Ah;
  }
  __syncthreads();
  block_cumsum<Q>(cum, wtot);
}

// cp.async copy of a (rows x cols) bf16 tile, rows `ld` elements apart in
// global memory, into 64-column blocks of 128-byte swizzled rows (block
// stride rows * 128 bytes).  Rows >= valid are zero-filled.
__device__ __forceinline__ void stage_tile(unsigned char* dst, const __nv_bfloat16* src, int64_t ld,
                                           int rows, int valid, int cols) {
  const int per_row = cols / 8;
  for (int i = threadIdx.x; i < rows * per_row; i += kThreads) {
    const int r = i / per_row;
    const int c8 = (i % per_row) * 8;
    unsigned char* d = dst + (c8 / 64) * (rows * 128) + tc::sw128_offset(r, c8 % 64);
    const bool ok = r < valid;
    cp_async16(d, ok ? src + r * ld + c8 : src, ok ? 16 : 0);
  }
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
  float cum[Q];
  float dtp[Q];
  float wtot[kThreads / 32];
  uint64_t mbar[2];
  uint32_t tmem;
};

template <int Q>
__global__ void __launch_bounds__(kThreads) ssd_chunk_state_kernel(const SsdParams p) {
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

  if (warp == 0) tc::tmem_alloc(&sm.tmem, 128);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar[0], 1);
    tc::mbar_init(&sm.mbar[1], 1);
    tc::mbar_fence_init();
  }
  stage_tile(sm.bt, p.B + (b * L + t0) * kN, kN, Q, len, kN);
  stage_tile(sm.xw[0], p.x + ((b * L + t0) * H + hg0) * kP, H * kP, Q, len, kP);
  cp_async_commit();
  stage_delta<Q>(p, b, t0, len, hg0, nh, sm.dl);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
  uint32_t ph[2] = {0u, 0u};
  bool ok = true;

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
    const int64_t h = hg0 + hi;
    const int bi = hi & 1;
    chunk_decays<Q>(p, p.A[h], p.bias ? p.bias[h] : 0.f, hi, len, sm.dl, sm.dtp, sm.cum, sm.wtot);
    const float cend = sm.cum[Q - 1];
    if (tid == 0) p.cum_end[(b * H + h) * p.nchunks + c] = cend;
    cp_async_wait_all();  // x of this head (and, the first time, B) has landed
    __syncthreads();
    // scale x rows in place: w_t = exp(cum_end - cum_t) dt'_t
    for (int i = tid; i < Q * (kP / 8); i += kThreads) {
      const int t = i / (kP / 8);
      const int p8 = (i % (kP / 8)) * 8;
      uint4* ptr = reinterpret_cast<uint4*>(sm.xw[bi] + tc::sw128_offset(t, p8));
      const float w = ex2_approx((cend - sm.cum[t]) * kLog2e) * sm.dtp[t];
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
    if (hi >= 1) drain(hi - 1);  // frees xw[bi ^ 1]
    if (hi + 1 < nh) {
      stage_tile(sm.xw[bi ^ 1], p.x + ((b * L + t0) * H + h + 1) * kP, H * kP, Q, len, kP);
      cp_async_commit();
    }
  }
  if (nh > 0) drain(nh - 1);
  if (!ok && tid == 0) atomicOr(p.status, 1);
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
  constexpr int kAhead = 4;                      // loads issued ahead of the dependent chain
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
  float cum[Q];
  float dtp[Q];
  float vk[128];                  // exp(cum_r - cum_k) dt'_k below the diagonal block
  __nv_bfloat16 dl[Q * kMaxGroup]; // the group's delta rows
  float hA[kMaxGroup], hbias[kMaxGroup], hD[kMaxGroup];
  float wtot[kThreads / 32];
  uint64_t mbar[2];
  uint32_t tmem;
};

template <int Q, bool HAS_Z>
__global__ void __launch_bounds__(kThreads) ssd_scan_kernel(const SsdParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ScanSmem<Q>& sm = *reinterpret_cast<ScanSmem<Q>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
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
  auto stage_head = [&](int hj) {
    const int64_t h = hg0 + hj;
    stage_tile(xbuf[hj & 1], p.x + ((b * L + t0) * H + h) * kP, H * kP, Q, len, kP);
    stage_tile(spbuf[hj & 1], p.sprev + ((b * H + h) * p.nchunks + c) * kP * kN, kN, kP, kP, kN);
    cp_async_commit();
  };

  if (warp == 0) tc::tmem_alloc(&sm.tmem, 512);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar[0], 1);
    tc::mbar_init(&sm.mbar[1], 1);
    tc::mbar_fence_init();
  }
  stage_tile(sm.c, p.C + (b * L + t0) * kN, kN, Q, len, kN);
  stage_tile(sm.bk, p.B + (b * L + t0) * kN, kN, Q, len, kN);
  cp_async_commit();
  stage_head(0);
  stage_delta<Q>(p, b, t0, len, hg0, nh, sm.dl);
  for (int j = tid; j < nh; j += kThreads) {
    sm.hA[j] = p.A[hg0 + j];
    sm.hbias[j] = p.bias ? p.bias[hg0 + j] : 0.f;
    sm.hD[j] = p.D ? p.D[hg0 + j] : 0.f;
  }
  cp_async_wait_all();
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  const int quarter = warp & 3;         // TMEM lanes 32 quarter ..+31 = rows of the row block
  const int chalf = warp >> 2;          // which 32 of each 64 columns this warp handles
  const int rl = 32 * quarter + (tid & 31);  // this thread's row within the row block
  const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
  uint32_t ph[2] = {0u, 0u};
  bool ok = true;
  auto wait_bar = [&](int i) {
    if (ok && !tc::mbar_wait(&sm.mbar[i], ph[i], kWaitPolls)) ok = false;
    ph[i] ^= 1;
    tc::fence_after_sync();
  };

  // G = C B^T for the chunk, shared by every head of the group.
  if (tid == 0) {
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
  wait_bar(0);  // the B chunk's region is free from here on

  for (int hi = 0; hi < nh; ++hi) {
    const int64_t h = hg0 + hi;
    const int bi = hi & 1;
    if (hi + 1 < nh) stage_head(hi + 1);  // into the other buffers (their last use has completed)
    chunk_decays<Q>(p, sm.hA[hi], sm.hbias[hi], hi, len, sm.dl, sm.dtp, sm.cum, sm.wtot);
    if (Q == 256) {  // factor below the diagonal block: reference step r = 127
      const float cr = sm.cum[127];
      for (int k = tid; k < 128; k += kThreads)
        sm.vk[k] = ex2_approx((cr - sm.cum[k]) * kLog2e) * sm.dtp[k];
    }
    if (hi + 1 < nh) {
      asm volatile("cp.async.wait_group 1;\n" ::: "memory");  // this head's x / S_prev landed
    } else {
      cp_async_wait_all();
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    const uint32_t xb = tc::smem_u32(xbuf[bi]);
    const uint32_t spb = tc::smem_u32(spbuf[bi]);
    const float Dh = sm.hD[hi];

    for (int i = 0; i < Q / 128; ++i) {
      const int tr = 128 * i + rl;  // this thread's row (step) in the chunk
      const float cum_t = sm.cum[tr];
      const uint32_t gcol = i == 0 ? kColG0 : kColG1;
      // Z_i = C_i S_prev^T (K = states)
      if (tid == 0 && ok) {
        const uint32_t ca = tc::smem_u32(sm.c) + i * 128 * 128;
        for (int ks = 0; ks < kN / 16; ++ks) {
          tc::mma_bf16(tmem + kColZ, tc::make_sdesc(ca + (ks / 4) * (Q * 128) + (ks % 4) * 32, 16, 1024),
                       tc::make_sdesc(spb + (ks / 4) * (kP * 128) + (ks % 4) * 32, 16, 1024),
                       tc::make_idesc_bf16(128, kP, 0, 0), ks > 0);
        }
      }
      // Y_i = sum over key blocks of (masked decays) x, 64 keys per step.  Each
      // warp handles 32 keys of a block; the next block's G slab is loaded from
      // tensor memory while the current one is turned into decays.
      const int nkb = 2 * (i + 1);  // 64-key blocks reaching this row block
      auto slab_active = [&](int kb) {  // warp-uniform: skip slabs above the diagonal
        return kb < 2 * i || (64 * kb + 32 * chalf - 128 * i) <= 32 * quarter + 31;
      };
      uint32_t gA[32], gB[32];  // double buffer of G slabs (named, so they stay in registers)
      if (slab_active(0)) tc::tmem_ld32_issue(tmem + lane_off + gcol + 32 * chalf, gA);
      auto key_block = [&](int kb, const uint32_t (&cur_raw)[32], uint32_t (&next_raw)[32]) {
        const int mb = kb & 1;  // shared-memory half of m used by this key block
        const bool active = slab_active(kb);
        tc::tmem_wait();
        uint32_t cur[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) cur[j] = cur_raw[j];
        if (kb + 1 < nkb && slab_active(kb + 1))
          tc::tmem_ld32_issue(tmem + lane_off + gcol + 64 * (kb + 1) + 32 * chalf, next_raw);
        if (kb >= 2) wait_bar(mb);  // the MMA that read this half two steps ago is done
        const bool below = i == 1 && kb < 2;          // keys 0..127 of rows 128..255
        const int kbase = 64 * kb;
        const int cb = 32 * chalf;
        const int k0 = kbase + cb;
        uint32_t packed[16];
        if (active) {
          if (below) {
            const float urow = ex2_approx((cum_t - sm.cum[127]) * kLog2e);
            float vv[32];
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(&vv[j]) = *reinterpret_cast<const float4*>(&sm.vk[k0 + j]);
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              packed[j / 2] = pack_bf16(__uint_as_float(cur[j]) * urow * vv[j],
                                        __uint_as_float(cur[j + 1]) * urow * vv[j + 1]);
          } else {
            float ck[32], dk[32];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              *reinterpret_cast<float4*>(&ck[j]) = *reinterpret_cast<const float4*>(&sm.cum[k0 + j]);
              *reinterpret_cast<float4*>(&dk[j]) = *reinterpret_cast<const float4*>(&sm.dtp[k0 + j]);
            }
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const int k = k0 + j;
              const float e0 = k <= tr ? ex2_approx((cum_t - ck[j]) * kLog2e) * dk[j] * __uint_as_float(cur[j]) : 0.f;
              const float e1 = k + 1 <= tr ? ex2_approx((cum_t - ck[j + 1]) * kLog2e) * dk[j + 1] * __uint_as_float(cur[j + 1]) : 0.f;
              packed[j / 2] = pack_bf16(e0, e1);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) packed[j] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          *reinterpret_cast<uint4*>(sm.m + mb * (128 * 128) + tc::sw128_offset(rl, cb + 8 * q)) =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (tid == 0 && ok) {
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
      wait_bar(0);
      wait_bar(1);

      // epilogue: y = Y + exp(cum_t) Z + D x (then the gate), row tr.  The
      // tensor-memory loads are warp-collective: every lane runs them.
      const bool row_ok = tr < len;
      const float ec = ex2_approx(cum_t * kLog2e);
      const int64_t row = ((b * L + t0 + (row_ok ? tr : 0)) * H + h) * kP;
      {
        const int cb = 32 * chalf;
        uint32_t yr[32], zr32[32];
        tc::tmem_ld32_issue(tmem + lane_off + kColY + cb, yr);
        tc::tmem_ld32_issue(tmem + lane_off + kColZ + cb, zr32);
        tc::tmem_wait();
        float yv[32], zv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          yv[j] = __uint_as_float(yr[j]);
          zv[j] = __uint_as_float(zr32[j]);
        }
        if (row_ok) {
#pragma unroll
        for (int q = 0; q < 32; q += 8) {
          const uint4 xr = *reinterpret_cast<const uint4*>(xbuf[bi] + tc::sw128_offset(tr, cb + q));
          const uint32_t* xw = &xr.x;
          uint4 zr = make_uint4(0, 0, 0, 0);
          if (HAS_Z) zr = *reinterpret_cast<const uint4*>(p.z + row + cb + q);
          const uint32_t* zw = &zr.x;
          uint4 o;
          uint32_t* ow = &o.x;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float v0 = yv[q + 2 * j] + ec * zv[q + 2 * j] + Dh * __uint_as_float(xw[j] << 16);
            float v1 = yv[q + 2 * j + 1] + ec * zv[q + 2 * j + 1] + Dh * __uint_as_float(xw[j] & 0xffff0000u);
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
  if (!ok && tid == 0) atomicOr(p.status, 1);
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace ssd
}  // namespace ssm

// ssd_fwd.cuh -- the Mamba-2 scalar-decay (SSD) scan as a chunked scan on the
// sm_100a tensor cores.
//
// Page "Mamba状态空间模型的硬件感知推理优化", section 4: with a scalar decay
// a_t per step, h_t = a_t h_{t-1} + b_t x_t has the closed form
// h_t = cumprod_t h_0 + sum_k (cumprod_t / cumprod_k) b_k x_k; the same
// section's "parallel-serial hybrid" evaluates it in chunks: parallel
// inside a chunk, serial between chunks.  Section 6.2: the cumulative decay
// is taken in log space, exp(cumsum(log a)).  Per batch b and head h, with
// dt'_t = softplus(delta + bias_h), cum_t = sum_{j <= t in chunk} dt'_j A_h
// and X'_t = dt'_t x_t (a headdim-vector):
//
//   intra-chunk:  Y_t = sum_{k <= t} (C_t . B_k) exp(cum_t - cum_k) X'_k
//   chunk state:  S_loc = sum_k exp(cum_end - cum_k) X'_k B_k^T      (P x N)
//   carried in:   Z_t = C_t S_prev^T,   y_t = Y_t + exp(cum_t) Z_t + D_h x_t
//   state pass:   S_next = exp(cum_end) S_prev + S_loc
//
// The dense contractions (C B^T, the masked product with X', B^T X', C S^T)
// run as tcgen05 MMAs (bf16 operands in 128-byte-swizzled shared memory,
// fp32 accumulators in tensor memory).  Two kernels:
//  * ssd_state_kernel, one block per (b, h): walks the chunks in order, one
//    MMA per chunk for S_loc^T = B^T (w o X') with w_k = exp(cum_end - cum_k);
//    the running state stays in registers (one state row per thread); the
//    state entering each chunk goes to the workspace in bf16 (it is only
//    ever used as an MMA operand), the final state to h_last in fp32.
//  * ssd_scan_kernel, one block per (b, chunk, h), the chunk in row blocks
//    of 128 steps: G = C_i B^T in tensor memory, the causal decay mask
//    applied per row in registers into a bf16 operand, Y = M X' and
//    Z = C_i S_prev^T by MMA, and the epilogue y = Y + exp(cum_t) Z + D x
//    (optional silu(z) gate).
#pragma once
#include "common.cuh"
#include "tc.cuh"

namespace ssm {

struct SsdParams {
  int64_t batch, seqlen, nheads, headdim, dstate, chunk, nchunks;
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
  __nv_bfloat16* sprev;  // (batch, nheads, nchunks, dstate, headdim) bf16: state entering each chunk
  int* status;           // bit 0: an MMA completion wait timed out
};

namespace ssd {

constexpr int kThreads = 128;
constexpr int kN = 128;   // dstate
constexpr int kP = 64;    // headdim
constexpr uint32_t kWaitPolls = 1u << 22;

// softplus for one value (same ranges as softplus_f).
__device__ __forceinline__ float step_size(float s, int softplus) {
  return softplus ? softplus_f(s) : s;
}

// Block-wide inclusive prefix sum over Q values held in v[t] (shared memory),
// Q / kThreads consecutive values per thread.  `warp_tot` holds kThreads / 32
// floats of scratch.
template <int Q>
__device__ __forceinline__ void block_cumsum(float* v, float* warp_tot) {
  constexpr int kPer = Q / kThreads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float loc[kPer];
  float run = 0.f;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    run += v[tid * kPer + j];
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
  for (int j = 0; j < kPer; ++j) v[tid * kPer + j] = loc[j] + off;
  __syncthreads();
}

// Copies a (rows x 128) bf16 tile whose rows are `ld` elements apart in global
// memory into shared memory as blocks of 64 columns with 128-byte rows
// (swizzled; block stride rows * 128 bytes).  Rows >= valid_rows are zero.
__device__ __forceinline__ void load_tile_128(unsigned char* dst, const __nv_bfloat16* src,
                                              int64_t ld, int rows, int valid_rows, int cols) {
  const int chunks = rows * (cols / 8);
  for (int i = threadIdx.x; i < chunks; i += kThreads) {
    const int r = i / (cols / 8);
    const int c8 = (i % (cols / 8)) * 8;
    unsigned char* d = dst + (c8 / 64) * (rows * 128) + tc::sw128_offset(r, c8 % 64);
    const bool ok = r < valid_rows;
    cp_async16(d, ok ? src + r * ld + c8 : src, ok ? 16 : 0);
  }
}

// ---------------------------------------------------------------------------
// chunk states and the state pass: one block per (b, h)
// ---------------------------------------------------------------------------
template <int Q>
struct StateSmem {
  unsigned char bt[Q * kN * 2];  // B chunk: MMA A operand (B^T, MN-major), 2 blocks of 64 states
  unsigned char xw[Q * kP * 2];  // (w o X'): MMA B operand (MN-major)
  float cum[Q];
  float dtp[Q];
  float wtot[kThreads / 32];
  uint64_t mbar;
  uint32_t tmem;
};

template <int Q>
__global__ void __launch_bounds__(kThreads) ssd_state_kernel(const SsdParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  StateSmem<Q>& sm = *reinterpret_cast<StateSmem<Q>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t b = blockIdx.x / p.nheads, h = blockIdx.x % p.nheads;
  const int64_t L = p.seqlen, H = p.nheads;
  const float Ah = p.A[h];
  const float biash = p.bias ? p.bias[h] : 0.f;

  if (warp == 0) tc::tmem_alloc(&sm.tmem, 64);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar, 1);
    tc::mbar_fence_init();
  }
  // running state: this thread owns state row n = tid, S[n][0..63]
  float S[kP];
  const int n = tid;
#pragma unroll
  for (int q = 0; q < kP; ++q)
    S[q] = p.h0 ? p.h0[((b * H + h) * kP + q) * kN + n] : 0.f;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  bool ok = true;

  for (int64_t c = 0; c < p.nchunks; ++c) {
    const int64_t t0 = c * Q;
    const int len = static_cast<int>(imin64(Q, L - t0));
    // B chunk (rows = time, 128 states) -> MN-major A operand of B^T
    load_tile_128(sm.bt, p.B + (b * L + t0) * kN, kN, Q, len, kN);
    cp_async_commit();
    // dt' and the log-decay prefix sums
    for (int i = tid; i < Q; i += kThreads) {
      const float s = i < len ? step_size(__bfloat162float(p.delta[(b * L + t0 + i) * H + h]) + biash,
                                          p.softplus)
                              : 0.f;
      sm.dtp[i] = s;
      sm.cum[i] = s * Ah;
    }
    __syncthreads();
    block_cumsum<Q>(sm.cum, sm.wtot);
    const float cum_end = sm.cum[Q - 1];
    // (w o X')_t = exp(cum_end - cum_t) dt'_t x_t, bf16, MN-major (rows = time)
    for (int i = tid; i < Q * (kP / 8); i += kThreads) {
      const int t = i / (kP / 8);
      const int p8 = (i % (kP / 8)) * 8;
      uint4 out = make_uint4(0, 0, 0, 0);
      if (t < len) {
        const float w = ex2_approx((cum_end - sm.cum[t]) * kLog2e) * sm.dtp[t];
        const uint4 raw = *reinterpret_cast<const uint4*>(p.x + ((b * L + t0 + t) * H + h) * kP + p8);
        const uint32_t* rw = &raw.x;
        uint32_t* ow = &out.x;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float lo = __uint_as_float(rw[j] << 16) * w;
          const float hi = __uint_as_float(rw[j] & 0xffff0000u) * w;
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(lo, hi);
          ow[j] = *reinterpret_cast<const uint32_t*>(&v2);
        }
      }
      *reinterpret_cast<uint4*>(sm.xw + tc::sw128_offset(t, p8)) = out;
    }
    cp_async_wait_all();
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0 && ok) {
      constexpr uint32_t idesc = tc::make_idesc_bf16(128, kP, 1, 1);
      const uint32_t a0 = tc::smem_u32(sm.bt), b0 = tc::smem_u32(sm.xw);
#pragma unroll 4
      for (int ks = 0; ks < Q / 16; ++ks) {
        tc::mma_bf16(tmem, tc::make_sdesc(a0 + ks * 2048, Q * 128, 1024),
                     tc::make_sdesc(b0 + ks * 2048, Q * 128, 1024), idesc, ks > 0);
      }
      tc::mma_commit(&sm.mbar);
    }
    if (ok && !tc::mbar_wait(&sm.mbar, static_cast<uint32_t>(c & 1), kWaitPolls)) ok = false;
    tc::fence_after_sync();
    // the state entering this chunk, as bf16 rows [n][p] (MMA operand of the scan)
    __nv_bfloat16* sp = p.sprev + (((b * H + h) * p.nchunks + c) * kN + n) * kP;
#pragma unroll
    for (int q = 0; q < kP; q += 8) {
      uint4 o;
      uint32_t* ow = &o.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 v2 = __floats2bfloat162_rn(S[q + 2 * j], S[q + 2 * j + 1]);
        ow[j] = *reinterpret_cast<const uint32_t*>(&v2);
      }
      *reinterpret_cast<uint4*>(sp + q) = o;
    }
    // S = exp(cum_end) S + S_loc^T[n, :]
    const float decay = ex2_approx(cum_end * kLog2e);
    float sl[32];
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      tc::tmem_ld32(lane_base + 32 * half, sl);
#pragma unroll
      for (int j = 0; j < 32; ++j) S[32 * half + j] = fmaf(decay, S[32 * half + j], sl[j]);
    }
    tc::fence_before_sync();
    __syncthreads();  // smem tiles and TMEM are reused by the next chunk
    tc::fence_after_sync();
  }
  if (p.h_last) {
#pragma unroll
    for (int q = 0; q < kP; ++q) p.h_last[((b * H + h) * kP + q) * kN + n] = S[q];
  }
  if (!ok && tid == 0) atomicOr(p.status, 1);
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------------------
// chunk scan: one block per (b, chunk, h)
// ---------------------------------------------------------------------------
template <int Q>
struct ScanSmem {
  unsigned char c[Q * kN * 2];     // C chunk: K-major A operand (rows = time)
  unsigned char bk[Q * kN * 2];    // B chunk: K-major B operand of G (rows = time)
  unsigned char xs[Q * kP * 2];    // X' = dt' x: MN-major B operand (rows = time)
  unsigned char sp[kN * kP * 2];   // S_prev [n][p]: MN-major B operand (rows = state)
  unsigned char m[128 * 128 * 2];  // masked decay block, K-major A operand (128 x 128)
  float cum[Q];
  float dtp[Q];
  float wtot[kThreads / 32];
  uint64_t mbar;
  uint32_t tmem;
};

template <int Q, bool HAS_Z>
__global__ void __launch_bounds__(kThreads) ssd_scan_kernel(const SsdParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ScanSmem<Q>& sm = *reinterpret_cast<ScanSmem<Q>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t L = p.seqlen, H = p.nheads;
  const int64_t t0 = c * Q;
  const int len = static_cast<int>(imin64(Q, L - t0));
  const float Ah = p.A[h];
  const float biash = p.bias ? p.bias[h] : 0.f;
  const float Dh = p.D ? p.D[h] : 0.f;
  constexpr uint32_t kColG = 0, kColZ = 256, kColY = 320;

  if (warp == 0) tc::tmem_alloc(&sm.tmem, 512);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar, 1);
    tc::mbar_fence_init();
  }
  load_tile_128(sm.c, p.C + (b * L + t0) * kN, kN, Q, len, kN);
  load_tile_128(sm.bk, p.B + (b * L + t0) * kN, kN, Q, len, kN);
  load_tile_128(sm.sp, p.sprev + ((b * H + h) * p.nchunks + c) * kN * kP, kP, kN, kN, kP);
  cp_async_commit();
  for (int i = tid; i < Q; i += kThreads) {
    const float s = i < len ? step_size(__bfloat162float(p.delta[(b * L + t0 + i) * H + h]) + biash,
                                        p.softplus)
                            : 0.f;
    sm.dtp[i] = s;
    sm.cum[i] = s * Ah;
  }
  __syncthreads();
  block_cumsum<Q>(sm.cum, sm.wtot);
  // X'_t = dt'_t x_t (bf16, MN-major rows = time)
  for (int i = tid; i < Q * (kP / 8); i += kThreads) {
    const int t = i / (kP / 8);
    const int p8 = (i % (kP / 8)) * 8;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (t < len) {
      const float w = sm.dtp[t];
      const uint4 raw = *reinterpret_cast<const uint4*>(p.x + ((b * L + t0 + t) * H + h) * kP + p8);
      const uint32_t* rw = &raw.x;
      uint32_t* ow = &out.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(rw[j] << 16) * w,
                                                        __uint_as_float(rw[j] & 0xffff0000u) * w);
        ow[j] = *reinterpret_cast<const uint32_t*>(&v2);
      }
    }
    *reinterpret_cast<uint4*>(sm.xs + tc::sw128_offset(t, p8)) = out;
  }
  cp_async_wait_all();
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * warp) << 16);
  uint32_t phase = 0;
  bool ok = true;

  for (int i = 0; i < Q / 128; ++i) {
    const int kend = 128 * (i + 1);  // causal: keys [0, kend) reach this row block
    if (tid == 0 && ok) {
      const uint32_t ca = tc::smem_u32(sm.c) + i * 128 * 128;  // rows 128 i.. of each 64-col block
      const uint32_t bb = tc::smem_u32(sm.bk);
      const uint32_t idg = i == 0 ? tc::make_idesc_bf16(128, 128, 0, 0)
                                  : tc::make_idesc_bf16(128, 256, 0, 0);
      constexpr uint32_t idz = tc::make_idesc_bf16(128, kP, 0, 1);
#pragma unroll
      for (int ks = 0; ks < kN / 16; ++ks) {
        const uint64_t ad = tc::make_sdesc(ca + (ks / 4) * (Q * 128) + (ks % 4) * 32, 16, 1024);
        tc::mma_bf16(tmem + kColG, ad,
                     tc::make_sdesc(bb + (ks / 4) * (Q * 128) + (ks % 4) * 32, 16, 1024), idg,
                     ks > 0);
        tc::mma_bf16(tmem + kColZ, ad,
                     tc::make_sdesc(tc::smem_u32(sm.sp) + ks * 2048, kN * 128, 1024), idz, ks > 0);
      }
      tc::mma_commit(&sm.mbar);
    }
    if (ok && !tc::mbar_wait(&sm.mbar, phase, kWaitPolls)) ok = false;
    phase ^= 1;
    tc::fence_after_sync();

    const int tr = 128 * i + tid;  // this thread's row (time step) in the chunk
    const float cum_t = sm.cum[tr];
    for (int half = 0; half < kend / 128; ++half) {
      // masked decays of keys [128 half, 128 half + 128) for row tr -> bf16 operand
#pragma unroll 1
      for (int cb = 0; cb < 128; cb += 32) {
        float g[32];
        tc::tmem_ld32(lane_base + kColG + 128 * half + cb, g);
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const int k0 = 128 * half + cb + j;
          const float e0 = k0 <= tr ? ex2_approx((cum_t - sm.cum[k0]) * kLog2e) * g[j] : 0.f;
          const float e1 = k0 + 1 <= tr ? ex2_approx((cum_t - sm.cum[k0 + 1]) * kLog2e) * g[j + 1] : 0.f;
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(e0, e1);
          packed[j / 2] = *reinterpret_cast<const uint32_t*>(&v2);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = cb + 8 * q;  // 0..127 within the half
          *reinterpret_cast<uint4*>(sm.m + (col / 64) * (128 * 128) + tc::sw128_offset(tid, col % 64)) =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid == 0 && ok) {
        constexpr uint32_t idy = tc::make_idesc_bf16(128, kP, 0, 1);
        const uint32_t ma = tc::smem_u32(sm.m);
        const uint32_t xb = tc::smem_u32(sm.xs) + (128 * half) * 128;
#pragma unroll
        for (int ks = 0; ks < 128 / 16; ++ks) {
          tc::mma_bf16(tmem + kColY, tc::make_sdesc(ma + (ks / 4) * (128 * 128) + (ks % 4) * 32, 16, 1024),
                       tc::make_sdesc(xb + ks * 2048, Q * 128, 1024), idy, half > 0 || ks > 0);
        }
        tc::mma_commit(&sm.mbar);
      }
      if (ok && !tc::mbar_wait(&sm.mbar, phase, kWaitPolls)) ok = false;
      phase ^= 1;
      tc::fence_after_sync();
    }

    // epilogue: y = Y + exp(cum_t) Z + D x (then the gate), row tr.  The
    // tensor-memory loads are warp-collective: every lane runs them.
    {
      const bool row_ok = tr < len;
      const float ec = ex2_approx(cum_t * kLog2e);
      const int64_t row = ((b * L + t0 + (row_ok ? tr : 0)) * H + h) * kP;
#pragma unroll
      for (int cb = 0; cb < kP; cb += 32) {
        float yv[32], zv[32];
        tc::tmem_ld32(lane_base + kColY + cb, yv);
        tc::tmem_ld32(lane_base + kColZ + cb, zv);
        if (!row_ok) continue;
#pragma unroll
        for (int q = 0; q < 32; q += 8) {
          const uint4 xr = *reinterpret_cast<const uint4*>(p.x + row + cb + q);
          const uint32_t* xw = &xr.x;
          uint4 zr = make_uint4(0, 0, 0, 0);
          if (HAS_Z) zr = *reinterpret_cast<const uint4*>(p.z + row + cb + q);
          const uint32_t* zw = &zr.x;
          uint4 o;
          uint32_t* ow = &o.x;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float v0 = yv[q + 2 * j] + ec * zv[q + 2 * j] + Dh * __uint_as_float(xw[j] << 16);
            float v1 = yv[q + 2 * j + 1] + ec * zv[q + 2 * j + 1] +
                       Dh * __uint_as_float(xw[j] & 0xffff0000u);
            if (HAS_Z) {
              v0 *= silu_f(__uint_as_float(zw[j] << 16));
              v1 *= silu_f(__uint_as_float(zw[j] & 0xffff0000u));
            }
            const __nv_bfloat162 v2 = __floats2bfloat162_rn(v0, v1);
            ow[j] = *reinterpret_cast<const uint32_t*>(&v2);
          }
          *reinterpret_cast<uint4*>(p.y + row + cb + q) = o;
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();  // G / Y / Z columns are rewritten by the next row block
    tc::fence_after_sync();
  }
  if (!ok && tid == 0) atomicOr(p.status, 1);
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace ssd
}  // namespace ssm

// scan_fwd.cuh -- the fused Mamba-1 selective-scan forward kernels (sm_100a).
//
// Computes, per channel (b, d) and state n (page "Mamba状态空间模型的硬件感知
// 推理优化", sections 1 and 3.1; page "Mamba ... 并行扫描", sections 2.2-2.3):
//   dt' = softplus(delta + bias_d);  dA = exp(dt' A[d,n]);
//   h[n] = dA h[n] + dt' B[b,n,t] u;  y = (sum_n C[b,n,t] h[n] + D_d u) silu(z).
//
// Work decomposition.  The scan is done sequentially in time by each thread
// (the work-optimal form: one multiply-add per state and step), with
// parallelism over channels and state groups: kNG = 4 lanes share one
// channel, each owning kNPT = 4 of the (up to) 16 states, so a 128-thread
// block covers kCH = 32 channels.  Each input element is read from HBM once:
// tiles of kTL time steps of u / delta / z (kCH rows) and B / C (16 rows)
// are staged into shared memory with 16-byte cp.async copies, two tiles in
// flight.  Per tile the block converts B and C to fp32 once (they are shared
// by every channel of the batch) and computes dt' and dt' * u per element
// once (shared by the 4 lanes of a channel).  The partial sums C.h of the 4
// lanes are reduced through shared memory in sub-tiles of 8 steps, after
// which each lane finishes 2 steps: skip term, gate, rounding to the output
// type.  y tiles leave through shared memory with 16-byte stores.
//
// Long sequences with few channels are split into L-segments so that the
// grid fills the GPU (page "Mamba ... 并行扫描", section 2.3: block-local
// scan, combine of block aggregates, fix-up).  Segments are joined with the
// combine operator (A1, B1) (+) (A2, B2) = (A2 A1, A2 B1 + B2): a first pass
// (MODE kAgg) scans every segment but the last from a zero state and stores
// its aggregate (sum of dt', end state); a small kernel folds the aggregates
// in order into each segment's incoming state, using prod_t exp(dt'_t A) =
// exp(A sum_t dt'_t); the full pass (MODE kFull) then runs every segment from
// its incoming state.  No block ever waits on another.
#pragma once
#include "common.cuh"

namespace ssm {

struct ScanParams {
  int64_t batch, dim, dstate, seqlen;
  const void* u;
  const void* delta;
  const void* z;
  void* y;
  const void* B;
  const void* C;
  int64_t u_sb, u_sd, dl_sb, dl_sd, z_sb, z_sd, y_sb, y_sd, B_sb, B_sn, C_sb, C_sn;
  const float* A;
  const float* D;
  const float* bias;
  int softplus;
  const float* h0;
  float* h_last;
  int64_t nseg, seg_len;
  float* carry_h;   // ((nseg - 1) * batch * dim) x 16
  float* carry_dt;  // (nseg - 1) * batch * dim
};

namespace fwd {

constexpr int kThreads = 128;
constexpr int kNG = 4;                  // lanes per channel
constexpr int kNPT = 4;                 // states per lane
constexpr int kMaxN = kNG * kNPT;       // 16
constexpr int kCH = kThreads / kNG;     // channels per block
constexpr int kTL = 64;                 // time steps per tile
constexpr int kSub = 8;                 // steps per reduction sub-tile
constexpr int kFull = 0, kAgg = 1;

template <typename T>
struct Smem {
  static constexpr int kEPC = 16 / (int)sizeof(T);  // elements per 16-byte chunk
  static constexpr int kRow = kTL + kEPC;            // raw row: tile + 16-byte pad
  T raw_u[2][kCH][kRow];
  T raw_dl[2][kCH][kRow];
  T raw_z[2][kCH][kRow];
  T raw_B[2][kMaxN][kRow];
  T raw_C[2][kMaxN][kRow];
  T yout[kCH][kRow];
  float dtp[kCH][kTL + 4];   // dt' per (channel, step)
  float du[kCH][kTL + 4];    // dt' * u
  float Bf[kTL][kMaxN];      // fp32 B, 16-byte chunks swizzled by (t >> 1) & 3
  float Cf[kTL][kMaxN];
  float red[kCH][kNG][kSub];  // partial C.h of each lane
};

__device__ __forceinline__ int bc_swizzle(int t) { return (t >> 1) & 3; }

template <typename T, int MODE, bool HAS_Z, bool VEC>
__global__ void __launch_bounds__(kThreads) scan_fwd_kernel(const ScanParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<T>& sm = *reinterpret_cast<Smem<T>*>(smem_raw);
  constexpr int kEPC = Smem<T>::kEPC;
  constexpr int kCPR = kTL / kEPC;  // 16-byte chunks per raw row
  constexpr bool kGate = HAS_Z && MODE == kFull;

  const int tid = threadIdx.x;
  const int cl = tid / kNG;
  const int g = tid % kNG;
  const int64_t b = blockIdx.y;
  const int64_t d0 = static_cast<int64_t>(blockIdx.x) * kCH;
  const int64_t d = d0 + cl;
  const bool ch_ok = d < p.dim;
  const int64_t seg = blockIdx.z;
  const int64_t l0 = seg * p.seg_len;
  const int64_t l1 = imin64(p.seqlen, l0 + p.seg_len);
  const int N = static_cast<int>(p.dstate);
  const int64_t bd = b * p.dim + d;

  const T* gu = static_cast<const T*>(p.u);
  const T* gdl = static_cast<const T*>(p.delta);
  const T* gz = static_cast<const T*>(p.z);
  const T* gB = static_cast<const T*>(p.B);
  const T* gC = static_cast<const T*>(p.C);

  // ---- per-thread constants and incoming state -------------------------------
  float A2[kNPT], h[kNPT];
#pragma unroll
  for (int k = 0; k < kNPT; ++k) {
    const int n = g * kNPT + k;
    const bool ok = ch_ok && n < N;
    A2[k] = ok ? p.A[d * N + n] * kLog2e : 0.f;
    float hin = 0.f;
    if (MODE == kFull && ok) {
      if (seg == 0) {
        hin = p.h0 ? p.h0[bd * N + n] : 0.f;
      } else {
        hin = p.carry_h[((seg - 1) * p.batch * p.dim + bd) * kMaxN + n];
      }
    }
    h[k] = hin;
  }
  const float biasd = (ch_ok && p.bias) ? p.bias[d] : 0.f;
  const float Dd = (ch_ok && p.D) ? p.D[d] : 0.f;
  float dtsum = 0.f;

  // ---- tile loads ----------------------------------------------------------------
  // Row r of a tile: [0, kCH) u, [kCH, 2kCH) delta, [2kCH, 2kCH + 16) B, then
  // (full pass) 16 rows of C and, with a gate, kCH rows of z.
  constexpr int kRowsAgg = 2 * kCH + kMaxN;
  constexpr int kRows = MODE == kFull ? kRowsAgg + kMaxN + (HAS_Z ? kCH : 0) : kRowsAgg;
  auto row_src = [&](int r, int buf, const T*& src, T*& dst) {
    if (r < kCH) {
      const int64_t dd = d0 + r;
      src = dd < p.dim ? gu + b * p.u_sb + dd * p.u_sd : nullptr;
      dst = sm.raw_u[buf][r];
    } else if (r < 2 * kCH) {
      const int64_t dd = d0 + r - kCH;
      src = dd < p.dim ? gdl + b * p.dl_sb + dd * p.dl_sd : nullptr;
      dst = sm.raw_dl[buf][r - kCH];
    } else if (r < 2 * kCH + kMaxN) {
      const int n = r - 2 * kCH;
      src = n < N ? gB + b * p.B_sb + n * p.B_sn : nullptr;
      dst = sm.raw_B[buf][n];
    } else if (r < 2 * kCH + 2 * kMaxN) {
      const int n = r - 2 * kCH - kMaxN;
      src = n < N ? gC + b * p.C_sb + n * p.C_sn : nullptr;
      dst = sm.raw_C[buf][n];
    } else {
      const int64_t dd = d0 + r - 2 * kCH - 2 * kMaxN;
      src = dd < p.dim ? gz + b * p.z_sb + dd * p.z_sd : nullptr;
      dst = sm.raw_z[buf][r - 2 * kCH - 2 * kMaxN];
    }
  };
  auto issue_load = [&](int buf, int64_t t0) {
    const int len = static_cast<int>(imin64(kTL, l1 - t0));
    if (VEC) {
      for (int i = tid; i < kRows * kCPR; i += kThreads) {
        const int r = i / kCPR;
        const int e = (i % kCPR) * kEPC;
        const T* src;
        T* dst;
        row_src(r, buf, src, dst);
        int nbytes = 0;
        const T* from = gu;  // any valid address when nothing is read
        if (src != nullptr && e < len) {
          nbytes = min(kEPC, len - e) * static_cast<int>(sizeof(T));
          from = src + t0 + e;
        }
        cp_async16(dst + e, from, nbytes);
      }
      cp_async_commit();
    } else {
      for (int i = tid; i < kRows * kTL; i += kThreads) {
        const int r = i / kTL;
        const int e = i % kTL;
        const T* src;
        T* dst;
        row_src(r, buf, src, dst);
        dst[e] = (src != nullptr && e < len) ? src[t0 + e] : from_f32<T>(0.f);
      }
    }
  };

  const int64_t ntiles = l1 > l0 ? (l1 - l0 + kTL - 1) / kTL : 0;
  if (ntiles > 0) issue_load(0, l0);

  for (int64_t k = 0; k < ntiles; ++k) {
    const int buf = static_cast<int>(k & 1);
    const int64_t t0 = l0 + k * kTL;
    const int len = static_cast<int>(imin64(kTL, l1 - t0));
    if (VEC) cp_async_wait_all();
    __syncthreads();  // tile k visible; the previous y tile has been stored

    // ---- per-tile preparation ------------------------------------------------------
    {  // B (and C) to fp32, transposed to [t][n]
      const int t = tid % kTL;
      const int half = tid / kTL;  // states [8 half, 8 half + 8)
      const int sw = bc_swizzle(t);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int chunk = 2 * half + j;
        float4 vb;
        vb.x = to_f32(sm.raw_B[buf][4 * chunk + 0][t]);
        vb.y = to_f32(sm.raw_B[buf][4 * chunk + 1][t]);
        vb.z = to_f32(sm.raw_B[buf][4 * chunk + 2][t]);
        vb.w = to_f32(sm.raw_B[buf][4 * chunk + 3][t]);
        *reinterpret_cast<float4*>(&sm.Bf[t][4 * (chunk ^ sw)]) = vb;
        if (MODE == kFull) {
          float4 vc;
          vc.x = to_f32(sm.raw_C[buf][4 * chunk + 0][t]);
          vc.y = to_f32(sm.raw_C[buf][4 * chunk + 1][t]);
          vc.z = to_f32(sm.raw_C[buf][4 * chunk + 2][t]);
          vc.w = to_f32(sm.raw_C[buf][4 * chunk + 3][t]);
          *reinterpret_cast<float4*>(&sm.Cf[t][4 * (chunk ^ sw)]) = vc;
        }
      }
    }
    {  // dt' and dt' u for steps [16 g, 16 g + 16) of this thread's channel
      const int tq = g * (kTL / kNG);
#pragma unroll
      for (int j = 0; j < kTL / kNG; j += 4) {
        float4 vdt, vdu;
        float* pdt = &vdt.x;
        float* pdu = &vdu.x;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = tq + j + q;
          const float s = to_f32(sm.raw_dl[buf][cl][t]) + biasd;
          float dt = p.softplus ? softplus_f(s) : s;
          dt = t < len ? dt : 0.f;  // steps past the end leave the state alone
          pdt[q] = dt;
          pdu[q] = dt * to_f32(sm.raw_u[buf][cl][t]);
        }
        *reinterpret_cast<float4*>(&sm.dtp[cl][tq + j]) = vdt;
        *reinterpret_cast<float4*>(&sm.du[cl][tq + j]) = vdu;
      }
    }
    __syncthreads();
    if (k + 1 < ntiles) issue_load(buf ^ 1, t0 + kTL);

    // ---- the scan over this tile ---------------------------------------------------
    const int nsub = (len + kSub - 1) / kSub;
    for (int s = 0; s < nsub; ++s) {
      const int tb = s * kSub;
      float dtv[kSub], duv[kSub];
      *reinterpret_cast<float4*>(&dtv[0]) = *reinterpret_cast<const float4*>(&sm.dtp[cl][tb]);
      *reinterpret_cast<float4*>(&dtv[4]) = *reinterpret_cast<const float4*>(&sm.dtp[cl][tb + 4]);
      *reinterpret_cast<float4*>(&duv[0]) = *reinterpret_cast<const float4*>(&sm.du[cl][tb]);
      *reinterpret_cast<float4*>(&duv[4]) = *reinterpret_cast<const float4*>(&sm.du[cl][tb + 4]);
      float yp[kSub];
#pragma unroll
      for (int tt = 0; tt < kSub; ++tt) {
        const int t = tb + tt;
        const int col = 4 * (g ^ bc_swizzle(t));
        const float4 bq = *reinterpret_cast<const float4*>(&sm.Bf[t][col]);
        const float bv[4] = {bq.x, bq.y, bq.z, bq.w};
        if (MODE == kFull) {
          const float4 cq = *reinterpret_cast<const float4*>(&sm.Cf[t][col]);
          const float cv[4] = {cq.x, cq.y, cq.z, cq.w};
          float acc = 0.f;
#pragma unroll
          for (int kk = 0; kk < kNPT; ++kk) {
            const float dA = ex2_approx(dtv[tt] * A2[kk]);
            h[kk] = fmaf(dA, h[kk], duv[tt] * bv[kk]);
            acc = fmaf(cv[kk], h[kk], acc);
          }
          yp[tt] = acc;
        } else {
#pragma unroll
          for (int kk = 0; kk < kNPT; ++kk) {
            const float dA = ex2_approx(dtv[tt] * A2[kk]);
            h[kk] = fmaf(dA, h[kk], duv[tt] * bv[kk]);
          }
          dtsum += dtv[tt];
        }
      }
      if (MODE == kFull) {
        *reinterpret_cast<float4*>(&sm.red[cl][g][0]) = make_float4(yp[0], yp[1], yp[2], yp[3]);
        *reinterpret_cast<float4*>(&sm.red[cl][g][4]) = make_float4(yp[4], yp[5], yp[6], yp[7]);
        __syncwarp();
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int gg = 0; gg < kNG; ++gg) {
          const float2 v = *reinterpret_cast<const float2*>(&sm.red[cl][gg][2 * g]);
          y0 += v.x;
          y1 += v.y;
        }
        __syncwarp();
        const float ys[2] = {y0, y1};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int t = tb + 2 * g + i;
          if (t < len) {
            const float uv = to_f32(sm.raw_u[buf][cl][t]);
            float yv = fmaf(Dd, uv, ys[i]);
            if (kGate) yv *= silu_f(to_f32(sm.raw_z[buf][cl][t]));
            sm.yout[cl][t] = from_f32<T>(yv);
          }
        }
      }
    }

    // ---- store the y tile ------------------------------------------------------------
    if (MODE == kFull) {
      __syncthreads();
      T* gy = static_cast<T*>(p.y);
      if (VEC) {
        for (int i = tid; i < kCH * kCPR; i += kThreads) {
          const int r = i / kCPR;
          const int e = (i % kCPR) * kEPC;
          const int64_t dd = d0 + r;
          if (dd >= p.dim || e >= len) continue;
          T* dst = gy + b * p.y_sb + dd * p.y_sd + t0 + e;
          if (e + kEPC <= len) {
            *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(&sm.yout[r][e]);
          } else {
            for (int q = 0; q < len - e; ++q) dst[q] = sm.yout[r][e + q];
          }
        }
      } else {
        for (int i = tid; i < kCH * kTL; i += kThreads) {
          const int r = i / kTL;
          const int e = i % kTL;
          const int64_t dd = d0 + r;
          if (dd < p.dim && e < len) gy[b * p.y_sb + dd * p.y_sd + t0 + e] = sm.yout[r][e];
        }
      }
    }
  }

  // ---- outgoing state ----------------------------------------------------------------
  if (!ch_ok) return;
  if (MODE == kFull) {
    if (p.h_last != nullptr && seg == p.nseg - 1) {
#pragma unroll
      for (int k = 0; k < kNPT; ++k) {
        const int n = g * kNPT + k;
        if (n < N) p.h_last[bd * N + n] = h[k];
      }
    }
  } else {
    const int64_t slot = seg * p.batch * p.dim + bd;
#pragma unroll
    for (int k = 0; k < kNPT; ++k) p.carry_h[slot * kMaxN + g * kNPT + k] = h[k];
    if (g == 0) p.carry_dt[slot] = dtsum;
  }
}

// Folds the segment aggregates in order: the state entering segment s + 1 is
// exp(A sum dt'_s) * (state entering s) + (end state of s from zero); it
// overwrites the aggregate of segment s in place.
__global__ void scan_carry_kernel(const ScanParams p) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = p.batch * p.dim * kMaxN;
  if (idx >= total) return;
  const int n = static_cast<int>(idx % kMaxN);
  const int64_t bd = idx / kMaxN;
  const int64_t d = bd % p.dim;
  const int N = static_cast<int>(p.dstate);
  if (n >= N) return;
  const float a = p.A[d * N + n];
  float hs = p.h0 ? p.h0[bd * N + n] : 0.f;
  for (int64_t s = 0; s + 1 < p.nseg; ++s) {
    const int64_t slot = s * p.batch * p.dim + bd;
    hs = fmaf(expf(a * p.carry_dt[slot]), hs, p.carry_h[slot * kMaxN + n]);
    p.carry_h[slot * kMaxN + n] = hs;
  }
}

}  // namespace fwd
}  // namespace ssm

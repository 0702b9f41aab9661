// scan_step.cuh -- one decode step of the selective scan (sm_100a).
//
// Page "Mamba与选择性SSM" (mlqm.cn), section 5.4: incremental decoding keeps
// only the fixed-size state between tokens; one step is the recurrence of the
// full scan applied once, reading and overwriting the state in place.
//
// The step is bound by the state's HBM traffic (16 fp32 read and written per
// channel), so four lanes share a channel and each moves one 16-byte quarter
// of its state: a warp touches 8 channels x 64 contiguous bytes.  The four
// partial sums C.h are combined with two butterfly shuffles.
#pragma once
#include "common.cuh"

namespace ssm {

struct StepParams {
  int64_t batch, dim, dstate;
  const void* u;
  const void* delta;
  const void* z;
  const void* B;
  const void* C;
  const float* A;
  const float* D;
  const float* bias;
  int softplus;
  float* state;
  void* y;
};

namespace step {
constexpr int kThreads = 256;
constexpr int kNG = 4;
constexpr int kNPT = 4;

template <typename T, bool HAS_Z, bool VEC4>
__global__ void __launch_bounds__(kThreads) scan_step_kernel(const StepParams p) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t ch = idx / kNG;
  const int g = static_cast<int>(idx % kNG);
  const bool ok = ch < p.batch * p.dim;
  const int N = static_cast<int>(p.dstate);
  float acc = 0.f, uv = 0.f;
  int64_t b = 0, d = 0;
  if (ok) {
    b = ch / p.dim;
    d = ch % p.dim;
    const float s = to_f32(static_cast<const T*>(p.delta)[ch]) + (p.bias ? p.bias[d] : 0.f);
    const float dt = p.softplus ? softplus_f(s) : s;
    uv = to_f32(static_cast<const T*>(p.u)[ch]);
    const float du = dt * uv;
    const T* Bb = static_cast<const T*>(p.B) + b * N;
    const T* Cb = static_cast<const T*>(p.C) + b * N;
    const float* Ad = p.A + d * N;
    float* st = p.state + ch * N;
    if (VEC4) {  // N == 16 and the state is 16-byte aligned
      float4 hv = *reinterpret_cast<const float4*>(st + kNPT * g);
      float hs[kNPT] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
      for (int k = 0; k < kNPT; ++k) {
        const int n = kNPT * g + k;
        const float dA = ex2_approx(dt * (Ad[n] * kLog2e));
        hs[k] = fmaf(dA, hs[k], du * to_f32(Bb[n]));
        acc = fmaf(to_f32(Cb[n]), hs[k], acc);
      }
      *reinterpret_cast<float4*>(st + kNPT * g) = make_float4(hs[0], hs[1], hs[2], hs[3]);
    } else {
#pragma unroll
      for (int k = 0; k < kNPT; ++k) {
        const int n = kNPT * g + k;
        if (n < N) {
          const float dA = ex2_approx(dt * (Ad[n] * kLog2e));
          const float hn = fmaf(dA, st[n], du * to_f32(Bb[n]));
          st[n] = hn;
          acc = fmaf(to_f32(Cb[n]), hn, acc);
        }
      }
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  if (ok && g == 0) {
    float yv = acc + (p.D ? p.D[d] * uv : 0.f);
    if (HAS_Z) yv *= silu_f(to_f32(static_cast<const T*>(p.z)[ch]));
    static_cast<T*>(p.y)[ch] = from_f32<T>(yv);
  }
}
}  // namespace step
}  // namespace ssm

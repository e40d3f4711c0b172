// la_step.cu -- one decode token of causal linear attention.
//
// "1.6 长上下文与高效注意力", section 线性注意力: inference keeps a constant-size
// state and adds one outer product per token.  With the state stored as S^T
// ([d_k][d_v], fp32) and the per-head decay gamma:
//     S^T[c][r] <- gamma S^T[c][r] + phi(k)_c v_r,     o_r = sum_c S^T[c][r] phi(q)_c.
// la_step_gated takes the decay per (sequence, head) as exp(g[n][h]) instead
// (a data-dependent decay: "1.6 长上下文与高效注意力", section 状态空间模型与 Mamba).
// The normalised form (la_step_norm) also carries z, the running key sum of
// the same section's displayed equation:
//     z[c] <- gamma z[c] + phi(k)_c,     o_r /= sum_c z[c] phi(q)_c.
// The state is read once and written once, so the kernel is bound by HBM
// bandwidth: one CTA per (sequence, head) streams its d_k x d_v slab with
// 16-byte loads and stores that bypass L1 and are marked for eviction first
// (each line is touched exactly once), then reduces o across row groups in
// shared memory.
#include <cuda_bf16.h>

#include "la_common.cuh"
#include "la_internal.h"

namespace la {
namespace {

constexpr int kStepThreads = 256;
constexpr int kRowsUnroll = 8;

// Shared memory: qh [dk], kh [dk], then (16-byte aligned) the row-group
// partial outputs [nrg][ncg] float4, then one normaliser partial per warp.
__host__ __device__ inline int step_red_offset(int dk) { return (2 * dk + 3) & ~3; }

template <typename Tin, bool NORM>
__global__ void __launch_bounds__(kStepThreads)
step_kernel(StepArgs a) {
  extern __shared__ float sm[];
  const int dk = a.dk, dv = a.dv;
  const int ncg = dv >> 2;              // float4 column groups
  const int nrg = kStepThreads / ncg;   // row groups
  float *qh = sm;                       // [dk]
  float *kh = sm + dk;                  // [dk]
  float4 *red = (float4 *)(sm + step_red_offset(dk));  // [nrg][ncg]
  float *zred = sm + step_red_offset(dk) + 4 * nrg * ncg;  // [kStepThreads / 32]

  const int64_t unit = blockIdx.x;  // n * H + h
  const int h = (int)(unit % a.H);
  const int64_t n = unit / a.H;
  const int tid = threadIdx.x;
  const Tin *Q = (const Tin *)a.q.data + n * a.q.sb + h * a.q.sh;
  const Tin *K = (const Tin *)a.k.data + n * a.k.sb + h * a.k.sh;
  const Tin *V = (const Tin *)a.v.data + n * a.v.sb + h * a.v.sh;
  const int cg = tid % ncg, rg = tid / ncg;
  float4 *S = (float4 *)(a.state + unit * (int64_t)dk * dv) + cg;
  float4 s[kRowsUnroll];  // this thread's first state rows: in flight while q, k, v arrive
  if (rg < nrg) {
#pragma unroll
    for (int u = 0; u < kRowsUnroll; ++u) {
      const int c = rg + u * nrg;
      if (c < dk) s[u] = __ldcs(S + (int64_t)c * ncg);
    }
  }
  for (int c = tid; c < dk; c += kStepThreads) {
    qh[c] = feature_map(to_f32<Tin>(Q[c]), a.phi);
    kh[c] = feature_map(to_f32<Tin>(K[c]), a.phi);
  }
  const float g = a.g ? expf(a.g[unit]) : a.gamma[h];  // data-dependent decay: exp(g[n][h])
  float4 vr = make_float4(0.f, 0.f, 0.f, 0.f);
  if (rg < nrg) {
    vr.x = to_f32<Tin>(V[4 * cg + 0]);
    vr.y = to_f32<Tin>(V[4 * cg + 1]);
    vr.z = to_f32<Tin>(V[4 * cg + 2]);
    vr.w = to_f32<Tin>(V[4 * cg + 3]);
  }
  __syncthreads();

  if (NORM) {  // z <- gamma z + kh, and this thread's share of z . qh
    float *Z = a.z + unit * (int64_t)dk;
    float part = 0.f;
    for (int c = tid; c < dk; c += kStepThreads) {
      const float zc = fmaf(g, Z[c], kh[c]);
      Z[c] = zc;
      part = fmaf(zc, qh[c], part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) zred[tid >> 5] = part;  // read after the barrier below
  }

  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if (rg < nrg) {
    for (int c0 = rg; c0 < dk; c0 += nrg * kRowsUnroll) {
      if (c0 != rg) {
#pragma unroll
        for (int u = 0; u < kRowsUnroll; ++u) {
          const int c = c0 + u * nrg;
          if (c < dk) s[u] = __ldcs(S + (int64_t)c * ncg);
        }
      }
#pragma unroll
      for (int u = 0; u < kRowsUnroll; ++u) {
        const int c = c0 + u * nrg;
        if (c < dk) {
          const float kc = kh[c], qc = qh[c];
          float4 x = s[u];
          x.x = fmaf(g, x.x, kc * vr.x);
          x.y = fmaf(g, x.y, kc * vr.y);
          x.z = fmaf(g, x.z, kc * vr.z);
          x.w = fmaf(g, x.w, kc * vr.w);
          __stcs(S + (int64_t)c * ncg, x);
          o.x = fmaf(x.x, qc, o.x);
          o.y = fmaf(x.y, qc, o.y);
          o.z = fmaf(x.z, qc, o.z);
          o.w = fmaf(x.w, qc, o.w);
        }
      }
    }
    red[rg * ncg + cg] = o;
  }
  __syncthreads();
  if (tid < ncg) {
    float4 acc = red[tid];
    for (int r = 1; r < nrg; ++r) {
      const float4 y = red[r * ncg + tid];
      acc.x += y.x; acc.y += y.y; acc.z += y.z; acc.w += y.w;
    }
    if (NORM) {
      float den = 0.f;
#pragma unroll
      for (int w = 0; w < kStepThreads / 32; ++w) den += zred[w];
      acc.x /= den; acc.y /= den; acc.z /= den; acc.w /= den;
    }
    Tin *O = (Tin *)a.out + n * a.o_sb + h * a.o_sh + 4 * tid;
    O[0] = from_f32<Tin>(acc.x);
    O[1] = from_f32<Tin>(acc.y);
    O[2] = from_f32<Tin>(acc.z);
    O[3] = from_f32<Tin>(acc.w);
  }
}

}  // namespace

bool step_supported(const StepArgs &a) {
  // d_v/4 column groups must divide the block (power of two, 1..256 groups).
  const int ncg = a.dv / 4;
  return a.dv % 4 == 0 && ncg >= 1 && ncg <= kStepThreads && (kStepThreads % ncg) == 0 &&
         a.dk >= 1 && a.dk <= 1024;
}

cudaError_t launch_step(const StepArgs &a, cudaStream_t stream) {
  const int64_t grid = a.N * a.H;
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int nrg = kStepThreads / (a.dv / 4);
  const size_t smem = step_red_offset(a.dk) * sizeof(float) + (size_t)nrg * (a.dv / 4) * sizeof(float4) +
                      (kStepThreads / 32) * sizeof(float);
  const bool norm = a.z != nullptr;
  if (a.dtype == LA_F32) {
    if (norm)
      step_kernel<float, true><<<(unsigned)grid, kStepThreads, smem, stream>>>(a);
    else
      step_kernel<float, false><<<(unsigned)grid, kStepThreads, smem, stream>>>(a);
  } else {
    if (norm)
      step_kernel<__nv_bfloat16, true><<<(unsigned)grid, kStepThreads, smem, stream>>>(a);
    else
      step_kernel<__nv_bfloat16, false><<<(unsigned)grid, kStepThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace la

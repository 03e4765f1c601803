// Inference form of causal linear attention (article "Lightning Attention-2
// 新一代注意力机制", section "Lightning Attention-2速度对比": linear attention
// converts losslessly to an RNN; section "Lightning Attention-2简介", point 2:
// the KV state accumulated block after block).
//
//   decode step, one new token per (b, h):  S += k^T v,  o = q S
//   state after a prefill:                  S += sum_t k_t^T v_t
//
// S is d x dv fp32 per (b, h), row-major, in the caller's memory. Both are
// HBM-bound (the step reads and writes the whole state for one token), so they
// run on CUDA cores with every warp access 128 contiguous bytes.
#pragma once

#include "la2_common.cuh"

namespace la2 {

constexpr int kDecodeWarps = 8;
constexpr int kRows = 128 / kDecodeWarps;  // state rows per thread at the largest d

// grid (B*H, ceil(dv / 32)); block 256. Lane l of every warp owns column
// 32*blockIdx.y + l; warp w owns state rows w, w + 8, ... The eight partial
// dot products q . S[:, j] meet in shared memory.
template <typename T>
__global__ void __launch_bounds__(32 * kDecodeWarps)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   T* __restrict__ o, float* __restrict__ state, int d, int dv) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float part[kDecodeWarps][32];
  const int64_t bh = blockIdx.x;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int j = blockIdx.y * 32 + lane;
  const T* qb = q + bh * d;
  const T* kb = k + bh * d;
  float acc = 0.f;
  if (j < dv) {
    const float vj = to_f32(v[bh * dv + j]);
    float* col = state + bh * static_cast<int64_t>(d) * dv + j;
#pragma unroll 8
    for (int i = w; i < d; i += kDecodeWarps) {
      const float s = col[static_cast<int64_t>(i) * dv] + to_f32(kb[i]) * vj;
      col[static_cast<int64_t>(i) * dv] = s;
      acc += to_f32(qb[i]) * s;
    }
  }
  part[w][lane] = acc;
  __syncthreads();
  if (w == 0 && j < dv) {
    float sum = 0.f;
#pragma unroll
    for (int x = 0; x < kDecodeWarps; ++x) sum += part[x][lane];
    o[bh * dv + j] = from_f32<T>(sum);
  }
}

// Four columns per lane (dv % 4 == 0, state 16-byte aligned): grid
// (B*H, ceil(dv / 128)); a warp covers 128 columns of a row with float4
// accesses, so each thread keeps 16-byte loads in flight instead of 4-byte ones.
template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}

template <typename T>
__global__ void __launch_bounds__(32 * kDecodeWarps, 3)
decode_step_v4_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      T* __restrict__ o, float* __restrict__ state, int d, int dv) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float4 part[kDecodeWarps][32];
  const int64_t bh = blockIdx.x;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int j = blockIdx.y * 128 + 4 * lane;  // first of this lane's four columns
  const T* qb = q + bh * d;
  const T* kb = k + bh * d;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (j < dv) {
    const float4 vj = load4<T>(v + bh * dv + j);
    float* col = state + bh * static_cast<int64_t>(d) * dv + j;
    // A group of this thread's rows is loaded before any is written back: the
    // writes go through the same pointer, so a fused load-update-store loop
    // would keep one row in flight per thread (d <= 128: at most kRows rows,
    // in two groups so that three CTAs fit on an SM).
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      float4 x[kRows / 2];
#pragma unroll
      for (int t = 0; t < kRows / 2; ++t) {
        const int i = w + (g * kRows / 2 + t) * kDecodeWarps;
        if (i < d) x[t] = *reinterpret_cast<const float4*>(col + static_cast<int64_t>(i) * dv);
      }
#pragma unroll
      for (int t = 0; t < kRows / 2; ++t) {
        const int i = w + (g * kRows / 2 + t) * kDecodeWarps;
        if (i < d) {
          const float ki = to_f32(kb[i]), qi = to_f32(qb[i]);
          x[t].x += ki * vj.x;
          x[t].y += ki * vj.y;
          x[t].z += ki * vj.z;
          x[t].w += ki * vj.w;
          *reinterpret_cast<float4*>(col + static_cast<int64_t>(i) * dv) = x[t];
          acc.x += qi * x[t].x;
          acc.y += qi * x[t].y;
          acc.z += qi * x[t].z;
          acc.w += qi * x[t].w;
        }
      }
    }
  }
  part[w][lane] = acc;
  __syncthreads();
  if (w == 0 && j < dv) {
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int x = 0; x < kDecodeWarps; ++x) {
      sum.x += part[x][lane].x;
      sum.y += part[x][lane].y;
      sum.z += part[x][lane].z;
      sum.w += part[x][lane].w;
    }
    T* ob = o + bh * dv + j;
    ob[0] = from_f32<T>(sum.x);
    ob[1] = from_f32<T>(sum.y);
    ob[2] = from_f32<T>(sum.z);
    ob[3] = from_f32<T>(sum.w);
  }
}

// state[bh] (row-major d x dv) += sum over the C chunk states of sequence bh,
// added in chunk order. `chunk_major`: the chunk states use the tensor-core
// layout (float4 j of row r at float4 index j*d + r), else row-major.
// grid ceil(d*dv / 256) x B*H.
__global__ void __launch_bounds__(256)
state_accumulate_kernel(const float* __restrict__ chunks, float* __restrict__ state, int64_t C,
                        int d, int dv, int chunk_major) {
  pdl_launch_dependents();
  pdl_wait();
  const int nel = d * dv;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nel) return;
  const int64_t bh = blockIdx.y;
  const int r = e / dv, c = e % dv;
  const int src = chunk_major ? ((c >> 2) * d + r) * 4 + (c & 3) : e;
  const float* p = chunks + bh * C * nel + src;
  float sum = 0.f;
  for (int64_t ch = 0; ch < C; ++ch) sum += p[ch * nel];
  state[bh * static_cast<int64_t>(nel) + e] += sum;
}

}  // namespace la2

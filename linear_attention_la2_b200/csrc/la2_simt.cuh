// CUDA-core kernels of libla2: chunk states, the state scan, and the fp32
// forward / backward block loops.
//
// Article "Lightning Attention-2 新一代注意力机制", section
// "Lightning Attention-2简介", point 2 (Fig. 3): every (b, h) sequence is cut
// into blocks of Bk rows; a block's output is the masked left product of the
// block plus the right product of its queries with the KV state accumulated
// over earlier blocks, and the state then absorbs the block's K^T V.
//
// Work unit = one chunk of one (b, h) sequence: rows [c*L, min(N, (c+1)*L)),
// L a multiple of Bk. A chunk starts from the exclusive prefix of the chunk
// states of its sequence (la2_chunk_state + la2_chunk_scan), so chunks of one
// sequence run in parallel. Everything accumulates in fp32; inputs of type T
// (float or bf16) are widened on load and outputs rounded to T on store.
//
// Decayed form (`lam` non-null, causal, one K/V head per query head): head h
// has a rate lam[h] in [0, 1] and the state is multiplied by it before each
// token, KV_t = lam KV_{t-1} + k_t^T v_t, so the mask of the left product is
// D[t][s] = lam^(t-s) for s <= t. (A reading: the article has no decay; with
// lam = 1 it is the article's op.) Per block of `rows` rows starting at row i0,
// with KV the state decayed to row i0 - 1:
//   O_t  = sum_{j<=t} lam^(t-j) (q_t . k_j) v_j + lam^(t+1) q_t KV
//   KV  <- lam^rows KV + sum_j lam^(rows-1-j) k_j^T v_j
// and in the reverse walk of dK/dV, with U the suffix decayed to row i0 + rows:
//   dK_j += lam^(rows-j) v_j U^T + sum_{t>=j} lam^(t-j) (do_t . v_j) q_t   (dV alike)
//   U   <- lam^rows U + sum_t lam^t q_t^T do_t
// Powers come from powf in a table of lam^0 .. lam^Bk per CTA.
#pragma once

#include <algorithm>

#include "la2_common.cuh"

namespace la2 {

constexpr int kSimtThreads = 256;

// ----------------------------------------------------------------------------
// Chunk states: S[bh][c] = sum over rows t of chunk c of a_t^T b_t  (da x db).
// (a, b) = (K, V) gives the KV state of a chunk; (Q, dO) gives the state the
// dK/dV pass of the backward carries. One CTA per (bh, c); each thread keeps
// up to 64 state elements in registers. With `group` > 1, bh is a K/V
// sequence and its state sums the chunk over the group's query sequences
// (q_seq0(bh) + j, j < group): the summed suffix state of grouped heads.
// ----------------------------------------------------------------------------
constexpr int kStateRowsPerTile = 32;

// Decayed form: `decay` 1 weights row s of the chunk by lam^(t1-1-s) (the
// state decayed to the chunk's last row, for the prefix of later chunks), 2 by
// lam^(s-t0) (decayed to its first row, for the suffix of earlier chunks).
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
chunk_state_kernel(const T* __restrict__ a, const T* __restrict__ b, float* __restrict__ out,
                   int64_t N, int da, int db, int64_t L, int64_t C, int H, int G, int group,
                   const float* __restrict__ lam, int decay) {
  extern __shared__ float smem[];
  float* As = smem;                              // [32][da]
  float* Bs = smem + kStateRowsPerTile * da;     // [32][db]
  const int64_t unit = blockIdx.x;
  const int64_t bh = unit / C, c = unit % C;
  const int64_t t0 = c * L, t1 = imin64(N, t0 + L);
  const int nel = da * db;
  float acc[64];
#pragma unroll
  for (int r = 0; r < 64; ++r) acc[r] = 0.f;

  for (int j = 0; j < group; ++j) {
  const int64_t src = group > 1 ? q_seq0(bh, H, G) + j : bh;
  const T* ab = a + src * N * da;
  const T* bb = b + src * N * db;
  for (int64_t s0 = t0; s0 < t1; s0 += kStateRowsPerTile) {
    const int rows = (int)imin64(kStateRowsPerTile, t1 - s0);
    for (int i = threadIdx.x; i < kStateRowsPerTile * da; i += blockDim.x) {
      const int r = i / da, col = i % da;
      float w = 1.f;
      if (decay && r < rows) {
        const float l = lam[bh % H];
        w = powf(l, static_cast<float>(decay == 1 ? t1 - 1 - (s0 + r) : (s0 + r) - t0));
      }
      As[i] = r < rows ? w * to_f32(ab[(s0 + r) * da + col]) : 0.f;
    }
    for (int i = threadIdx.x; i < kStateRowsPerTile * db; i += blockDim.x) {
      const int r = i / db, col = i % db;
      Bs[i] = r < rows ? to_f32(bb[(s0 + r) * db + col]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 64; ++r) {
      const int idx = threadIdx.x + r * kSimtThreads;
      if (idx < nel) {
        const int ci = idx / db, ei = idx % db;
        float s = acc[r];
        for (int t = 0; t < rows; ++t) s = fmaf(As[t * da + ci], Bs[t * db + ei], s);
        acc[r] = s;
      }
    }
    __syncthreads();
  }
  }
  float* o = out + (bh * C + c) * (int64_t)nel;
#pragma unroll
  for (int r = 0; r < 64; ++r) {
    const int idx = threadIdx.x + r * kSimtThreads;
    if (idx < nel) o[idx] = acc[r];
  }
}

// ----------------------------------------------------------------------------
// Scan of chunk states along c, per (bh, element), in place.
//   mode 0: exclusive prefix  P_c = sum_{c' < c} S_c'   (causal, forward order)
//   mode 1: exclusive suffix  R_c = sum_{c' > c} S_c'   (causal, reverse order)
//   mode 2: total into slot 0  T = sum_c S_c             (non-causal)
//   mode 3: decayed exclusive prefix P_c = f P_{c-1} + S_{c-1}, f = lam^L
//   mode 4: decayed exclusive suffix R_c = S_{c+1} + f R_{c+1}
// (modes 3, 4: chunk states decayed to their last / first row, lam[seq % H];
// every chunk but the last has L rows, and the last one's length never enters)
// `ext` (optional) adds a base to every prefix / suffix: the sum of n_ext
// states [n_ext][nseq][d][dv] (row-major fp32) of the parts of the sequence
// before (mode 0) or after (mode 1) this one. `f4_layout` says the chunk
// states are in the tensor-core layout (state_f4: float4 j of row r at j*d + r).
// ----------------------------------------------------------------------------
__device__ __forceinline__ int64_t state_row_major_index(int e, int d, int dv, int f4_layout) {
  if (!f4_layout) return e;
  const int f4 = e >> 2, j = f4 / d, r = f4 - j * d;
  return static_cast<int64_t>(r) * dv + 4 * j + (e & 3);
}

__global__ void __launch_bounds__(kSimtThreads)
chunk_scan_kernel(float* __restrict__ s, int64_t C, int nel, int mode, const float* __restrict__ ext,
                  int64_t n_ext, int64_t nseq, int d, int dv, int f4_layout,
                  const float* __restrict__ lam, int H, int64_t L) {
  pdl_launch_dependents();
  pdl_wait();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nel) return;
  float* p = s + (int64_t)blockIdx.y * C * nel + e;
  if (mode == 3 || mode == 4) {
    const float f = powf(lam[blockIdx.y % H], static_cast<float>(L));
    float run = 0.f;
    for (int64_t i = 0; i < C; ++i) {
      const int64_t c = mode == 3 ? i : C - 1 - i;
      const float x = p[c * nel];
      p[c * nel] = run;
      run = fmaf(f, run, x);
    }
    return;
  }
  constexpr int U = 8;  // independent loads in flight per thread
  float run = 0.f;
  if (ext) {
    const int64_t rm = state_row_major_index(e, d, dv, f4_layout);
    for (int64_t i = 0; i < n_ext; ++i) run += ext[(i * nseq + blockIdx.y) * nel + rm];
  }
  if (mode == 2) {
    for (int64_t c0 = 0; c0 < C; c0 += U) {
      float x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) x[u] = c0 + u < C ? p[(c0 + u) * nel] : 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) run += x[u];
    }
    p[0] = run;
    return;
  }
  for (int64_t i0 = 0; i0 < C; i0 += U) {
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u;
      const int64_t c = mode == 0 ? i : C - 1 - i;
      x[u] = i < C ? p[c * nel] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u;
      const int64_t c = mode == 0 ? i : C - 1 - i;
      if (i < C) p[c * nel] = run;
      run += x[u];
    }
  }
}

// Shared-memory helpers: load `rows` rows of a [*, w] tile, zero the rest.
// Tiles stay in the input type T (fp32 inputs: fp32; bf16 inputs: bf16);
// every product is accumulated in fp32.
template <typename T>
__device__ __forceinline__ void load_tile(T* dst, const T* src, int rows, int Bk, int w) {
  for (int i = threadIdx.x; i < Bk * w; i += blockDim.x) {
    const int r = i / w;
    dst[i] = r < rows ? src[i] : from_f32<T>(0.f);
  }
}

__device__ __forceinline__ void load_state(float* dst, const float* src, int nel) {
  for (int i = threadIdx.x; i < nel; i += blockDim.x) dst[i] = src ? src[i] : 0.f;
}

// ----------------------------------------------------------------------------
// Forward block loop (CUDA cores). Per block i of the chunk:
//   O_i = ((Q_i K_i^T) ⊙ M_B) V_i + Q_i KV ;  KV += K_i^T V_i
// Non-causal: O_i = Q_i T with T the total K^T V of the sequence.
// Shared memory: KV [d][dv], Q [Bk][d], K [Bk][d], V [Bk][dv], S [Bk][Bk].
// ----------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                T* __restrict__ o, const float* __restrict__ states, int64_t N, int d, int dv,
                int Bk, int64_t L, int64_t C, int causal, int H, int G, const float* __restrict__ lam) {
  extern __shared__ float smem[];
  float* KV = smem;
  T* Qs = reinterpret_cast<T*>(KV + d * dv);
  T* Ks = Qs + Bk * d;
  T* Vs = Ks + Bk * d;
  T* S = Vs + Bk * dv;  // masked (Q K^T) block, rounded to T
  float* pw = reinterpret_cast<float*>(S + Bk * Bk);  // decayed form: lam^0 .. lam^Bk
  const bool dec = lam != nullptr;
  const int64_t unit = blockIdx.x;
  const int64_t bh = unit / C, c = unit % C;
  const int64_t bkv = kv_seq(bh, H, G);  // K/V sequence (and its states)
  const int64_t t0 = c * L, t1 = imin64(N, t0 + L);
  const T* qb = q + bh * N * d;
  const T* kb = k + bkv * N * d;
  const T* vb = v + bkv * N * dv;
  T* ob = o + bh * N * dv;
  const int64_t nel = (int64_t)d * dv;
  const float* init = nullptr;
  if (!causal) init = states + bkv * C * nel;           // total in slot 0
  else if (states) init = states + (bkv * C + c) * nel;  // exclusive prefix
  load_state(KV, init, (int)nel);
  if (dec)
    for (int i = threadIdx.x; i <= Bk; i += blockDim.x) pw[i] = powf(lam[bh % H], static_cast<float>(i));

  for (int64_t i0 = t0; i0 < t1; i0 += Bk) {
    const int rows = (int)imin64(Bk, t1 - i0);
    load_tile(Qs, qb + i0 * d, rows, Bk, d);
    if (causal) {
      load_tile(Ks, kb + i0 * d, rows, Bk, d);
      load_tile(Vs, vb + i0 * dv, rows, Bk, dv);
    }
    __syncthreads();
    if (causal) {
      for (int i = threadIdx.x; i < Bk * Bk; i += blockDim.x) {
        const int t = i / Bk, j = i % Bk;
        float s = 0.f;
        if (j <= t)
          for (int cc = 0; cc < d; ++cc) s = fmaf(to_f32(Qs[t * d + cc]), to_f32(Ks[j * d + cc]), s);
        if (dec && j <= t) s *= pw[t - j];
        S[i] = from_f32<T>(s);  // M_B: lower-triangular ones, diagonal kept (D_B when decayed)
      }
      __syncthreads();
    }
    for (int i = threadIdx.x; i < rows * dv; i += blockDim.x) {
      const int t = i / dv, e = i % dv;
      float acc = 0.f;
      if (causal)
        for (int j = 0; j <= t; ++j) acc = fmaf(to_f32(S[t * Bk + j]), to_f32(Vs[j * dv + e]), acc);
      if (dec) {
        float x = 0.f;
        for (int cc = 0; cc < d; ++cc) x = fmaf(to_f32(Qs[t * d + cc]), KV[cc * dv + e], x);
        acc = fmaf(pw[t + 1], x, acc);
      } else {
        for (int cc = 0; cc < d; ++cc) acc = fmaf(to_f32(Qs[t * d + cc]), KV[cc * dv + e], acc);
      }
      ob[(i0 + t) * dv + e] = from_f32<T>(acc);
    }
    __syncthreads();
    if (causal) {
      for (int i = threadIdx.x; i < d * dv; i += blockDim.x) {
        const int cc = i / dv, e = i % dv;
        float acc = dec ? pw[rows] * KV[i] : KV[i];
        if (dec)
          for (int t = 0; t < rows; ++t)
            acc = fmaf(pw[rows - 1 - t] * to_f32(Ks[t * d + cc]), to_f32(Vs[t * dv + e]), acc);
        else
          for (int t = 0; t < rows; ++t) acc = fmaf(to_f32(Ks[t * d + cc]), to_f32(Vs[t * dv + e]), acc);
        KV[i] = acc;
      }
      __syncthreads();
    }
  }
}

// ----------------------------------------------------------------------------
// Backward, dQ pass (blocks ascending, state KV = sum_{j<i} K_j^T V_j):
//   dQ_i = ((dO_i V_i^T) ⊙ M_B) K_i + dO_i KV^T ;  KV += K_i^T V_i
// Non-causal: dQ_i = dO_i T^T with T = K^T V over the whole sequence.
// Shared memory: KV [d][dv], dO [Bk][dv], V [Bk][dv], K [Bk][d], A [Bk][Bk].
// ----------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
bwd_dq_simt_kernel(const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ dout,
                   T* __restrict__ dq, const float* __restrict__ states, int64_t N, int d, int dv,
                   int Bk, int64_t L, int64_t C, int causal, int H, int G,
                   const float* __restrict__ lam) {
  extern __shared__ float smem[];
  float* KV = smem;
  T* dOs = reinterpret_cast<T*>(KV + d * dv);
  T* Vs = dOs + Bk * dv;
  T* Ks = Vs + Bk * dv;
  T* A = Ks + Bk * d;  // masked (dO V^T) block, rounded to T
  float* pw = reinterpret_cast<float*>(A + Bk * Bk);  // decayed form: lam^0 .. lam^Bk
  const bool dec = lam != nullptr;
  const int64_t unit = blockIdx.x;
  const int64_t bh = unit / C, c = unit % C;
  const int64_t bkv = kv_seq(bh, H, G);
  const int64_t t0 = c * L, t1 = imin64(N, t0 + L);
  const T* kb = k + bkv * N * d;
  const T* vb = v + bkv * N * dv;
  const T* gb = dout + bh * N * dv;
  T* dqb = dq + bh * N * d;
  const int64_t nel = (int64_t)d * dv;
  const float* init = nullptr;
  if (!causal) init = states + bkv * C * nel;
  else if (states) init = states + (bkv * C + c) * nel;
  load_state(KV, init, (int)nel);
  if (dec)
    for (int i = threadIdx.x; i <= Bk; i += blockDim.x) pw[i] = powf(lam[bh % H], static_cast<float>(i));

  for (int64_t i0 = t0; i0 < t1; i0 += Bk) {
    const int rows = (int)imin64(Bk, t1 - i0);
    load_tile(dOs, gb + i0 * dv, rows, Bk, dv);
    if (causal) {
      load_tile(Vs, vb + i0 * dv, rows, Bk, dv);
      load_tile(Ks, kb + i0 * d, rows, Bk, d);
    }
    __syncthreads();
    if (causal) {
      for (int i = threadIdx.x; i < Bk * Bk; i += blockDim.x) {
        const int t = i / Bk, j = i % Bk;
        float s = 0.f;
        if (j <= t)
          for (int e = 0; e < dv; ++e) s = fmaf(to_f32(dOs[t * dv + e]), to_f32(Vs[j * dv + e]), s);
        if (dec && j <= t) s *= pw[t - j];
        A[i] = from_f32<T>(s);
      }
      __syncthreads();
    }
    for (int i = threadIdx.x; i < rows * d; i += blockDim.x) {
      const int t = i / d, cc = i % d;
      float acc = 0.f;
      if (causal)
        for (int j = 0; j <= t; ++j) acc = fmaf(to_f32(A[t * Bk + j]), to_f32(Ks[j * d + cc]), acc);
      if (dec) {
        float x = 0.f;
        for (int e = 0; e < dv; ++e) x = fmaf(to_f32(dOs[t * dv + e]), KV[cc * dv + e], x);
        acc = fmaf(pw[t + 1], x, acc);
      } else {
        for (int e = 0; e < dv; ++e) acc = fmaf(to_f32(dOs[t * dv + e]), KV[cc * dv + e], acc);
      }
      dqb[(i0 + t) * d + cc] = from_f32<T>(acc);
    }
    __syncthreads();
    if (causal) {
      for (int i = threadIdx.x; i < d * dv; i += blockDim.x) {
        const int cc = i / dv, e = i % dv;
        float acc = dec ? pw[rows] * KV[i] : KV[i];
        if (dec)
          for (int t = 0; t < rows; ++t)
            acc = fmaf(pw[rows - 1 - t] * to_f32(Ks[t * d + cc]), to_f32(Vs[t * dv + e]), acc);
        else
          for (int t = 0; t < rows; ++t) acc = fmaf(to_f32(Ks[t * d + cc]), to_f32(Vs[t * dv + e]), acc);
        KV[i] = acc;
      }
      __syncthreads();
    }
  }
}

// ----------------------------------------------------------------------------
// Backward, dK/dV pass (blocks descending, state U = sum_{l>i} Q_l^T dO_l):
//   dK_i = ((dO_i V_i^T) ⊙ M_B)^T Q_i + V_i U^T
//   dV_i = ((Q_i K_i^T) ⊙ M_B)^T dO_i + K_i U ;  U += Q_i^T dO_i
// Non-causal: dK_i = V_i U^T, dV_i = K_i U with U = Q^T dO over the sequence.
// One CTA per (K/V sequence, chunk). With grouped heads (G > 1) the causal
// terms add up over the group's query heads and U sums all of them (one state
// for the group). Each thread accumulates strips of 32 columns of one row of
// dK_i and dV_i in registers (at most two strips of each; the host keeps
// Bk * ceil(d / 32) and Bk * ceil(dv / 32) within 2 * kSimtThreads).
// Shared memory: U [d][dv], Q, K [Bk][d], V, dO [Bk][dv], A, P [Bk][Bk].
// ----------------------------------------------------------------------------
constexpr int kStrip = 32;
constexpr int kStripsPerThread = 2;

// acc[c] (+)= sum over t in [t_lo, rows) of W[t * Bk + j] * X[t * w + c0 + c]
template <typename T>
__device__ __forceinline__ void strip_masked(float (&acc)[kStrip], const T* W, const T* X, int j, int c0,
                                             int w, int rows, int Bk) {
  for (int t = j; t < rows; ++t) {
    const float a = to_f32(W[t * Bk + j]);
    const T* x = X + t * w + c0;
#pragma unroll
    for (int c = 0; c < kStrip; ++c)
      if (c0 + c < w) acc[c] = fmaf(a, to_f32(x[c]), acc[c]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
bwd_dkdv_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const T* __restrict__ dout, T* __restrict__ dk, T* __restrict__ dvv,
                     const float* __restrict__ states, int64_t N, int d, int dv, int Bk,
                     int64_t L, int64_t C, int causal, int H, int G, const float* __restrict__ lam) {
  extern __shared__ float smem[];
  float* U = smem;
  T* Qs = reinterpret_cast<T*>(U + d * dv);
  T* Ks = Qs + Bk * d;
  T* Vs = Ks + Bk * d;
  T* dOs = Vs + Bk * dv;
  T* A = dOs + Bk * dv;  // masked (dO V^T) block, rounded to T
  T* P = A + Bk * Bk;    // masked (Q K^T) block, rounded to T
  float* pw = reinterpret_cast<float*>(P + Bk * Bk);  // decayed form (one head a sequence): lam^0..lam^Bk
  const bool dec = lam != nullptr;
  const int64_t unit = blockIdx.x;
  const int64_t bh = unit / C, c = unit % C;  // the K/V sequence
  const int64_t t0 = c * L, t1 = imin64(N, t0 + L);
  const int64_t q0 = q_seq0(bh, H, G);
  const int heads = causal ? G : 1;
  const T* kb = k + bh * N * d;
  const T* vb = v + bh * N * dv;
  T* dkb = dk + bh * N * d;
  T* dvb = dvv + bh * N * dv;
  const int64_t nel = (int64_t)d * dv;
  const float* init = nullptr;
  if (!causal) init = states + bh * C * nel;
  else if (states) init = states + (bh * C + c) * nel;  // exclusive suffix
  load_state(U, init, (int)nel);
  if (dec)
    for (int i = threadIdx.x; i <= Bk; i += blockDim.x) pw[i] = powf(lam[bh % H], static_cast<float>(i));
  // strips: dK strip s = (row s / sk, columns 32 * (s % sk)), likewise dV
  const int sk = (d + kStrip - 1) / kStrip, sv = (dv + kStrip - 1) / kStrip;

  const int64_t nblk = (t1 - t0 + Bk - 1) / Bk;
  for (int64_t bi = nblk - 1; bi >= 0; --bi) {
    const int64_t i0 = t0 + bi * Bk;
    const int rows = (int)imin64(Bk, t1 - i0);
    load_tile(Ks, kb + i0 * d, rows, Bk, d);
    load_tile(Vs, vb + i0 * dv, rows, Bk, dv);
    __syncthreads();
    // the later blocks' part, from U before this block's update:
    // dK[j][cc] = sum_e V[j][e] U[cc][e],  dV[j][e] = sum_cc K[j][cc] U[cc][e]
    float ak[kStripsPerThread][kStrip], av[kStripsPerThread][kStrip];
#pragma unroll
    for (int r = 0; r < kStripsPerThread; ++r) {
      const int sid = threadIdx.x + r * kSimtThreads;
      const int j = sid / sk, c0 = (sid % sk) * kStrip;
#pragma unroll
      for (int cc = 0; cc < kStrip; ++cc) ak[r][cc] = 0.f;
      if (j < rows) {
        for (int e = 0; e < dv; ++e) {
          const float x = to_f32(Vs[j * dv + e]);
#pragma unroll
          for (int cc = 0; cc < kStrip; ++cc)
            if (c0 + cc < d) ak[r][cc] = fmaf(x, U[(c0 + cc) * dv + e], ak[r][cc]);
        }
        if (dec)
#pragma unroll
          for (int cc = 0; cc < kStrip; ++cc) ak[r][cc] *= pw[rows - j];
      }
    }
#pragma unroll
    for (int r = 0; r < kStripsPerThread; ++r) {
      const int sid = threadIdx.x + r * kSimtThreads;
      const int j = sid / sv, e0 = (sid % sv) * kStrip;
#pragma unroll
      for (int e = 0; e < kStrip; ++e) av[r][e] = 0.f;
      if (j < rows) {
        for (int cc = 0; cc < d; ++cc) {
          const float x = to_f32(Ks[j * d + cc]);
#pragma unroll
          for (int e = 0; e < kStrip; ++e)
            if (e0 + e < dv) av[r][e] = fmaf(x, U[cc * dv + e0 + e], av[r][e]);
        }
        if (dec)
#pragma unroll
          for (int e = 0; e < kStrip; ++e) av[r][e] *= pw[rows - j];
      }
    }
    for (int g = 0; causal && g < heads; ++g) {
      const int64_t hq = q0 + g;
      __syncthreads();  // U read above (g = 0) or Q, dO of the previous head done with
      load_tile(Qs, q + hq * N * d + i0 * d, rows, Bk, d);
      load_tile(dOs, dout + hq * N * dv + i0 * dv, rows, Bk, dv);
      __syncthreads();
      for (int i = threadIdx.x; i < Bk * Bk; i += blockDim.x) {
        const int t = i / Bk, j = i % Bk;  // t: query row, j: key row
        float a = 0.f, p = 0.f;
        if (j <= t) {
          for (int e = 0; e < dv; ++e) a = fmaf(to_f32(dOs[t * dv + e]), to_f32(Vs[j * dv + e]), a);
          for (int cc = 0; cc < d; ++cc) p = fmaf(to_f32(Qs[t * d + cc]), to_f32(Ks[j * d + cc]), p);
        }
        if (dec && j <= t) {
          a *= pw[t - j];
          p *= pw[t - j];
        }
        A[i] = from_f32<T>(a);
        P[i] = from_f32<T>(p);
      }
      __syncthreads();
      // dK[j] += sum_{t >= j} A[t][j] Q[t],  dV[j] += sum_{t >= j} P[t][j] dO[t]
#pragma unroll
      for (int r = 0; r < kStripsPerThread; ++r) {
        const int sid = threadIdx.x + r * kSimtThreads;
        const int j = sid / sk;
        if (j < rows) strip_masked(ak[r], A, Qs, j, (sid % sk) * kStrip, d, rows, Bk);
      }
#pragma unroll
      for (int r = 0; r < kStripsPerThread; ++r) {
        const int sid = threadIdx.x + r * kSimtThreads;
        const int j = sid / sv;
        if (j < rows) strip_masked(av[r], P, dOs, j, (sid % sv) * kStrip, dv, rows, Bk);
      }
      for (int i = threadIdx.x; i < d * dv; i += blockDim.x) {
        const int cc = i / dv, e = i % dv;
        float acc = dec ? pw[rows] * U[i] : U[i];
        if (dec)
          for (int t = 0; t < rows; ++t)
            acc = fmaf(pw[t] * to_f32(Qs[t * d + cc]), to_f32(dOs[t * dv + e]), acc);
        else
          for (int t = 0; t < rows; ++t) acc = fmaf(to_f32(Qs[t * d + cc]), to_f32(dOs[t * dv + e]), acc);
        U[i] = acc;
      }
    }
#pragma unroll
    for (int r = 0; r < kStripsPerThread; ++r) {
      const int sid = threadIdx.x + r * kSimtThreads;
      const int j = sid / sk, c0 = (sid % sk) * kStrip;
      if (j < rows)
#pragma unroll
        for (int cc = 0; cc < kStrip; ++cc)
          if (c0 + cc < d) dkb[(i0 + j) * d + c0 + cc] = from_f32<T>(ak[r][cc]);
    }
#pragma unroll
    for (int r = 0; r < kStripsPerThread; ++r) {
      const int sid = threadIdx.x + r * kSimtThreads;
      const int j = sid / sv, e0 = (sid % sv) * kStrip;
      if (j < rows)
#pragma unroll
        for (int e = 0; e < kStrip; ++e)
          if (e0 + e < dv) dvb[(i0 + j) * dv + e0 + e] = from_f32<T>(av[r][e]);
    }
    __syncthreads();  // K, V, U settled before the next block's loads
  }
}

// Strips of 32 columns the dK/dV loop keeps per block: every one must have a
// thread (at most kStripsPerThread each).
inline bool bwd_dkdv_simt_fits(int d, int dv, int Bk) {
  const int strips = Bk * ((std::max(d, dv) + kStrip - 1) / kStrip);
  return strips <= kStripsPerThread * kSimtThreads;
}

// (`decay`: plus the table lam^0 .. lam^Bk)
inline size_t fwd_simt_smem(int d, int dv, int Bk, size_t es, bool decay = false) {
  return sizeof(float) * (size_t)d * dv + es * ((size_t)Bk * (2 * d + dv) + (size_t)Bk * Bk) +
         (decay ? sizeof(float) * (Bk + 1) : 0);
}
inline size_t bwd_dq_simt_smem(int d, int dv, int Bk, size_t es, bool decay = false) {
  return sizeof(float) * (size_t)d * dv + es * ((size_t)Bk * (2 * dv + d) + (size_t)Bk * Bk) +
         (decay ? sizeof(float) * (Bk + 1) : 0);
}
inline size_t bwd_dkdv_simt_smem(int d, int dv, int Bk, size_t es, bool decay = false) {
  return sizeof(float) * (size_t)d * dv + es * ((size_t)Bk * (2 * d + 2 * dv) + 2 * (size_t)Bk * Bk) +
         (decay ? sizeof(float) * (Bk + 1) : 0);
}
inline size_t chunk_state_smem(int da, int db) {
  return sizeof(float) * (size_t)kStateRowsPerTile * (da + db);
}

}  // namespace la2

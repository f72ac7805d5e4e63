// decode.cu -- one decoding step: the newest token's query over the
// structured key set of its position.
//
// For the query at position i = T - 1 (its own key and value are the last
// cache entry) the kept keys are the same disjoint parts as in prefill
// ("LM-Infinite", section 方法: the starting span and the recent window;
// "SepLLM", section 五.2: every earlier separator): sinks j < n_start,
// window max(n_start, i - w) <= j <= i, separators n_start <= j < i - w.
// A key farther than L_pretrain takes the capped logit <R(L) q, k_j> with
// the unrotated key, the others <R(i) q, R(j) k_j>.
//
// Split-K over the kept keys (memory-bound: each kept K and V row is read
// once): a CTA takes a chunk of kChunk kept keys of one (batch, kv head) for
// all query heads of that kv head's group; each warp walks its keys with the
// head dimension spread over the lanes (a lane owns rotary pairs
// c = PPL*lane .. PPL*lane + PPL - 1 and their partners c + d/2), loads kU
// keys' K, V and rotary entries before using any of them, and keeps an
// online softmax per query head.  The chunk's (max, sum, unnormalised O)
// per head go to the workspace; a second kernel merges the chunks.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 128;  // kept keys per CTA
constexpr int kU = 4;        // keys per warp whose loads are in flight together

struct KeySet {
  int n_sink, win_lo, n_win, n_sep;
  __device__ __forceinline__ int n() const { return n_sink + n_win + n_sep; }
};

// cache length of sequence b: the per-sequence length when given (a
// streaming cache), else T
__device__ __forceinline__ int cache_len(const DecodeArgs& a, int b) { return a.seq_len ? a.seq_len[b] : a.T; }

__device__ __forceinline__ KeySet key_set(const DecodeArgs& a, int b) {
  KeySet s;
  const int Tb = cache_len(a, b);
  const int i = Tb - 1;
  s.n_sink = min(a.n_start, Tb);
  s.win_lo = max(s.n_sink, i - a.window);
  s.n_win = max(0, i - s.win_lo + 1);
  const int thr = i - a.window;  // separators kept: n_start <= j < i - w
  s.n_sep = (a.sep_prefix && thr > 0) ? a.sep_prefix[(size_t)b * (a.T + 1) + min(thr, a.T)] : 0;
  return s;
}

__device__ __forceinline__ int key_at(const DecodeArgs& a, const KeySet& s, int b, int e) {
  if (e < s.n_sink) return e;
  e -= s.n_sink;
  if (e < s.n_win) return s.win_lo + e;
  return a.sep_pos[(size_t)b * a.T + (e - s.n_win)];
}

// grid (ceil(T / kChunk), B * Hkv)
template <int D, int REP>
__global__ void __launch_bounds__(kThreads) decode_partial_kernel(DecodeArgs a) {
  constexpr int half = D / 2;
  constexpr int PPL = half / 32;  // rotary pairs per lane: 2 (d = 128) or 1 (d = 64)
  __shared__ float red_m[kThreads / 32][REP];
  __shared__ float red_l[kThreads / 32][REP];
  __shared__ float red_o[kThreads / 32][REP][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.y;
  const int g = bg % a.Hkv, b = bg / a.Hkv;
  const KeySet ks = key_set(a, b);
  const int e_begin = blockIdx.x * kChunk;
  if (e_begin >= ks.n()) return;  // this batch has fewer chunks
  const int e_end = min(ks.n(), e_begin + kChunk);
  const int i = cache_len(a, b) - 1;
  const int c0 = PPL * lane;

  // the query of each head of the group, rotated to i (qi) and to the cap (qc), fp32
  float qi0[REP][PPL], qi1[REP][PPL], qc0[REP][PPL], qc1[REP][PPL];
#pragma unroll
  for (int r = 0; r < REP; ++r) {
    const int h = g * REP + r;
    const __nv_bfloat16* qp = a.Q + (size_t)b * a.q_sb + (size_t)h * a.q_sh;
#pragma unroll
    for (int e = 0; e < PPL; ++e) {
      const int c = c0 + e;
      const float x0 = __bfloat162float(qp[c]), x1 = __bfloat162float(qp[c + half]);
      const float2 ti = a.tab ? a.tab[(size_t)i * half + c] : make_float2(1.f, 0.f);
      const float2 tl = (a.tab && a.L > 0) ? a.tab[(size_t)a.L * half + c] : make_float2(1.f, 0.f);
      qi0[r][e] = x0 * ti.x - x1 * ti.y;
      qi1[r][e] = x1 * ti.x + x0 * ti.y;
      qc0[r][e] = x0 * tl.x - x1 * tl.y;
      qc1[r][e] = x1 * tl.x + x0 * tl.y;
    }
  }
  float m[REP], l[REP], o0[REP][PPL], o1[REP][PPL];
#pragma unroll
  for (int r = 0; r < REP; ++r) {
    m[r] = -CUDART_INF_F;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < PPL; ++e) o0[r][e] = o1[r][e] = 0.f;
  }
  const __nv_bfloat16* kb = a.K + (size_t)b * a.k_sb + (size_t)g * a.k_sh;
  const __nv_bfloat16* vb = a.V + (size_t)b * a.v_sb + (size_t)g * a.v_sh;
  const float sl2 = a.scale_log2;

  // warp w takes keys e_begin + w, + 4, ... of the chunk
  for (int e0 = e_begin + warp; e0 < e_end; e0 += (kThreads / 32) * kU) {
    int jj[kU];
    float k0[kU][PPL], k1[kU][PPL], v0[kU][PPL], v1[kU][PPL], cs[kU][PPL], sn[kU][PPL];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int e = e0 + u * (kThreads / 32);
      jj[u] = (e < e_end) ? key_at(a, ks, b, e) : -1;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int j = jj[u] < 0 ? 0 : jj[u];
      const __nv_bfloat16* kp = kb + (size_t)j * a.k_st;
      const __nv_bfloat16* vp = vb + (size_t)j * a.v_st;
#pragma unroll
      for (int e = 0; e < PPL; ++e) {
        k0[u][e] = __bfloat162float(kp[c0 + e]);
        k1[u][e] = __bfloat162float(kp[c0 + e + half]);
        v0[u][e] = __bfloat162float(vp[c0 + e]);
        v1[u][e] = __bfloat162float(vp[c0 + e + half]);
        const float2 t = a.tab ? a.tab[(size_t)j * half + c0 + e] : make_float2(1.f, 0.f);
        cs[u][e] = t.x;
        sn[u][e] = t.y;
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (jj[u] < 0) continue;  // uniform over the warp
      const bool capped = a.L > 0 && (i - jj[u]) > a.L;
      float z[REP];
#pragma unroll
      for (int r = 0; r < REP; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < PPL; ++e) {
          if (capped) {
            acc = fmaf(qc0[r][e], k0[u][e], fmaf(qc1[r][e], k1[u][e], acc));
          } else {
            const float kr0 = k0[u][e] * cs[u][e] - k1[u][e] * sn[u][e];
            const float kr1 = k1[u][e] * cs[u][e] + k0[u][e] * sn[u][e];
            acc = fmaf(qi0[r][e], kr0, fmaf(qi1[r][e], kr1, acc));
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        z[r] = acc * sl2;
        if (a.alibi) {  // -m_h * min(i - j, L), in log2 units of the scaled logit
          const int dist = (a.L > 0) ? min(i - jj[u], a.L) : (i - jj[u]);
          z[r] -= exp2f(-8.f * (float)(g * REP + r + 1) / (float)a.Hq) * 1.4426950408889634f * (float)dist;
        }
      }
#pragma unroll
      for (int r = 0; r < REP; ++r) {
        const float m_new = fmaxf(m[r], z[r]);
        const float alpha = ex2_approx(m[r] - m_new);  // 0 on the first key (m = -inf)
        const float p = ex2_approx(z[r] - m_new);
        l[r] = l[r] * alpha + p;
#pragma unroll
        for (int e = 0; e < PPL; ++e) {
          o0[r][e] = fmaf(o0[r][e], alpha, p * v0[u][e]);
          o1[r][e] = fmaf(o1[r][e], alpha, p * v1[u][e]);
        }
        m[r] = m_new;
      }
    }
  }
  // merge the four warps of the CTA
#pragma unroll
  for (int r = 0; r < REP; ++r) {
    if (lane == 0) {
      red_m[warp][r] = m[r];
      red_l[warp][r] = l[r];
    }
#pragma unroll
    for (int e = 0; e < PPL; ++e) {
      red_o[warp][r][c0 + e] = o0[r][e];
      red_o[warp][r][c0 + e + half] = o1[r][e];
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < REP * D; x += kThreads) {
    const int r = x / D, c = x % D;
    float M = -CUDART_INF_F;
    for (int w = 0; w < kThreads / 32; ++w) M = fmaxf(M, red_m[w][r]);
    float L = 0.f, O = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) {
      const float f = (red_m[w][r] == -CUDART_INF_F) ? 0.f : ex2_approx(red_m[w][r] - M);
      L += red_l[w][r] * f;
      O += red_o[w][r][c] * f;
    }
    const int h = g * REP + r;
    float* part = a.part + (((size_t)b * a.Hq + h) * a.n_chunks + blockIdx.x) * (D + 2);
    part[2 + c] = O;
    if (c == 0) {
      part[0] = M;
      part[1] = L;
    }
  }
}

// grid (B * Hq), D threads: merge the chunks of one (batch, head)
template <int D>
__global__ void decode_combine_kernel(DecodeArgs a) {
  const int bh = blockIdx.x;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const KeySet ks = key_set(a, b);
  const int nc = (ks.n() + kChunk - 1) / kChunk;
  const float* part = a.part + (size_t)bh * a.n_chunks * (D + 2);
  const int c = threadIdx.x;
  float M = -CUDART_INF_F;
  for (int x = 0; x < nc; ++x) M = fmaxf(M, part[x * (D + 2)]);
  float L = 0.f, O = 0.f;
  for (int x = 0; x < nc; ++x) {
    const float mx = part[x * (D + 2)];
    const float f = (mx == -CUDART_INF_F) ? 0.f : ex2_approx(mx - M);
    L += part[x * (D + 2) + 1] * f;
    O += part[x * (D + 2) + 2 + c] * f;
  }
  __nv_bfloat16* op = a.O + (size_t)b * a.o_sb + (size_t)h * a.o_sh;
  op[c] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
  if (c == 0) a.lse[bh] = (L > 0.f) ? (M + __log2f(L)) * 0.69314718055994531f : -CUDART_INF_F;
}

template <int D, int REP>
cudaError_t launch_dr(const DecodeArgs& a, cudaStream_t st) {
  dim3 grid(a.n_chunks, a.B * a.Hkv);
  decode_partial_kernel<D, REP><<<grid, kThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<D><<<a.B * a.Hq, D, 0, st>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t st) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_dr<D, 1>(a, st);
    case 2: return launch_dr<D, 2>(a, st);
    case 4: return launch_dr<D, 4>(a, st);
    case 8: return launch_dr<D, 8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int decode_chunks(int T) { return (T + kChunk - 1) / kChunk; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  if (a.d == 128) return launch_d<128>(a, st);
  if (a.d == 64) return launch_d<64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn

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
// all query heads of that kv head's group; each warp walks its 32 keys with
// the head dimension spread over the lanes (a lane owns rotary pairs
// c = PPL*lane .. PPL*lane + PPL - 1 and their partners c + d/2), first the
// logits (several keys' K rows and rotary entries loaded before any is
// used), then, with the chunk's per-head maximum known, the weighted V rows.
// The chunk's (max, sum, unnormalised O) per head go to the workspace; a
// second kernel merges the chunks.
#include <algorithm>

#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "select.cuh"
#include "simt.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 128;  // kept keys per CTA

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
  s.n_sep = (a.sep_words && thr > 0) ? sep_before(a.sep_words, a.T, b, thr) : 0;
  return s;
}

__device__ __forceinline__ int key_at(const DecodeArgs& a, const KeySet& s, int b, int e) {
  if (e < s.n_sink) return e;
  e -= s.n_sink;
  if (e < s.n_win) return s.win_lo + e;
  return a.sep_pos[(size_t)b * a.T + (e - s.n_win)];
}

// grid (B * Hkv, chunks): the (batch, kv head) index varies fastest, so the
// chunks that hold keys (the low ones) are dispatched before the empty ones.
//
// A key is spread over LPK lanes (8, or 16 for eight query heads per kv
// head), each holding EPL rotary pairs (16 or 8 elements of the row), so a
// warp works on 32 / LPK keys at once with 16-byte loads.  Two passes over
// the CTA's chunk of kept keys: (1) logits -- the raw key rotated on the fly
// to R(j) k_j, or for a capped key (i - j > L) to R(i - L) k_j, which gives
// the capped logit <R(L) q, k_j> = <R(i) q, R(i - L) k_j> with the one query
// R(i) q; the lanes' partial dot products of all heads summed by one
// transposed butterfly over the key's lanes; logits to shared memory; (2)
// with the chunk's per-head maximum and the weights p = 2^(z - m) taken once
// per (key, head): O += p v.  No running rescale.
// Lane layout of the logit pass.  A key is spread over LPK lanes (8, or 16
// for eight query heads per kv head), each holding EPL rotary pairs (16 or 8
// elements of the row), so a warp works on 32 / LPK keys at once with
// 16-byte loads; KPW key slots per warp, UNR warp steps in flight.
template <int D, int REP>
struct Tiling {
  static constexpr int half = D / 2;
  static constexpr int LPK = (REP >= 8) ? 16 : 8;       // lanes per key
  static constexpr int KPS = 32 / LPK;                  // keys per warp step
  static constexpr int EPL = half / LPK;                // rotary pairs per lane
  static constexpr int KPW = kChunk / (kThreads / 32);  // keys per warp: 32
  static constexpr int UNR = (REP >= 4) ? 1 : 2;        // warp steps whose loads are in flight together
  static_assert(REP <= LPK && KPW % (KPS * UNR) == 0 && (EPL == 8 || EPL == 4 || EPL == 2), "decode tiling");
};

// EPL consecutive bf16 as floats (16, 8 or 4 bytes)
template <int EPL>
__device__ __forceinline__ void load_e(const __nv_bfloat16* p, float* out) {
  if constexpr (EPL == 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const float2 f = __bfloat1622float2(h[y]);
      out[2 * y] = f.x;
      out[2 * y + 1] = f.y;
    }
  } else if constexpr (EPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int y = 0; y < 2; ++y) {
      const float2 f = __bfloat1622float2(h[y]);
      out[2 * y] = f.x;
      out[2 * y + 1] = f.y;
    }
  } else {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    out[0] = f.x;
    out[1] = f.y;
  }
}

// This lane's pairs [p0, p0 + EPL) of the query of each head of kv group g,
// rotated to i, in fp32.
template <int D, int REP>
__device__ __forceinline__ void rotated_query(const DecodeArgs& a, int b, int g, int i, int p0,
                                              float (&q0)[REP][Tiling<D, REP>::EPL],
                                              float (&q1)[REP][Tiling<D, REP>::EPL]) {
  constexpr int half = D / 2, EPL = Tiling<D, REP>::EPL;
#pragma unroll
  for (int r = 0; r < REP; ++r) {
    const __nv_bfloat16* qp = a.Q + (size_t)b * a.q_sb + (size_t)(g * REP + r) * a.q_sh;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float x0 = __bfloat162float(qp[p0 + e]), x1 = __bfloat162float(qp[p0 + e + half]);
      const float2 t = a.tab ? a.tab[(size_t)i * half + p0 + e] : make_float2(1.f, 0.f);
      q0[r][e] = x0 * t.x - x1 * t.y;
      q1[r][e] = x1 * t.x + x0 * t.y;
    }
  }
}

// The logit pass over one warp's KPW key slots [w_lo, w_lo + KPW): the raw
// key rotated on the fly to R(j) k_j, or for a capped key (i - j > L) to
// R(i - L) k_j, which gives the capped logit <R(L) q, k_j> = <R(i) q,
// R(i - L) k_j> with the one query R(i) q; the lanes' partial dot products
// of all heads summed by one transposed butterfly over the key's lanes.
// key_of(slot) gives the slot's key position (-1: none); emit(r, slot, j,
// dot) receives head r's unscaled logit on one lane per (key, head).
template <int D, int REP, class KeyOf, class Emit>
__device__ __forceinline__ void logits_pass(const DecodeArgs& a, int i, const __nv_bfloat16* kb, int w_lo,
                                            int lane, const float (&q0)[REP][Tiling<D, REP>::EPL],
                                            const float (&q1)[REP][Tiling<D, REP>::EPL], KeyOf key_of,
                                            Emit emit) {
  using TL = Tiling<D, REP>;
  constexpr int half = D / 2, LPK = TL::LPK, KPS = TL::KPS, EPL = TL::EPL, KPW = TL::KPW, UNR = TL::UNR;
  const int sub = lane % LPK, kg = lane / LPK;
  const int p0 = sub * EPL;
  for (int u0 = 0; u0 < KPW; u0 += KPS * UNR) {
    int jj[UNR];
    float k0[UNR][EPL], k1[UNR][EPL];
    float2 cs[UNR][EPL];
#pragma unroll
    for (int x = 0; x < UNR; ++x) {
      jj[x] = key_of(w_lo + u0 + x * KPS + kg);
      const int j = jj[x] < 0 ? 0 : jj[x];
      const int rpos = (a.L > 0 && i - j > a.L) ? i - a.L : j;  // capped keys: R(i - L) k_j
      load_e<EPL>(kb + (size_t)j * a.k_st + p0, k0[x]);
      load_e<EPL>(kb + (size_t)j * a.k_st + p0 + half, k1[x]);
      if (a.tab) {
        const float4* tp = reinterpret_cast<const float4*>(a.tab + (size_t)rpos * half + p0);
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
          const float4 t = tp[e / 2];
          cs[x][e] = make_float2(t.x, t.y);
          cs[x][e + 1] = make_float2(t.z, t.w);
        }
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) cs[x][e] = make_float2(1.f, 0.f);
      }
    }
#pragma unroll
    for (int x = 0; x < UNR; ++x) {
      float v[REP];
#pragma unroll
      for (int r = 0; r < REP; ++r) v[r] = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const float kr0 = k0[x][e] * cs[x][e].x - k1[x][e] * cs[x][e].y;
        const float kr1 = k1[x][e] * cs[x][e].x + k0[x][e] * cs[x][e].y;
#pragma unroll
        for (int r = 0; r < REP; ++r) v[r] = fmaf(q0[r][e], kr0, fmaf(q1[r][e], kr1, v[r]));
      }
      group_reduce_transposed<REP, LPK>(v, 0xffffffffu, lane);
      // lane sub now holds head sub / (LPK / REP)
      constexpr int DUP = LPK / REP;
      if (sub % DUP == 0) emit(sub / DUP, w_lo + u0 + x * KPS + kg, jj[x], v[0]);
    }
  }
}

// grid (B * Hkv, chunks): the (batch, kv head) index varies fastest, so the
// chunks that hold keys (the low ones) are dispatched before the empty ones.
// Two passes over the CTA's chunk of kept keys: (1) logits (logits_pass) to
// shared memory; (2) with the chunk's per-head maximum and the weights
// p = 2^(z - m) taken once per (key, head): O += p v.  No running rescale.
template <int D, int REP>
__global__ void __launch_bounds__(kThreads) decode_partial_kernel(DecodeArgs a) {
  using TL = Tiling<D, REP>;
  constexpr int half = D / 2, LPK = TL::LPK, KPS = TL::KPS, EPL = TL::EPL, KPW = TL::KPW, UNR = TL::UNR;
  __shared__ float s_p[REP][kChunk];            // logits, then weights
  __shared__ float s_m[REP], s_l[REP];
  __shared__ float red_o[kThreads / 32][REP][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPK, kg = lane / LPK;
  const int bg = blockIdx.x;
  const int g = bg % a.Hkv, b = bg / a.Hkv;
  const KeySet ks = key_set(a, b);
  const int e_begin = blockIdx.y * kChunk;
  if (e_begin >= ks.n()) return;  // this batch has fewer chunks
  const int n_here = min(ks.n() - e_begin, kChunk);
  const int i = cache_len(a, b) - 1;
  const int p0 = sub * EPL;  // this lane's pairs [p0, p0 + EPL)
  float q0[REP][EPL], q1[REP][EPL];
  rotated_query<D, REP>(a, b, g, i, p0, q0, q1);
  const __nv_bfloat16* kb = a.K + (size_t)b * a.k_sb + (size_t)g * a.k_sh;
  const __nv_bfloat16* vb = a.V + (size_t)b * a.v_sb + (size_t)g * a.v_sh;
  const float sl2 = a.scale_log2;
  const int w_lo = warp * KPW;

  // ---- pass 1: logits ----
  logits_pass<D, REP>(
      a, i, kb, w_lo, lane, q0, q1,
      [&](int el) { return el < n_here ? key_at(a, ks, b, e_begin + el) : -1; },
      [&](int r, int el, int j, float dot) {
        float z = dot * sl2;
        if (a.alibi && j >= 0) {  // -m_h * min(i - j, L), in log2 units of the scaled logit
          const int dist = (a.L > 0) ? min(i - j, a.L) : (i - j);
          z -= exp2f(-8.f * (float)(g * REP + r + 1) / (float)a.Hq) * 1.4426950408889634f * (float)dist;
        }
        s_p[r][el] = (j >= 0) ? z : -CUDART_INF_F;
      });
  __syncthreads();
  // ---- per-head maximum, weights and their sum (warp r takes heads r, r + 4, ...) ----
  for (int r = warp; r < REP; r += kThreads / 32) {
    float mx = -CUDART_INF_F;
    for (int e = lane; e < kChunk; e += 32) mx = fmaxf(mx, s_p[r][e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int e = lane; e < kChunk; e += 32) {
      const float p = (mx == -CUDART_INF_F) ? 0.f : ex2_approx(s_p[r][e] - mx);
      s_p[r][e] = p;
      sum += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      s_m[r] = mx;
      s_l[r] = sum;
    }
  }
  __syncthreads();
  // ---- pass 2: O += p v ----
  float o0[REP][EPL], o1[REP][EPL];
#pragma unroll
  for (int r = 0; r < REP; ++r)
#pragma unroll
    for (int e = 0; e < EPL; ++e) o0[r][e] = o1[r][e] = 0.f;
  for (int u0 = 0; u0 < KPW; u0 += KPS * UNR) {
    float v0[UNR][EPL], v1[UNR][EPL];
    int els[UNR];
#pragma unroll
    for (int x = 0; x < UNR; ++x) {
      els[x] = w_lo + u0 + x * KPS + kg;
      const int j = (els[x] < n_here) ? key_at(a, ks, b, e_begin + els[x]) : 0;
      load_e<EPL>(vb + (size_t)j * a.v_st + p0, v0[x]);
      load_e<EPL>(vb + (size_t)j * a.v_st + p0 + half, v1[x]);
    }
#pragma unroll
    for (int x = 0; x < UNR; ++x) {
#pragma unroll
      for (int r = 0; r < REP; ++r) {
        const float p = s_p[r][els[x]];  // 0 for keys past the chunk's end
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          o0[r][e] = fmaf(p, v0[x][e], o0[r][e]);
          o1[r][e] = fmaf(p, v1[x][e], o1[r][e]);
        }
      }
    }
  }
  // merge the warp's key slots (lanes sub, sub + LPK, ...), then the warps (fixed order)
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1)
#pragma unroll
    for (int r = 0; r < REP; ++r)
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        o0[r][e] += __shfl_xor_sync(0xffffffffu, o0[r][e], o);
        o1[r][e] += __shfl_xor_sync(0xffffffffu, o1[r][e], o);
      }
  if (kg == 0) {
#pragma unroll
    for (int r = 0; r < REP; ++r)
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        red_o[warp][r][p0 + e] = o0[r][e];
        red_o[warp][r][p0 + e + half] = o1[r][e];
      }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < REP * D; x += kThreads) {
    const int r = x / D, c = x % D;
    float O = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) O += red_o[w][r][c];
    const int h = g * REP + r;
    float* part = a.part + (((size_t)b * a.Hq + h) * a.n_chunks + blockIdx.y) * (D + 2);
    part[2 + c] = O;
    if (c == 0) {
      part[0] = s_m[r];
      part[1] = s_l[r];
    }
  }
}

// ---------------------------------------------------------------------------
// top-k middle tokens of the decoding query ("LM-Infinite", section 方法,
// optional top-k): candidates n_start <= j < i - w that are not separators,
// ranked per query head by the unscaled logit (the capped one past L), ties
// to the smaller position.  Reading every candidate key is what the method
// asks for here; the K rows are read once per kv group.
// ---------------------------------------------------------------------------

// grid (B * Hkv, candidate chunks of kChunk positions): every candidate's
// logit for every query head of the group (the logit pass over consecutive
// positions), then per head the chunk's k best (separators excluded by
// their flag bit) into tk_cz / tk_cj: the top k of the whole row is the top
// k of the chunks' top k, so the selection merges k entries per chunk
// rather than every candidate.
template <int D, int REP>
__global__ void __launch_bounds__(kThreads) decode_topk_logits_kernel(DecodeArgs a) {
  using TL = Tiling<D, REP>;
  constexpr int EPL = TL::EPL, LPK = TL::LPK, KPW = TL::KPW;
  __shared__ float s_z[REP][kChunk];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x % a.Hkv, b = blockIdx.x / a.Hkv;
  const int i = a.T - 1;
  const int jend = i - a.window;  // candidates j < i - w
  const int j0 = a.n_start + blockIdx.y * kChunk;
  if (j0 >= jend) return;
  const int p0 = (lane % LPK) * EPL;
  float q0[REP][EPL], q1[REP][EPL];
  rotated_query<D, REP>(a, b, g, i, p0, q0, q1);
  const __nv_bfloat16* kb = a.K + (size_t)b * a.k_sb + (size_t)g * a.k_sh;
  const uint2* words = a.sep_words ? a.sep_words + (size_t)b * (a.T / 32 + 1) : nullptr;
  logits_pass<D, REP>(
      a, i, kb, warp * KPW, lane, q0, q1, [&](int el) { return j0 + el < jend ? j0 + el : -1; },
      [&](int r, int el, int j, float dot) {
        const bool sep = j >= 0 && words && ((__ldg(&words[j >> 5].y) >> (j & 31)) & 1u);
        s_z[r][el] = (j >= 0 && !sep) ? dot : -CUDART_INF_F;
      });
  __syncthreads();
  // per head: k rounds of a warp argmax by (z desc, j asc) over the chunk
  // (lane l holds keys l, l + 32, l + 64, l + 96)
  const int k = a.topk;
  const int chunk = blockIdx.y;
  for (int r = warp; r < REP; r += kThreads / 32) {
    float zv[kChunk / 32];
    int jv[kChunk / 32];
#pragma unroll
    for (int u = 0; u < kChunk / 32; ++u) {
      const int el = lane + 32 * u;
      zv[u] = s_z[r][el];
      jv[u] = (zv[u] == -CUDART_INF_F) ? -1 : j0 + el;
    }
    const size_t base = (((size_t)b * a.Hq + (size_t)g * REP + r) * a.tk_nchunks + chunk) * k;
    for (int y = 0; y < k; ++y) {
      float bz = -CUDART_INF_F;
      int bj = -1;
#pragma unroll
      for (int u = 0; u < kChunk / 32; ++u)
        if (sel_before(zv[u], jv[u], bz, bj)) {
          bz = zv[u];
          bj = jv[u];
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (sel_before(oz, oj, bz, bj)) {
          bz = oz;
          bj = oj;
        }
      }
#pragma unroll
      for (int u = 0; u < kChunk / 32; ++u)
        if (jv[u] == bj && bj >= 0) {  // the winner leaves its list (positions are distinct)
          jv[u] = -1;
          zv[u] = -CUDART_INF_F;
        }
      if (lane == 0) {
        a.tk_cz[base + y] = bj >= 0 ? bz : -CUDART_INF_F;
        a.tk_cj[base + y] = bj;
      }
    }
  }
}

constexpr int kSelThreads = 512;
constexpr int kSelMaxK = 16;

// grid (B * Hq): the k best candidates of one (batch, head) from the chunks'
// top k -- a strided pass keeping a sorted list per thread, then k rounds of
// a block argmax -- written out, and the selected keys' softmax partial
// (their maximum, sum of weights and weighted V rows) for the chunk merge.
template <int D>
__global__ void __launch_bounds__(kSelThreads) decode_topk_select_kernel(DecodeArgs a) {
  __shared__ float red_z[kSelThreads / 32];
  __shared__ int red_j[kSelThreads / 32];
  __shared__ float s_z[kSelMaxK];
  __shared__ int s_j[kSelMaxK];
  const int bh = blockIdx.x;
  const int b = bh / a.Hq, h = bh % a.Hq, g = h / (a.Hq / a.Hkv);
  const int n_c = a.tk_nchunks * a.topk;  // the chunks' picks (-1 padding)
  const float* czr = a.tk_cz + (size_t)bh * n_c;
  const int32_t* cjr = a.tk_cj + (size_t)bh * n_c;
  float vals[kSelMaxK];
  int idxs[kSelMaxK];
#pragma unroll
  for (int y = 0; y < kSelMaxK; ++y) {
    vals[y] = -CUDART_INF_F;
    idxs[y] = -1;
  }
  // each thread visits its entries in increasing position order (chunks in
  // order, each chunk's picks by (z desc, j asc) but a thread sees one
  // chunk's entries a stride apart), so ties are settled by position
  for (int e = (int)threadIdx.x; e < n_c; e += kSelThreads) {
    const int j = cjr[e];
    if (j < 0) continue;
    const float z = czr[e];
    if (sel_before(z, j, vals[kSelMaxK - 1], idxs[kSelMaxK - 1])) {
      float v = z;
      int jj = j;
#pragma unroll
      for (int y = 0; y < kSelMaxK; ++y) {
        if (sel_before(v, jj, vals[y], idxs[y])) {
          const float tv = vals[y];
          const int tj = idxs[y];
          vals[y] = v;
          idxs[y] = jj;
          v = tv;
          jj = tj;
        }
      }
    }
  }
  block_topk_rounds<kSelMaxK>(a.topk, vals, idxs, red_z, red_j, [&](int r, float wz, int wj) {
    s_j[r] = wj;
    s_z[r] = wj >= 0 ? wz : -CUDART_INF_F;
  });
  __syncthreads();
  const int k = a.topk;
  if ((int)threadIdx.x < k) {
    a.tk_idx[(size_t)bh * k + threadIdx.x] = s_j[threadIdx.x];
    a.tk_z[(size_t)bh * k + threadIdx.x] = s_z[threadIdx.x];
  }
  // scaled log2-unit logits of the picks; with ALiBi every candidate is
  // past the cap (w >= L) and takes -m_h L
  const float sl2 = a.scale_log2;
  const float bias = a.alibi ? exp2f(-8.f * (float)(h + 1) / (float)a.Hq) * 1.4426950408889634f * (float)a.L : 0.f;
  float m = -CUDART_INF_F;
  for (int r = 0; r < k; ++r)
    if (s_j[r] >= 0) m = fmaxf(m, s_z[r] * sl2 - bias);
  float* part = a.tk_part + (size_t)bh * (D + 2);
  const __nv_bfloat16* vb = a.V + (size_t)b * a.v_sb + (size_t)g * a.v_sh;
  for (int c = threadIdx.x; c < D; c += kSelThreads) {
    float l = 0.f, o = 0.f;
    for (int r = 0; r < k; ++r) {
      if (s_j[r] < 0) continue;
      const float p = ex2_approx(s_z[r] * sl2 - bias - m);
      l += p;
      o = fmaf(p, __bfloat162float(vb[(size_t)s_j[r] * a.v_st + c]), o);
    }
    part[2 + c] = o;
    if (c == 0) {
      part[0] = m;
      part[1] = l;
    }
  }
}

// grid (B * Hq), 4 D threads: merge the chunks of one (batch, head).  The
// chunk maxima and weights are read in parallel into shared memory; thread
// group q of 4 sums chunks q, q + 4, ... of each output column (independent
// loads), then the four groups are added in a fixed order.
constexpr int kCombineGroups = 4;
constexpr int kCombineMaxChunks = 4096;
template <int D>
__global__ void __launch_bounds__(kCombineGroups * D) decode_combine_kernel(DecodeArgs a) {
  __shared__ float s_f[kCombineMaxChunks + 1];
  __shared__ float s_red[kCombineGroups * D];
  __shared__ float s_ml[2];
  const int bh = blockIdx.x;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const KeySet ks = key_set(a, b);
  const int nc0 = min((ks.n() + kChunk - 1) / kChunk, kCombineMaxChunks);
  // the chunks' partials, then the top-k keys' one
  const int nc = nc0 + (a.tk_part ? 1 : 0);
  const float* part0 = a.part + (size_t)bh * a.n_chunks * (D + 2);
  auto slot = [&](int x) { return x < nc0 ? part0 + (size_t)x * (D + 2) : a.tk_part + (size_t)bh * (D + 2); };
  const int tid = threadIdx.x;
  float mx = -CUDART_INF_F;
  for (int x = tid; x < nc; x += blockDim.x) {
    s_f[x] = slot(x)[0];
    mx = fmaxf(mx, s_f[x]);
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) s_red[tid >> 5] = mx;
  __syncthreads();
  if (tid == 0) {
    float M = -CUDART_INF_F;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) M = fmaxf(M, s_red[w]);
    s_ml[0] = M;
  }
  __syncthreads();
  const float M = s_ml[0];
  float lsum = 0.f;
  for (int x = tid; x < nc; x += blockDim.x) {
    const float f = (s_f[x] == -CUDART_INF_F) ? 0.f : ex2_approx(s_f[x] - M);
    s_f[x] = f;
    lsum += slot(x)[1] * f;
  }
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  __syncthreads();  // s_red is reused
  if ((tid & 31) == 0) s_red[tid >> 5] = lsum;
  __syncthreads();
  if (tid == 0) {
    float L = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) L += s_red[w];
    s_ml[1] = L;
  }
  const int q = tid / D, c = tid % D;
  float O = 0.f;
#pragma unroll 4
  for (int x = q; x < nc; x += kCombineGroups) O = fmaf(slot(x)[2 + c], s_f[x], O);
  __syncthreads();
  s_red[q * D + c] = O;
  __syncthreads();
  if (q == 0) {
    float Ot = 0.f;
    for (int y = 0; y < kCombineGroups; ++y) Ot += s_red[y * D + c];
    const float L = s_ml[1];
    __nv_bfloat16* op = a.O + (size_t)b * a.o_sb + (size_t)h * a.o_sh;
    op[c] = __float2bfloat16_rn(L > 0.f ? Ot / L : 0.f);
    if (c == 0) a.lse[bh] = (L > 0.f) ? (M + __log2f(L)) * 0.69314718055994531f : -CUDART_INF_F;
  }
}

template <int D, int REP>
cudaError_t launch_dr(const DecodeArgs& a, cudaStream_t st) {
  // without separators or per-sequence lengths the kept-key count is a
  // closed form: launch exactly its chunks
  int chunks = a.n_chunks;
  if (!a.sep_words && !a.seq_len) {
    const int i = a.T - 1, ns = std::min(a.n_start, a.T);
    const int win_lo = std::max(ns, i - a.window);
    chunks = std::min(chunks, std::max(1, (ns + std::max(0, i - win_lo + 1) + kChunk - 1) / kChunk));
  }
  cudaError_t e;
  if (a.topk > 0) {
    const int ncand = a.T - 1 - a.window - a.n_start;
    if (ncand > 0) {
      dim3 gt(a.B * a.Hkv, a.tk_nchunks);
      decode_topk_logits_kernel<D, REP><<<gt, kThreads, 0, st>>>(a);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    decode_topk_select_kernel<D><<<a.B * a.Hq, kSelThreads, 0, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  dim3 grid(a.B * a.Hkv, chunks);
  decode_partial_kernel<D, REP><<<grid, kThreads, 0, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<D><<<a.B * a.Hq, kCombineGroups * D, 0, st>>>(a);
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
int decode_topk_chunks(int n_candidates) { return n_candidates > 0 ? (n_candidates + kChunk - 1) / kChunk : 0; }
int decode_max_len() { return kCombineMaxChunks * kChunk; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  if (a.d == 128) return launch_d<128>(a, st);
  if (a.d == 64) return launch_d<64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn

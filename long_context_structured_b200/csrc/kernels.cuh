// kernels.cuh -- launch interfaces of the library's kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sattn {

constexpr int kTile = 128;  // query-tile rows (BM) and key-tile columns (BN)
constexpr int kMaxHeads = 256;

// ---------------------------------------------------------------------------
// K1: rotary table and the prep pass
// ---------------------------------------------------------------------------
// tab[p][c] = (cos, sin)(p * scale * theta^(-2c/d)), computed in fp64, stored
// fp32; scale < 1 is position interpolation.
cudaError_t launch_rope_table(float2* tab, int npos, int d, double theta, double scale, cudaStream_t st);
// rows [0, n_low) and [row_lo, npos) only (the others are not written)
cudaError_t launch_rope_table_rows(float2* tab, int npos, int d, double theta, double scale, int n_low, int row_lo,
                                   cudaStream_t st);

struct PrepArgs {
  int B, Hq, Hkv, T, d;
  const void* Q;  // bf16 or fp32 per `f32`
  const void* K;
  int64_t q_sb, q_sh, q_st, k_sb, k_sh, k_st;
  bool f32;
  const float2* tab;  // nullptr: no rotation
  int L;              // distance cap (0 = none)
  __nv_bfloat16* Qr;  // [B,Hq,T,d] R(i) q_i            (may be null)
  __nv_bfloat16* Qc;  // [B,Hq,T,d] R(L) q_i            (may be null)
  __nv_bfloat16* Kr;  // [B,Hkv,T,d] R(j) k_j           (may be null)
  float* sink_z;      // [B,Hq,T,n_sink] side logits    (may be null)
  int n_sink;
  int alibi;          // nonzero: sink logits carry the clipped ALiBi bias (in q.k units)
  uint32_t* kmax;     // [B*Hkv] max_j ||k_j|| as float bits (may be null)
  // input row r is position pos0 + r (no sink logits then); Kr holds
  // kr_rows rows per (b, kv head) (0: T) and row r goes to row kr_row0 + r
  int pos0, kr_rows, kr_row0;
  const int32_t* status;  // when not null: nothing is written once it reports a failure
};
cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st);

// ---------------------------------------------------------------------------
// K2: block map
// ---------------------------------------------------------------------------
struct BlockmapArgs {
  int B, T, n_start, window;
  const uint8_t* is_sep;  // may be null
  void* scratch;          // blockmap_scratch_bytes(B, T, window) of workspace
  int32_t* sep_pos;       // [B, T]
  int32_t* sep_count;     // [B]
  int32_t* ranges;        // [B, nQT, 2]
  uint8_t* cls;           // [B, nQT, nKT] or null
};
cudaError_t launch_blockmap(const BlockmapArgs& a, cudaStream_t st);
// streaming multiprocessors of the current device (cached per device)
int sm_count();

// scratch of launch_blockmap: word prefix of the separator flags, far and
// near tile classes (0 for invalid sizes)
size_t blockmap_scratch_bytes(int B, int T, int window);

// The separator word prefix, the first part of the block map's scratch: per
// sequence T/32 + 1 entries; entry x holds in .x the number of separators
// (j >= n_start) before position 32 x and in .y a bit for each of the 32
// positions from 32 x that is one.
// Separators (j >= n_start) before position x, x clamped to [0, T].
__device__ __forceinline__ int sep_before(const uint2* words, int T, int b, int x) {
  x = max(0, min(T, x));
  const uint2 e = __ldg(words + (size_t)b * (T / 32 + 1) + (x >> 5));
  return (int)e.x + __popc(e.y & ((1u << (x & 31)) - 1u));
}

// Bit c (c < 64): position j64 + c (j64 a multiple of 32) is a separator
// j >= n_start with lo <= j64 + c <= hi.
__device__ __forceinline__ uint64_t sep_bits64(const uint2* words, int T, int b, int j64, int lo, int hi) {
  if (hi < lo || hi < j64 || lo > j64 + 63) return 0ull;
  const uint2* wb = words + (size_t)b * (T / 32 + 1);
  const int w0 = j64 >> 5;
  const uint64_t m0 = w0 <= T / 32 ? __ldg(wb + w0).y : 0u;
  const uint64_t m1 = w0 + 1 <= T / 32 ? __ldg(wb + w0 + 1).y : 0u;
  uint64_t m = m0 | m1 << 32;
  const int a = max(0, lo - j64), e = min(63, hi - j64);  // keep bits [a, e]
  m &= (e == 63 ? ~0ull : ((1ull << (e + 1)) - 1ull)) & ~((1ull << a) - 1ull);
  return m;
}

// ---------------------------------------------------------------------------
// K3: separator K/V gather into dense per-(b, kv-head) arrays
// ---------------------------------------------------------------------------
struct GatherArgs {
  int B, Hkv, T, Tpad, d;
  const __nv_bfloat16* Ksrc;
  int64_t k_sb, k_sh, k_st;
  const __nv_bfloat16* Vsrc;
  int64_t v_sb, v_sh, v_st;
  const int32_t* sep_pos;    // [B, T]
  const int32_t* sep_count;  // [B]
  __nv_bfloat16* Ks;         // [B, Hkv, Tpad, d]
  __nv_bfloat16* Vs;
};
cudaError_t launch_sep_gather(const GatherArgs& a, cudaStream_t st);

// ---------------------------------------------------------------------------
// K5: tcgen05 attention
// ---------------------------------------------------------------------------
struct AttnArgs {
  int B, Hq, Hkv, T, d, nQT;
  float scale_log2;  // log2(e) / sqrt(d)
  // band tiles over the main K/V
  int ns_band;       // keys j < ns_band never go through the band (sinks use the side path)
  int w_eff;         // band keeps j >= i - w_eff
  int w_sepband;     // > w_eff: band tiles reach back to i - w_sepband and also keep the separators
                     // with i - w_sepband <= j < i - w_eff (the uncapped ones when the window is
                     // below the cap); 0 otherwise
  // side keys (fp32 logits)
  const float* sink_z;  // [B, Hq, T, n_sink]
  int n_sink;
  const int32_t* tk_idx;  // [B, Hq, T, topk]
  const float* tk_z;
  int topk;
  const __nv_bfloat16* V;  // raw V for side keys
  int64_t v_sb, v_sh, v_st;
  // gathered tiles: 0 none, 1 separators, 2 segmented prefix, 3 cross-attention
  // over a compressed context (every row keeps all cross_len gathered rows)
  int gather_mode;
  int cross_len;
  bool q2;                     // gathered tiles use the second query tile (Qc)
  const int32_t* sep_pos;      // [B, T]
  const uint2* sep_words;      // separator word prefix (sep_before)
  const int32_t* ranges;       // [B, nQT, 2]
  int window;                  // w for the separator rule (sep kept iff pos < i - w)
  // segmented execution
  int seg_S, seg_M, seg_N, seg_R;
  int16_t long_slot[kMaxHeads]; // head -> index among long heads, -1 for local
  const int32_t* prefix_cnt;   // [B, Hl, N - seg_s0] number of prefix keys
  int n_long;
  int seg_s0;                  // prefix planes and counts held for segments seg_s0 .. N-1
  // query rows: row r of the Q / O / LSE tensors is position q_pos0 + r
  // (a multiple of the tile), those tensors hold T_q rows (0: T); keys and
  // masks use positions (T: the sequence so far)
  int q_pos0, T_q;
  // ALiBi: s_ij gets -m_h * min(i - j, L) (L = 0: no clip), m_h = 2^(-8 (h+1) / Hq)
  int alibi, alibi_cap;
  // outputs
  __nv_bfloat16* O;
  int64_t o_sb, o_sh, o_st;
  float* lse;
  int32_t* status;
};
// ALiBi slope of query head h, times sqrt(d): the bias per unit distance in
// units of the unscaled logit q.k
__device__ __forceinline__ float alibi_slope_qk(int h, int Hq, int d) {
  return exp2f(-8.f * (float)(h + 1) / (float)Hq) * sqrtf((float)d);
}
struct AttnMaps {
  CUtensorMap q, q2, k, v, kg, vg;
};
// two query tiles per CTA; not for q2 (capped separator tiles) and, in
// segmented mode, only when the segment length is a multiple of 256
cudaError_t launch_attn_tc2(const AttnArgs& a, const AttnMaps& m, cudaStream_t st);
// one query tile per CTA with the score tile triple-buffered in TMEM; every case
cudaError_t launch_attn_tc3(const AttnArgs& a, const AttnMaps& m, cudaStream_t st);

// ---------------------------------------------------------------------------
// K6: fp32 attention on CUDA cores
// ---------------------------------------------------------------------------
struct AttnF32Args {
  int B, Hq, Hkv, T, d;
  const float* Q;
  const float* K;
  const float* V;
  int64_t q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st;
  const float2* tab;  // null: no rotation
  int L, n_start, window;
  const int32_t* sep_pos;    // [B, T] or null
  const int32_t* sep_count;  // [B]
  const int32_t* tk_idx;     // [B, Hq, T, topk] or null
  const float* tk_z;
  int topk;
  int alibi;                 // ALiBi bias clipped at L (no rotation)
  float* O;
  int64_t o_sb, o_sh, o_st;
  float* lse;
};
cudaError_t launch_attn_f32(const AttnF32Args& a, cudaStream_t st);

// ---------------------------------------------------------------------------
// SharedLLM tree cross-attention: compressed context and rotated queries
// ---------------------------------------------------------------------------
struct TreeArgs {
  int B, Hq, Hkv, Tq, d;            // Tq query rows per (b, h)
  int n_chunks, chunk_len, depth, alpha_leaf, n_kept, Spad;
  const float2* tab;                // rotary table (null: no rotation), positions 0..n_chunks
  const __nv_bfloat16* Q;           // [B, Hq, Tq, d] strided
  int64_t q_sb, q_sh, q_st;
  const __nv_bfloat16* K;           // [B, Hkv, n_chunks * chunk_len, d] strided
  const __nv_bfloat16* V;
  int64_t k_sb, k_sh, k_st, v_sb, v_sh, v_st;
  __nv_bfloat16* Qr;                // [B, Hq, Tq, d]: R(n) q
  __nv_bfloat16* Kt;                // [B, Hkv, Spad, d]: kept keys of chunk c, R(c) k
  __nv_bfloat16* Vt;
  int32_t* kept_index;              // [n_kept] or null: kept offsets within a chunk
};
cudaError_t launch_tree_prep(const TreeArgs& a, cudaStream_t st);
int tree_kept_count(int chunk_len, int depth, int alpha_leaf);  // host; < 0 on bad arguments

// ---------------------------------------------------------------------------
// streaming KV cache (SepLLM's Initial | Separator | Past | Local)
// ---------------------------------------------------------------------------
struct StreamArgs {
  int B, Hkv, d, a, s, w, c;
  int64_t position;                 // stream index of the appended token
  const __nv_bfloat16* K_new;       // [B, Hkv, d]
  const __nv_bfloat16* V_new;
  const uint8_t* sep_new;           // [B] or null
  int32_t* sizes;                   // [B, 4]: Initial, Separator, Past, Local
  int32_t* len;                     // [B] cache length (sum of the sizes)
  int32_t* ctrl;                    // [B, 2]: compacting, slots before the compaction
  int32_t* pos;                     // [B, c] stream index per slot
  uint8_t* flag;                    // [B, c] separator flag per slot
  int32_t* dst;                     // [B, c] compaction destination (-1: dropped)
  __nv_bfloat16* K;                 // [B, Hkv, c, d]
  __nv_bfloat16* V;
  __nv_bfloat16* Ks;                // scratch copies for compaction
  __nv_bfloat16* Vs;
  int32_t* pos_s;
  uint8_t* flag_s;
};
cudaError_t launch_stream_append(const StreamArgs& a, cudaStream_t st);

// ---------------------------------------------------------------------------
// backward pass, fp32 on CUDA cores
// ---------------------------------------------------------------------------
struct BwdF32Args {
  int B, Hq, Hkv, T, d;
  const float* Q;
  const float* K;
  const float* V;
  const float* O;
  const float* dO;           // strides of O
  int64_t q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st, o_sb, o_sh, o_st;
  const float* lse;          // [B, Hq, T] natural log, from the forward
  const float2* tab;         // null: no rotation
  int L, n_start, window;
  const uint8_t* is_sep;     // [B, T] or null
  const int32_t* sep_pos;    // [B, T] or null
  const int32_t* sep_count;  // [B]
  const int32_t* tk_idx;     // [B, Hq, T, topk] or null: the forward's selection
  int topk;
  int alibi;
  float* Dsum;               // [B, Hq, T] workspace: dO_i . O_i
  float* dQ;
  float* dK;
  float* dV;
  int64_t dq_sb, dq_sh, dq_st, dk_sb, dk_sh, dk_st, dv_sb, dv_sh, dv_st;
};
cudaError_t launch_bwd_f32(const BwdF32Args& a, cudaStream_t st);

// ---------------------------------------------------------------------------
// backward pass, bf16 on tensor cores (sinks on CUDA cores)
// ---------------------------------------------------------------------------
struct BwdArgs {
  int B, Hq, Hkv, T, d, nQT, Tpad;
  float scale_log2;             // log2(e) / sqrt(d)
  int n_start, window, L;       // L: distance cap (0 = none)
  int sep_split;                // separators with i - j > sep_split go through the compacted tiles
  int w_sepband;                // > window: band tiles reach back to i - w_sepband for the separators
                                // with window < i - j <= w_sepband; 0 otherwise
  int alibi, alibi_cap;
  const float2* tab;            // rotary table (null: no rotation)
  // the forward's inputs and outputs (raw layouts, explicit strides)
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const __nv_bfloat16* O;
  const __nv_bfloat16* dO;      // strides of O
  int64_t q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st, o_sb, o_sh, o_st;
  const float* lse;             // [B, Hq, T] natural log
  // products of the prep pass
  const __nv_bfloat16* Qr;      // [B, Hq, T, d] R(i) q_i
  const __nv_bfloat16* Qc;      // [B, Hq, T, d] R(L) q_i (capped separators)
  const float* sink_z;          // [B, Hq, T, n_sink] fp32 sink logits (capped rule, ALiBi bias included)
  int n_sink;
  // separators (compacted by the block map)
  int gather;                   // 1: separators present
  int capped_sep;               // gathered tiles take Qc and raw keys
  const int32_t* sep_pos;       // [B, T]
  const int32_t* sep_count;     // [B]
  const uint2* sep_words;       // separator word prefix (sep_before)
  const int32_t* ranges;        // [B, nQT, 2]
  // row statistics, padded to Tpad rows (pad: D = 0, -lse2 = -inf)
  float* Dsum;                  // [B, Hq, Tpad] dO_i . O_i
  float* nlse2;                 // [B, Hq, Tpad] -LSE_i * log2(e)
  // sinks
  float* sink_ds;               // [B, Hq, T, n_sink] dS of the sink pairs (unscaled)
  float* sink_p;                // [B, Hq, T, n_sink] P of the sink pairs
  float* sink_part;             // [B, Hkv, n_sink, nRB, 2, d] partial key-side sums per row block
  int nRB;                      // row blocks of the sink reduction
  // fp32 scratch
  float* dq_side;               // [B, Hq, T, d] dq of the capped separators (raw frame, scaled)
  float* dk_band;               // [B, Hkv, T, d] band-tile dk (raw frame)
  float* dv_band;
  float* dk_sep;                // [B, Hkv, Tpad, d] separator dk, compacted order (raw frame)
  float* dv_sep;
  // outputs (strides of Q, K, V)
  __nv_bfloat16* dQ;
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  int32_t* status;
  int dq_mode;                  // dq kernel: 0 band (+ uncapped separators), 1 capped separators only
  bool side_valid;              // dq_side holds data (else it is not read)
  int fold_sinks;               // dq kernel (mode 0): add the sink pairs' dq from sink_ds and the sink key rows
  // top-k keys (fp32 side keys; the forward's selection is an input)
  int topk;
  const int32_t* tk_idx;        // [B, Hq, T, topk] selected keys (-1: none)
  float* tk_ds;                 // [B, Hq, T, topk] dS of the selected pairs (unscaled)
  float* tk_p;                  // [B, Hq, T, topk] P of the selected pairs
  int* tk_cnt;                  // [B, Hkv, T] selections per key
  int* tk_off;                  // [B, Hkv, T] offset of each key's codes within its (b, kv head) segment
  int* tk_cur;                  // [B, Hkv, T] fill cursors
  int* tk_code;                 // [B, Hkv, rep * T * topk] codes ((local head * T + row) * topk + slot) by key
  int* tk_sorted;               // same layout, each key's codes in ascending order
};
struct BwdMaps {
  CUtensorMap q, qc, dO, k, v, kg, vg;
};
cudaError_t launch_bwd_rows(const BwdArgs& a, cudaStream_t st);
cudaError_t launch_bwd_sink_keys(const BwdArgs& a, cudaStream_t st);
cudaError_t launch_bwd_dq(const BwdArgs& a, const BwdMaps& m, cudaStream_t st);
cudaError_t launch_bwd_dkv(const BwdArgs& a, const BwdMaps& m, cudaStream_t st);
cudaError_t launch_bwd_combine(const BwdArgs& a, cudaStream_t st);
// top-k pairs: the rows' P, dS and dq part (added to dq_side when add_side,
// else written there)
cudaError_t launch_bwd_topk_rows(const BwdArgs& a, bool add_side, cudaStream_t st);
// top-k pairs, key side: dk and dv of every selected key, added to dk_band /
// dv_band in a fixed order (after the dk/dv kernel has written them)
cudaError_t launch_bwd_topk_keys(const BwdArgs& a, cudaStream_t st);
int bwd_sink_row_block();  // rows per partial sum of the sink-key reduction

// ---------------------------------------------------------------------------
// K4: top-k middle-token selection
// ---------------------------------------------------------------------------
struct TopkArgs {
  int B, Hq, Hkv, T, d, nQT;
  int n_start, window, topk, L;
  const uint8_t* is_sep;       // [B, T] or null
  // raw inputs for the exact fp32 re-rank
  const void* Q;
  const void* K;
  bool f32;
  int64_t q_sb, q_sh, q_st, k_sb, k_sh, k_st;
  const float2* tab;           // null: no rotation
  const uint32_t* kmax;        // [B*Hkv] max key norm (float bits)
  int32_t* idx;                // [B, Hq, T, topk]
  float* z;
  int32_t* fallback_rows;      // [B*Hq*T] rows whose bf16 shortlist was not certified
  int32_t* status;             // status[2] counts fallback rows
  // candidates from the tensor-core scoring pass: every key whose coarse
  // score exceeds the row's threshold
  int2* cand_idx;              // [B*Hq*T, kCandCap] (key position, coarse score bits), in key order
  float* cand_thr;             // [B*Hq*T] the row's threshold (-inf: every candidate is listed)
  int32_t* cand_cnt;           // [B*Hq*T] keys above the threshold (> kCandCap: the list overflowed)
};
constexpr int kCandCap = 192;  // list entries per row (a multiple of 32)
struct TopkMaps {
  CUtensorMap qsel, ksel;      // bf16 scoring operands: (Qc, K) capped, (Qr, Kr) otherwise
  CUtensorMap qsel2, ksel2;    // with 0 < window < L: (Qr, Kr) for the pairs within the cap
};
// scoring on the tensor cores into per-row candidate lists
cudaError_t launch_topk_score(const TopkArgs& a, const TopkMaps& m, cudaStream_t st);
// exact re-rank of the lists and certification (uncertified rows are queued
// for launch_topk_exact)
cudaError_t launch_topk_rerank(const TopkArgs& a, cudaStream_t st);
// exact fp32 scan for the rows listed in fallback_rows (count in status[2]),
// or for every row when all_rows is set
cudaError_t launch_topk_exact(const TopkArgs& a, bool all_rows, cudaStream_t st);

// ---------------------------------------------------------------------------
// K7: segmented execution -- retrieval and prefix assembly
// ---------------------------------------------------------------------------
struct SegRetrArgs {
  int B, Hq, Hkv, T, d, S, N, R, blk, n_long;
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int64_t q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st;
  int16_t long_heads[kMaxHeads]; // head id of each long slot
  const float2* tab;
  // segments retrieved: s_lo .. N-1 (s_lo >= 1); the per-segment arrays
  // below hold segments s_base .. N-1 (Ns = N - s_base of them)
  int s_lo, s_base;
  // segment-end query of segment s_lo (q_{s_lo S - 1}) when not null, in
  // place of Q's row (a step that holds only its own segment's queries)
  const __nv_bfloat16* q_end;  // [B, Hq, d]
  int64_t qe_sb, qe_sh;
  int32_t* prefix_blocks;      // [B, Hq, Ns, R/blk] (all heads; -1 filled)
  int32_t* prefix_cnt;         // [B, n_long, Ns]
  __nv_bfloat16* Kpre;         // [B, n_long, Ns, R, d] rotated at virtual positions
  __nv_bfloat16* Vpre;
  float* score;                // [B, n_long, Ns, T / blk] block scores (workspace)
};
// largest shared-memory sort buffer of the block selection (bytes)
constexpr size_t kSegSelectSmemMax = 128 * 1024;
// bytes of the block-score workspace
size_t segment_score_bytes(int B, int n_long, int N, int T, int blk);
// whether the block selection's sort fits in shared memory
bool segment_retrieval_supported(int T, int S, int blk);
cudaError_t launch_segment_retrieval(const SegRetrArgs& a, cudaStream_t st);

// backward of segmented execution (CUDA cores)
struct SegBwdArgs {
  int B, Hq, Hkv, T, d, S, N, M, R, blk;
  float scale_log2;            // log2(e) / sqrt(d)
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const __nv_bfloat16* O;
  const __nv_bfloat16* dO;     // strides of O
  int64_t q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st, o_sb, o_sh, o_st;
  const float* lse;            // [B, Hq, T]
  const int32_t* prefix_blocks;  // [B, Hq, N, R/blk], the forward's retrieval (-1: none)
  int16_t long_slot[kMaxHeads];  // head -> index among long heads, -1 for local
  const float2* tab;           // rotary table over positions [0, T) (null: no rotation)
  float* Dsum;                 // [B, Hq, T] dO_i . O_i
  __nv_bfloat16* dQ;           // strides of Q
  __nv_bfloat16* dK;           // strides of K
  __nv_bfloat16* dV;           // strides of V
  int64_t dq_sb, dq_sh, dq_st, dk_sb, dk_sh, dk_st, dv_sb, dv_sh, dv_st;
};
cudaError_t launch_segment_bwd(const SegBwdArgs& a, cudaStream_t st);

// ---------------------------------------------------------------------------
// segmented execution one segment at a time: the carried state
// ---------------------------------------------------------------------------
struct SegStateArgs {
  int B, Hq, Hkv, d, S, T_cap, seg;
  int32_t* header;              // state header: magic, segments taken, S, T_cap
  const __nv_bfloat16* Q;       // the segment's [B, Hq, S, d]
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int64_t q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st;
  __nv_bfloat16* Khist;         // [B, Hkv, T_cap, d] raw keys of every position taken
  __nv_bfloat16* Vhist;
  __nv_bfloat16* q_end;         // [B, Hq, d] the last segment's last query
  int32_t* status;
};
cudaError_t launch_segstate_reset(int32_t* header, int S, int T_cap, cudaStream_t st);
cudaError_t launch_segstate_append(const SegStateArgs& a, cudaStream_t st);
cudaError_t launch_segstate_finish(const SegStateArgs& a, cudaStream_t st);

// ---------------------------------------------------------------------------
// decoding step: one query per (batch, head) at position T - 1
// ---------------------------------------------------------------------------
struct DecodeArgs {
  int B, Hq, Hkv, T, d;
  int n_start, window, L;
  float scale_log2;
  const __nv_bfloat16* Q;  // [B, Hq, 1, d]
  int64_t q_sb, q_sh;
  const __nv_bfloat16* K;  // [B, Hkv, T, d] cache, unrotated
  int64_t k_sb, k_sh, k_st;
  const __nv_bfloat16* V;
  int64_t v_sb, v_sh, v_st;
  // rotation (rope != 0): pair c at position p rotates by the angle p * rope_scale * inv_freq[c]
  int rope;
  double rope_scale;
  double inv_freq[64];          // theta^(-2c/d), c < d/2
  float2 step_cs[64];           // (cos, sin) of the rotation by KPS positions (set by the launcher)
  float turn_hi[64], turn_lo[64];  // turns per position of pair c, as hi + lo (set by the launcher)
  const uint2* sep_words;       // separator word prefix (sep_before) or null (no separators)
  const int32_t* sep_pos;       // [B, T]
  const int32_t* seq_len;       // [B] cache length per sequence (<= T), or null: T for all
  float* part;                  // [B, Hq, n_chunks, d + 2] chunk partials
  int32_t* status;              // the workspace's status word (a wait that gave up)
  int alibi;                    // ALiBi bias clipped at L (no rotation)
  int n_chunks;
  // top-k middle tokens of the query (topk > 0; seq_len must be null)
  int topk;
  int tk_nchunks;                // candidate chunks of 128 positions (decode_topk_chunks)
  float* tk_cz;                 // [B, Hq, tk_nchunks, topk] each chunk's best logits (unscaled)
  int32_t* tk_cj;               // [B, Hq, tk_nchunks, topk] their positions (-1 padding)
  int32_t* tk_idx;              // [B, Hq, topk] the selection (-1 padding)
  float* tk_z;                  // [B, Hq, topk] its logits (-inf padding)
  float* tk_part;               // [B, Hq, d + 2] the selected keys' partial (max, sum, O)
  __nv_bfloat16* O;             // [B, Hq, 1, d]
  int64_t o_sb, o_sh;
  float* lse;                   // [B, Hq]
};
// chunks of kept keys a decoding step of cache length T may need
int decode_chunks(int T);
int decode_topk_chunks(int n_candidates);  // candidate chunks of the top-k logit pass
int decode_max_len();  // longest key set one decoding step merges
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);

}  // namespace sattn

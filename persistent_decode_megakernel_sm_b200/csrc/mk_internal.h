// mk_internal.h - structures shared by the host planner and the persistent
// kernel.  Nothing here is part of the public ABI.
#pragma once
#include <stdint.h>

namespace mk {

// ---------------------------------------------------------------------------
// kernel geometry
// ---------------------------------------------------------------------------
constexpr int NCW = 8;                       // consumer warps
constexpr int WARP_WP = NCW;                 // weight producer warp
constexpr int WARP_XP = NCW + 1;             // activation producer warp
constexpr int WARP_MV = NCW + 2;             // tensor-memory mover warp
constexpr int NTHREADS = (NCW + 3) * 32;
constexpr int NCT = NCW * 32;                // consumer threads
// Ring shape (tunable at build time).
#ifndef MK_TILE_CAP
#define MK_TILE_CAP 65536
#endif
#ifndef MK_NSTAGE
#define MK_NSTAGE 2
#endif
// Second weight stage in tensor memory (TMEM, 256 KB per SM): bf16 GEMV
// chunks are copied out of the shared-memory ring into TMEM slots as soon as
// they land, which frees the ring for the next bulk copies; the consumers read
// their mma A fragments from TMEM.  The producer can then run up to NSTAGE +
// NTS chunks ahead of the consumers.  0 keeps every chunk in shared memory.
#ifndef MK_TSLOTS
#define MK_TSLOTS 0
#endif
constexpr int TILE_CAP = MK_TILE_CAP;        // weight tile bytes per GEMV chunk (gains follow)
constexpr int NTS = MK_TSLOTS;               // TMEM slots
constexpr int TSLOT_COLS = TILE_CAP / 512;   // TMEM columns per slot: 4 columns (16 B x 128 lanes) hold 4 tiles
constexpr int TMEM_COLS = 512;               // the whole tensor memory of the SM (one CTA per SM)
static_assert(NTS * TSLOT_COLS <= TMEM_COLS, "TMEM slots exceed the tensor memory");
// Cache positions per GQA attention chunk: 64 or 128 (K and V of a head_dim
// 128 chunk fill 32 or 64 KB of one stage).
#ifndef MK_ATT_CT
#define MK_ATT_CT 128
#endif
constexpr int ATT_CT = MK_ATT_CT;
static_assert(ATT_CT == 64 || ATT_CT == 128, "attention chunks of 64 or 128 positions");
constexpr int STAGE_BYTES = (TILE_CAP > 2 * ATT_CT * 128 * 2) ? TILE_CAP : 2 * ATT_CT * 128 * 2;
constexpr int NSTAGE = MK_NSTAGE;            // weight ring depth
constexpr int XSLOTS = 2;                    // activation ring depth
constexpr int XSLOT_BYTES = 22528;           // one activation window: M rows x (cols + pad)
constexpr int XROW_PAD = 32;                 // bytes between activation rows (bank spread)
constexpr int ATT_BYTES = 40960;             // GEMV reduction / attention scratch
constexpr int NEWKV_BYTES = 8704;            // K/V rows of the step's own new positions
constexpr int MISC_BYTES = 4096;
constexpr int SMEM_BYTES = NSTAGE * STAGE_BYTES + XSLOTS * XSLOT_BYTES + ATT_BYTES + NEWKV_BYTES + MISC_BYTES;
#ifndef MK_RMAX
#define MK_RMAX 8
#endif
constexpr int RMAX = MK_RMAX;                // row tiles per chunk (4 or 8)
static_assert(RMAX == 4 || RMAX == 8, "row tiles per chunk: 4 or 8");
// Most col tiles per warp in one GEMV chunk; the ring stage and the
// activation window cap a chunk too.  16 lets a one-row group at B = 1 fill
// a whole 64 KB stage (128 bf16 col tiles) instead of half of one.
#ifndef MK_CPW
#define MK_CPW 16
#endif
constexpr int CPW = MK_CPW;
constexpr int MAXM = 8;                      // activation rows per step (S * Q)
static_assert(2 * ATT_CT * 128 * 2 <= STAGE_BYTES, "a K/V chunk of head_dim 128 fills at most one stage");
constexpr int TRACE_FIELDS = 20;             // int64 per traced task
constexpr int TILE_BF16 = 512;               // 16x16 bf16 tile in A-fragment order
constexpr int TILE_FP8 = 256;                // 16x16 e4m3 tile in A-fragment order

// GQA K / V rows (head_dim bf16 values) are stored with their 16-byte groups
// permuted by the position: group c of the row at position pos sits at
// group c ^ (pos & 7).  A chunk of consecutive rows, copied to shared memory
// as one block, then spreads any 8 consecutive rows' accesses to one group
// over all banks.  Element index of dim e of the row at position pos:
__host__ __device__ inline int kv_swz(int pos, int e) { return (((e >> 3) ^ (pos & 7)) << 3) | (e & 7); }

// Latent attention (MLA) items use the activation ring, the attention scratch
// and the new-KV rows as one contiguous shared-memory region: while a CTA runs
// a latent-attention item its activation producer is parked on the next
// task's dependency (the per-head value projection, which waits for every
// attention item of the layer), so the activation ring is idle.
constexpr int MLA_SCRATCH_BYTES = XSLOTS * XSLOT_BYTES + ATT_BYTES + NEWKV_BYTES;

// One latent cache row [c (R) | k_rope (dr)] bf16 in shared memory, padded by
// 16 bytes so that the 8 rows of an mma fragment load hit distinct banks.
__host__ __device__ inline int mla_pitch(int R, int dr) { return (R + dr) * 2 + 16; }
// Cache positions per streamed chunk (one ring stage, a multiple of 8, <= 64).
__host__ __device__ inline int mla_ct(int R, int dr) {
  int n = STAGE_BYTES / mla_pitch(R, dr);
  n = n > 64 ? 64 : n;
  return n & ~7;
}
// Byte offsets inside the latent-attention scratch: query A fragments (hi, lo
// bf16 parts), probability A fragments for <= 64 positions (hi, lo), per-warp
// row maxima (two parities), the step's own new latent rows (<= MAXM).
struct MlaLayout {
  int qhi, qlo, phi, plo, smax, newr, total;
};
__host__ __device__ inline MlaLayout mla_layout(int Hq, int R, int dr) {
  const int mt = (Hq + 15) / 16, KW = (R + dr) / 16;
  MlaLayout L;
  L.qhi = 0;
  L.qlo = mt * KW * 512;
  L.phi = 2 * mt * KW * 512;
  L.plo = L.phi + mt * 4 * 512;
  L.smax = L.plo + mt * 4 * 512;
  L.newr = L.smax + 2 * NCW * 32 * 4;
  L.total = L.newr + MAXM * mla_pitch(R, dr);
  return L;
}
__host__ __device__ inline int mla_smem_need(int Hq, int R, int dr) { return mla_layout(Hq, R, dr).total; }

// ---------------------------------------------------------------------------
// tasks
// ---------------------------------------------------------------------------
enum TaskType : int16_t {
  T_GEMV = 1,      // out rows [rt0, rt1) of a matrix
  T_ATTN = 2,      // one split-KV attention item (GQA)
  T_MOE_GU = 3,    // expert gate/up row tiles (shared: static; routed: union of the router's picks)
  T_MOE_DOWN = 4,  // down projection, K = shared + selected experts' hidden units
  T_PREFETCH = 5,  // weight producer only: bring row tiles [rt0, rt1) of matrix `m` into L2 ahead of their task
  T_EMBED = 6,     // x[m][c0:c1) = embedding rows of the step's tokens (+ RMS partial sums)
  T_MLA = 7,       // one split-KV latent-attention item (one query row, all heads)
  T_MLA_COMB = 8,  // this CTA's slice of the latent-attention split combine
};

enum InKind : int16_t {
  IN_X_NORM = 0,   // residual x [M][H] with RMSNorm (scales from per-CTA partial sums)
  IN_EMB_NORM = 1, // embedding rows of the tokens, RMSNorm computed in the prologue
  IN_BUF = 2,      // plain fp32 buffer [M][ld]
};

enum Epi : int16_t {
  EPI_STORE = 0,       // out[m][row] = v
  EPI_RESID = 1,       // x[m][row] += v (+ per-CTA sums of squares)
  EPI_SWIGLU = 2,      // tile rows 0..7 gate, 8..15 up: h[m][i] = silu(g) u
  EPI_LOGITS = 3,      // logits + per-CTA argmax partial
  EPI_SWIGLU_MOE = 4,  // expert slot s: h[s][m][i] = w(s, m) silu(g) u
};

enum BufId : int16_t {
  B_X = 0, B_QKV = 1, B_ATTN = 2, B_H = 3, B_RLOG = 4,
  B_QL = 5,  // latent attention: query heads absorbed into the latent space [M][Hq * R]
  B_OL = 6,  // latent attention: attention-weighted latent rows per head [M][Hq * R]
  B_XF = 7,   // x * (the next norm's gain) in the GEMV's B-fragment layout, bf16 hi / lo
  B_XF16 = 8, // the same as f16 hi / lo, for fp8 expert weights
  NBUF = 9
};

struct Mat {
  const uint8_t* w;          // tiles [RT][KT][tile] (expert arrays: [ne][RT][KT][tile])
  const float* scales;       // fp8: [nbr][nbc] (GU: [2][nbr][nbc], gate then up), per expert
  int32_t rows, cols, RT, KT;  // of one expert
  int32_t fp8;
  int32_t nbr, nbc;
  int32_t gu;                // rows interleaved gate/up by 8
  int32_t ne;                // experts in the array (1 for a plain matrix)
  int64_t estride;           // bytes between experts' tiles
  int64_t sstride;           // floats between experts' scales
};

struct Task {
  int16_t type, layer;
  int16_t in_kind, epi;
  int16_t in_buf, out_buf;
  int16_t moe, gain;         // moe: 1 shared experts, 2 routed experts; gain: 0 attn, 1 ffn, 2 final
  int16_t xg_rt, phase;      // xg_rt > 0: rows come in groups of xg_rt row tiles (one per head), each reading
  int32_t xg_stride;         //      its own activation columns, xg_stride floats further per group
  int32_t mat;               // matrix table index
  int32_t rt0, rt1;          // row tiles (GEMV) / item index (ATTN)
  int32_t wait_ctr, wait_tgt;
  int32_t sig_ctr;           // counter incremented when the task is done (-1: none)
  int32_t ss_src;            // IN_X_NORM: which partial-sum array (0: after O, 1: after down)
  int32_t ss_dst;            // EPI_RESID: partial-sum array written
  int32_t mat2;              // T_MOE_DOWN: the shared experts' down matrix
  // Copies taken when the plan is built, so that starting a task needs no
  // dependent global loads: the matrix descriptor and the input's norm gain.
  Mat m;                     // mats[mat]
  const uint16_t* gvec;      // the norm gain of an IN_X_NORM input (null otherwise)
  const uint16_t* gnext;     // EPI_RESID / T_EMBED: the gain of the norm that reads the new x
  int32_t xf16;              // ... and whether an f16 fragment copy is written too (fp8 experts read it)
};

// ---------------------------------------------------------------------------
// device-resident model description
// ---------------------------------------------------------------------------

struct Layer {
  const uint16_t* attn_norm;
  const uint16_t* ffn_norm;
  int32_t m_qkv, m_o, m_gu, m_down;
  int32_t m_router, m_shgu, m_shdown, m_exgu, m_exdown;  // MoE (-1 when dense)
  int32_t m_ukt, m_uv;       // latent attention: per-head W_uk^T [Hq R, dn] and W_uv [Hq dv, R] (-1 otherwise)
};

struct Model {
  int32_t L, H, Hq, Hkv, d, I, V;
  int32_t E, NS, K, Ie;
  int32_t R, dr, fp8;
  float eps;
  const uint16_t* embed;     // [V][H] row-major bf16
  const uint16_t* final_norm;
  int32_t m_lm;
  const float2* rope;        // [max_ctx][rotary dims / 2] (cos, sin)
  int32_t rope_ctx;
  const Layer* layers;
  const Mat* mats;
};

// Per-launch arguments (passed by value).
struct Launch {
  const Model* model;
  const Task* tasks;
  const int32_t* task_off;   // [nCTA + 1]
  // step inputs
  const int32_t* tokens;     // dev [M]
  const int32_t* positions;  // dev [S] or null (then pos_const)
  int32_t pos_const;
  int32_t S, Q, M;
  // KV cache
  uint16_t* kv_k;
  uint16_t* kv_v;
  int32_t kv_seqs, kv_ctx;
  // outputs
  float* logits;             // [M][V] or null
  int32_t* argmax;           // [M]
  int32_t* accepted;         // [1] or null
  int32_t* router_idx;       // trace or null
  float* router_w;
  // scratch
  float* buf[NBUF];
  int32_t ld[NBUF];
  float* ss_part;            // [2][nCTA][MAXM]
  float* am_val;             // [nCTA][MAXM]
  int32_t* am_idx;
  float* att_part;           // [items][rows][d + 2]
  int32_t att_rows_max;
  uint32_t* ctr;             // counters
  int32_t ctr_layer_stride;  // counters per layer
  int32_t ctr_pair_base;     // offset of per-(layer, pair) counters
  int32_t ctr_lm, ctr_done;
  int32_t n_ctr;
  int32_t* status;           // [0] error code, [1] abort flag, [2] detail
  int64_t timeout_ns;
  int32_t stall_ctr;         // test hook: >= 0 -> first consumer waits on this counter
  int32_t n_items;           // attention items per layer
  int32_t n_pairs;           // S * Hkv
  int64_t* trace;            // [nCTA][trace_cap][8] or null
  int32_t trace_cap;
  // One kernel per phase (the multi-kernel comparison path): this launch runs
  // tasks [task_off[c], task_end[c]) of CTA c; phase_mode 1 = a phase that is
  // not the step's last, 2 = the last (it clears the counters at exit).
  // 0 = the whole step in one launch (task_end unused).
  const int32_t* task_end;
  int32_t phase_mode;
};

// counter slots inside one layer
enum CtrSlot {
  C_QKV = 0, C_ATTN = 1, C_O = 2, C_GU = 3, C_DOWN = 4, C_ROUTER = 5, C_STALL = 6,
  C_UKT = 7,  // latent attention: absorbed queries written
  C_UV = 8,   // latent attention: per-head value up-projection written
  C_COMB = 9, // latent attention: splits combined
  NCTR_LAYER = 10
};

enum DevErr { DERR_NONE = 0, DERR_TIMEOUT = 4, DERR_BOUNDS = 5 };

}  // namespace mk

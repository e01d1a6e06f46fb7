// mk_host.cu - C ABI of the decode megakernel: model creation, weight
// layout (seeded fill and loading from caller buffers), KV caches, the
// static task planner and the cooperative launch.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "../../include/mk.h"
#include "../../synth/synth.h"
#include "mk_internal.h"

namespace mk {
// the kernel instance of a model family, without and with tracing compiled in
namespace plain { const void* step_kernel_for(bool mla, bool moe, bool fp8); }
namespace traced { const void* step_kernel_for(bool mla, bool moe, bool fp8); }
}

using namespace mk;

// ---------------------------------------------------------------------------
// logical source of every element of a tiled matrix
// ---------------------------------------------------------------------------
enum MapType { MAP_PLAIN = 0, MAP_GU = 1, MAP_CONCAT = 2, MAP_UKT = 3 };

struct MatMap {
  int32_t type;
  int32_t kindA, kindB;   // tensor kinds (synth ids)
  int32_t layer, expert;
  int32_t rowsA;          // MAP_CONCAT: rows taken from kindA
  int32_t lcolsA, lcolsB; // logical column count of the source tensors
  int32_t Hq, dn, R;      // MAP_UKT
  float sigA, sigB;
};

// tiled (row, col) -> logical (kind selector 0/1, lrow, lcol)
__host__ __device__ static inline void map_elem(const MatMap& mp, int row, int col, int& which, int64_t& lrow,
                                                int64_t& lcol) {
  switch (mp.type) {
    case MAP_GU: {
      const int rt = row >> 4, rr = row & 15;
      which = rr < 8 ? 0 : 1;
      lrow = (int64_t)rt * 8 + (rr & 7);
      lcol = col;
      break;
    }
    case MAP_CONCAT:
      if (row < mp.rowsA) { which = 0; lrow = row; }
      else { which = 1; lrow = row - mp.rowsA; }
      lcol = col;
      break;
    case MAP_UKT: {
      // tiled row = h * R + c, tiled col = i  <->  W_uk[h * dn + i][c]
      const int h = row / mp.R, c = row % mp.R;
      which = 0;
      lrow = (int64_t)h * mp.dn + col;
      lcol = c;
      break;
    }
    default:
      which = 0;
      lrow = row;
      lcol = col;
  }
}

__host__ __device__ static inline void frag_elem(int rt, int ct, int lane, int e, int& row, int& col) {
  const int g = lane >> 2, t = lane & 3;
  row = rt * 16 + g + 8 * ((e >> 1) & 1);
  col = ct * 16 + 2 * t + (e & 1) + 8 * (e >> 2);
}

// Seeded fill, directly in tile order.
__global__ void fill_tiles_kernel(uint8_t* w, int RT, int KT, int rows, int cols, int fp8, MatMap mp, uint64_t keyA,
                                  uint64_t keyB, float scA, float scB) {
  const int64_t n = (int64_t)RT * KT * 32;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int lane = (int)(i & 31);
    const int64_t tile = i >> 5;
    const int rt = (int)(tile / KT), ct = (int)(tile % KT);
    if (!fp8) {
      uint16_t v[8];
      for (int e = 0; e < 8; ++e) {
        int row, col;
        frag_elem(rt, ct, lane, e, row, col);
        v[e] = 0;
        if (row < rows && col < cols) {
          int which;
          int64_t lr, lc;
          map_elem(mp, row, col, which, lr, lc);
          const int64_t lcols = which ? mp.lcolsB : mp.lcolsA;
          v[e] = syn_bf16_normal(which ? keyB : keyA, (uint64_t)(lr * lcols + lc), which ? scB : scA);
        }
      }
      uint4 o;
      o.x = v[0] | ((uint32_t)v[1] << 16);
      o.y = v[2] | ((uint32_t)v[3] << 16);
      o.z = v[4] | ((uint32_t)v[5] << 16);
      o.w = v[6] | ((uint32_t)v[7] << 16);
      reinterpret_cast<uint4*>(w)[i] = o;
    } else {
      uint8_t v[8];
      for (int e = 0; e < 8; ++e) {
        int row, col;
        frag_elem(rt, ct, lane, e, row, col);
        v[e] = 0;
        if (row < rows && col < cols) {
          int which;
          int64_t lr, lc;
          map_elem(mp, row, col, which, lr, lc);
          const int64_t lcols = which ? mp.lcolsB : mp.lcolsA;
          v[e] = syn_e4m3_normal(which ? keyB : keyA, (uint64_t)(lr * lcols + lc), scA);
        }
      }
      uint2 o;
      o.x = v[0] | ((uint32_t)v[1] << 8) | ((uint32_t)v[2] << 16) | ((uint32_t)v[3] << 24);
      o.y = v[4] | ((uint32_t)v[5] << 8) | ((uint32_t)v[6] << 16) | ((uint32_t)v[7] << 24);
      reinterpret_cast<uint2*>(w)[i] = o;
    }
  }
}

// Re-tile one logical source tensor (row-major, on the device) into the
// elements of a tiled matrix that it owns.
__global__ void retile_kernel(uint8_t* w, int RT, int KT, int rows, int cols, int fp8, MatMap mp, int which_src,
                              const uint8_t* src, int64_t src_cols) {
  const int64_t n = (int64_t)RT * KT * 32;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int lane = (int)(i & 31);
    const int64_t tile = i >> 5;
    const int rt = (int)(tile / KT), ct = (int)(tile % KT);
    for (int e = 0; e < 8; ++e) {
      int row, col;
      frag_elem(rt, ct, lane, e, row, col);
      if (row >= rows || col >= cols) continue;
      int which;
      int64_t lr, lc;
      map_elem(mp, row, col, which, lr, lc);
      if (which != which_src) continue;
      if (!fp8) {
        reinterpret_cast<uint16_t*>(w)[i * 8 + e] = reinterpret_cast<const uint16_t*>(src)[lr * src_cols + lc];
      } else {
        w[i * 8 + e] = src[lr * src_cols + lc];
      }
    }
  }
}

__global__ void fill_bf16_kernel(uint16_t* dst, int64_t n, uint64_t key, float sc, int gain) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = gain ? syn_bf16_gain(key, (uint64_t)i, sc) : syn_bf16_normal(key, (uint64_t)i, sc);
}

__global__ void fill_scales_kernel(float* dst, int64_t n, uint64_t key, float base) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = syn_block_scale(key, (uint64_t)i, base);
}

// Synthetic KV context: sequence s, kv head g, position t, element i of
// layer l has index ((s * G + g) << 32) + t * d + i in stream (KV_K|KV_V, l).
__global__ void fill_kv_kernel(uint16_t* dst, int L, int S, int G, int Tmax, int d, int T, uint64_t seed, int kind,
                               float sc, int permuted) {
  const int64_t n = (int64_t)L * S * G * T * d;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int e = (int)(i % d);
    int64_t r = i / d;
    const int t = (int)(r % T);
    r /= T;
    const int g = (int)(r % G);
    r /= G;
    const int s = (int)(r % S);
    const int l = (int)(r / S);
    const uint64_t key = syn_key(seed, syn_stream((uint32_t)kind, (uint32_t)l, 0));
    const uint64_t idx = ((uint64_t)(s * G + g) << 32) + (uint64_t)t * d + e;
    dst[((((int64_t)l * S + s) * G + g) * Tmax + t) * d + (permuted ? kv_swz(t, e) : e)] = syn_bf16_normal(key, idx, sc);
  }
}

// Copy GQA K or V rows out of the cache in logical order (undo the in-row
// permutation of the 16-byte groups).
__global__ void unpermute_kv_kernel(uint16_t* dst, const uint16_t* src, int64_t rows, int Tmax, int d) {
  const int64_t n = rows * d;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / d;
    const int e = (int)(i - r * d);
    const int t = (int)(r % Tmax);
    dst[i] = src[r * d + kv_swz(t, e)];
  }
}

// The inverse: rows in logical order into the cache's permuted row layout.
__global__ void permute_kv_kernel(uint16_t* dst, const uint16_t* src, int64_t rows, int Tmax, int d) {
  const int64_t n = rows * d;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / d;
    const int e = (int)(i - r * d);
    const int t = (int)(r % Tmax);
    dst[r * d + kv_swz(t, e)] = src[i];
  }
}

// ---------------------------------------------------------------------------
// handle
// ---------------------------------------------------------------------------
struct MatHost {
  Mat m;
  MatMap map;
  size_t bytes;
};

struct PlanKey {
  int S, Q;
  bool operator<(const PlanKey& o) const { return S < o.S || (S == o.S && Q < o.Q); }
};

struct Plan {
  Task* d_tasks = nullptr;
  int32_t* d_off = nullptr;
  int n_items = 0, n_pairs = 0;
  int n_tasks = 0;
  // multi-kernel path: the non-empty phases, each CTA's task range per phase
  std::vector<Task> host_tasks;
  std::vector<int32_t> host_off;
  int n_phases = 0;
  int32_t* d_pbeg = nullptr;  // [phases][ncta]
  int32_t* d_pend = nullptr;
  int n_kphases = 0;
};

// One CUDA graph of the multi-kernel step per (batch, cache, logits wanted).
struct GraphKey {
  int S;
  const void* kv;
  bool logits;
  const void* rtrace;  // router trace buffer (baked into the kernel arguments)
  bool operator<(const GraphKey& o) const {
    if (S != o.S) return S < o.S;
    if (kv != o.kv) return kv < o.kv;
    if (logits != o.logits) return logits < o.logits;
    return rtrace < o.rtrace;
  }
};

struct mk_handle {
  mk_model_desc desc{};
  int device = 0;
  int ncta = 0;
  std::vector<void*> allocs;
  std::vector<MatHost> mats;
  std::vector<Layer> layers;
  Model model{};
  Model* d_model = nullptr;
  Mat* d_mats = nullptr;
  Layer* d_layers = nullptr;
  uint16_t* embed = nullptr;
  uint16_t* final_norm = nullptr;
  std::vector<uint16_t*> attn_norm, ffn_norm;
  float2* rope = nullptr;
  int64_t weight_bytes = 0;
  // scratch
  float* buf[NBUF] = {};
  int32_t ld[NBUF] = {};
  float* ss_part = nullptr;
  float* am_val = nullptr;
  int32_t* am_idx = nullptr;
  float* att_part = nullptr;
  int att_rows_max = 0;
  int att_dpart = 0;  // values per attention partial row (head_dim, or kv_lora_rank for latent attention)
  int n_items_max = 0;
  int max_pairs = 0;
  uint32_t* ctr = nullptr;
  int n_ctr = 0;
  int32_t* status = nullptr;
  float* logits_tmp = nullptr;
  int32_t* argmax_tmp = nullptr;
  int32_t* spec_dev = nullptr;   // speculative generation: tokens [8] | argmax [8] | accepted [1]
  std::map<PlanKey, Plan> plans;
  // multi-kernel comparison path: fixed step buffers and the captured graphs
  int32_t* mk_tokens = nullptr;  // [MAXM]
  int32_t* mk_pos = nullptr;     // [MAXM]
  int32_t* mk_argmax = nullptr;  // [MAXM]
  float* mk_logits = nullptr;    // [MAXM][vocab]
  cudaStream_t mk_capture = nullptr;
  std::map<GraphKey, cudaGraphExec_t> graphs;
  int32_t* trace_idx = nullptr;
  float* trace_w = nullptr;
  int64_t* task_trace = nullptr;
  int32_t task_trace_cap = 0;
  int64_t stall_ns = 0;
  int64_t timeout_ns = 1000000000LL;
  bool sticky = false;
  bool initialised = false;
  uint64_t noalloc_id = 0;  // identity of this handle for mk_decode_step_noalloc's installed task list
  const void* kernel = nullptr;         // the step kernel instance of this model's family
  const void* kernel_traced = nullptr;  // ... with tracing compiled in (launched while a trace buffer is set)
  std::string err;
};

struct mk_kv {
  mk_handle* h;
  int max_seqs, max_ctx;
  uint16_t* k = nullptr;
  uint16_t* v = nullptr;
  int64_t bytes = 0;
};

// Why the calling thread's last mk_create failed (it returns no handle).
static thread_local std::string g_create_error = "null handle";

static mk_status fail(mk_handle* h, mk_status s, const std::string& msg) {
  if (h) h->err = msg;
  return s;
}

#define CK(call)                                                                                     \
  do {                                                                                               \
    cudaError_t e_ = (call);                                                                         \
    if (e_ != cudaSuccess) return fail(h, MK_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

static mk_status dalloc(mk_handle* h, void** p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(h, MK_ERR_OOM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed");
  }
  h->allocs.push_back(*p);
  return MK_OK;
}

static int cdiv(int a, int b) { return (a + b - 1) / b; }

static mk_status add_mat(mk_handle* h, int rows, int cols, int fp8, int gu, const MatMap& mp, int* out_idx,
                         int ne = 1) {
  MatHost mh{};
  mh.m.rows = rows;
  mh.m.cols = cols;
  mh.m.RT = cdiv(rows, 16);
  mh.m.KT = cdiv(cols, 16);
  mh.m.fp8 = fp8;
  mh.m.gu = gu;
  mh.m.ne = ne;
  mh.map = mp;
  const size_t tb = fp8 ? TILE_FP8 : TILE_BF16;
  const size_t one = (size_t)mh.m.RT * mh.m.KT * tb;
  mh.m.estride = (int64_t)one;
  mh.bytes = one * ne;
  void* p = nullptr;
  mk_status s = dalloc(h, &p, mh.bytes);
  if (s != MK_OK) return s;
  mh.m.w = reinterpret_cast<const uint8_t*>(p);
  h->weight_bytes += (int64_t)mh.bytes;
  if (fp8) {
    const int lrows = gu ? rows / 2 : rows;
    mh.m.nbr = cdiv(lrows, 128);
    mh.m.nbc = cdiv(cols, 128);
    const size_t per = (size_t)(gu ? 2 : 1) * mh.m.nbr * mh.m.nbc;
    mh.m.sstride = (int64_t)per;
    const size_t sb = per * ne * sizeof(float);
    s = dalloc(h, &p, sb);
    if (s != MK_OK) return s;
    mh.m.scales = reinterpret_cast<const float*>(p);
    h->weight_bytes += (int64_t)sb;
  }
  *out_idx = (int)h->mats.size();
  h->mats.push_back(mh);
  return MK_OK;
}

static bool desc_ok(const mk_model_desc* d, std::string& why) {
  if (!d) { why = "null descriptor"; return false; }
  if (d->layers < 1 || d->hidden < 16 || d->hidden % 16) { why = "hidden must be a positive multiple of 16"; return false; }
  if (d->vocab < 2) { why = "vocab < 2"; return false; }
  if (d->max_batch < 1 || d->max_batch > MAXM) { why = "max_batch must be in [1, 8]"; return false; }
  if (d->max_ctx < 2) { why = "max_ctx < 2"; return false; }
  if (d->kv_lora_rank > 0) {
    // latent attention: one item holds all heads of one query row (<= 2 m-tiles), the latent
    // rows [c | k_rope] are moved as whole rows (16-byte multiples), each consumer warp owns
    // kv_lora_rank / 8 latent dims (whole 8-dim tiles, at most 8 of them)
    if (d->n_q_heads < 1 || d->n_q_heads > 32) { why = "latent attention needs 1 <= n_q_heads <= 32"; return false; }
    if (d->kv_lora_rank % 64 || d->kv_lora_rank > 512) { why = "kv_lora_rank must be a multiple of 64, <= 512"; return false; }
    if (d->rope_dim < 16 || d->rope_dim % 16) { why = "rope_dim must be a positive multiple of 16"; return false; }
    if (d->head_dim < 16 || d->head_dim % 16) { why = "head_dim must be a positive multiple of 16"; return false; }
    if (mla_smem_need(d->n_q_heads, d->kv_lora_rank, d->rope_dim) > MLA_SCRATCH_BYTES) {
      why = "latent attention shapes exceed the shared-memory scratch";
      return false;
    }
  } else {
    if (d->head_dim != 64 && d->head_dim != 128) { why = "head_dim must be 64 or 128"; return false; }
    if (d->n_kv_heads < 1 || d->n_q_heads % d->n_kv_heads) { why = "n_q_heads must be a multiple of n_kv_heads"; return false; }
    if ((d->n_q_heads / d->n_kv_heads) * MAXM > 48) { why = "query heads per kv head must be <= 6"; return false; }
  }
  if (d->n_routed == 0) {
    if (d->ffn < 8 || d->ffn % 8) { why = "ffn must be a positive multiple of 8"; return false; }
  } else {
    if (d->n_routed > 256 || d->top_k < 1 || d->top_k > 8 || d->top_k > d->n_routed) {
      why = "MoE needs 1 <= top_k <= min(8, n_routed) and n_routed <= 256";
      return false;
    }
    if (d->expert_ffn < 16 || d->expert_ffn % 16 || d->n_shared < 0 || d->n_shared > 8) {
      why = "expert_ffn must be a positive multiple of 16, n_shared in [0, 8]";
      return false;
    }
  }
  if (d->expert_fp8 && d->n_routed == 0) { why = "fp8 weights are supported for experts only"; return false; }
  if (d->expert_fp8 && (d->hidden > 16384 || d->expert_ffn > 16384)) {
    // the kernel stages a row group's block scales (<= 128 column blocks) in shared memory
    why = "fp8 experts need hidden and expert_ffn <= 16384";
    return false;
  }
  return true;
}

extern "C" {

mk_status mk_create(const mk_model_desc* desc, int device, mk_handle** out) {
  if (!out) return MK_ERR_INVALID;
  *out = nullptr;
  std::string why;
  if (!desc_ok(desc, why)) {
    g_create_error = "invalid model description: " + why;
    return MK_ERR_INVALID;
  }
  mk_handle* h = new mk_handle();
  h->desc = *desc;
  h->device = device;
  mk_status s;
#define TRY(x)                      \
  do {                              \
    s = (x);                        \
    if (s != MK_OK) goto fail_out;  \
  } while (0)
  {
    if (cudaSetDevice(device) != cudaSuccess) { s = MK_ERR_CUDA; h->err = "cudaSetDevice failed"; goto fail_out; }
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) { s = MK_ERR_CUDA; goto fail_out; }
    if (prop.major < 10) { s = MK_ERR_INVALID; h->err = "needs an sm_100 device"; goto fail_out; }
    h->ncta = prop.multiProcessorCount;
    const mk_model_desc& d = *desc;
    const int L = d.layers, H = d.hidden, Hq = d.n_q_heads, G = d.n_kv_heads, hd = d.head_dim;
    const bool mla = d.kv_lora_rank > 0;
    const int R = d.kv_lora_rank, dr = d.rope_dim;
    // ---- weights ----
    TRY(dalloc(h, (void**)&h->embed, (size_t)d.vocab * H * 2));
    TRY(dalloc(h, (void**)&h->final_norm, (size_t)H * 2));
    h->weight_bytes += (int64_t)d.vocab * H * 2 + H * 2;
    h->layers.resize(L);
    h->attn_norm.resize(L);
    h->ffn_norm.resize(L);
    for (int l = 0; l < L; ++l) {
      Layer& ly = h->layers[l];
      TRY(dalloc(h, (void**)&h->attn_norm[l], (size_t)H * 2));
      TRY(dalloc(h, (void**)&h->ffn_norm[l], (size_t)H * 2));
      h->weight_bytes += 4LL * H;
      ly.attn_norm = h->attn_norm[l];
      ly.ffn_norm = h->ffn_norm[l];
      MatMap mp{};
      ly.m_ukt = ly.m_uv = -1;
      if (!mla) {
        mp.layer = l;
        mp.type = MAP_PLAIN;
        mp.kindA = SYN_WQKV;
        mp.lcolsA = H;
        TRY(add_mat(h, (Hq + 2 * G) * hd, H, 0, 0, mp, &ly.m_qkv));
      } else {
        // queries [nope | rope] per head, then the latent c and the shared rope key
        mp.layer = l;
        mp.type = MAP_CONCAT;
        mp.kindA = SYN_MLA_WQ;
        mp.kindB = SYN_MLA_WDKV;
        mp.rowsA = Hq * (hd + dr);
        mp.lcolsA = mp.lcolsB = H;
        TRY(add_mat(h, Hq * (hd + dr) + R + dr, H, 0, 0, mp, &ly.m_qkv));
        // W_uk transposed per head: row h * R + c reads W_uk[h * dn + i][c] over i
        mp = MatMap{};
        mp.layer = l;
        mp.type = MAP_UKT;
        mp.kindA = SYN_MLA_WUK;
        mp.lcolsA = R;
        mp.Hq = Hq;
        mp.dn = hd;
        mp.R = R;
        TRY(add_mat(h, Hq * R, hd, 0, 0, mp, &ly.m_ukt));
        mp = MatMap{};
        mp.layer = l;
        mp.kindA = SYN_MLA_WUV;
        mp.lcolsA = R;
        TRY(add_mat(h, Hq * hd, R, 0, 0, mp, &ly.m_uv));
      }
      mp = MatMap{};
      mp.layer = l;
      mp.kindA = SYN_WO;
      mp.lcolsA = Hq * hd;
      TRY(add_mat(h, H, Hq * hd, 0, 0, mp, &ly.m_o));
      ly.m_gu = ly.m_down = ly.m_router = ly.m_shgu = ly.m_shdown = ly.m_exgu = ly.m_exdown = -1;
      if (d.n_routed == 0) {
        mp = MatMap{};
        mp.layer = l;
        mp.type = MAP_GU;
        mp.kindA = SYN_WGATE;
        mp.kindB = SYN_WUP;
        mp.lcolsA = mp.lcolsB = H;
        TRY(add_mat(h, 2 * d.ffn, H, 0, 1, mp, &ly.m_gu));
        mp = MatMap{};
        mp.layer = l;
        mp.kindA = SYN_WDOWN;
        mp.lcolsA = d.ffn;
        TRY(add_mat(h, H, d.ffn, 0, 0, mp, &ly.m_down));
      } else {
        const int Ie = d.expert_ffn, E = d.n_routed, NS = d.n_shared, f8 = d.expert_fp8 ? 1 : 0;
        mp = MatMap{};
        mp.layer = l;
        mp.kindA = SYN_ROUTER;
        mp.lcolsA = H;
        TRY(add_mat(h, E, H, 0, 0, mp, &ly.m_router));
        if (NS > 0) {
          mp = MatMap{};
          mp.layer = l;
          mp.type = MAP_GU;
          mp.kindA = SYN_SH_GATE;
          mp.kindB = SYN_SH_UP;
          mp.lcolsA = mp.lcolsB = H;
          TRY(add_mat(h, 2 * Ie, H, f8, 1, mp, &ly.m_shgu, NS));
          mp = MatMap{};
          mp.layer = l;
          mp.kindA = SYN_SH_DOWN;
          mp.lcolsA = Ie;
          TRY(add_mat(h, H, Ie, f8, 0, mp, &ly.m_shdown, NS));
        }
        mp = MatMap{};
        mp.layer = l;
        mp.type = MAP_GU;
        mp.kindA = SYN_EX_GATE;
        mp.kindB = SYN_EX_UP;
        mp.lcolsA = mp.lcolsB = H;
        TRY(add_mat(h, 2 * Ie, H, f8, 1, mp, &ly.m_exgu, E));
        mp = MatMap{};
        mp.layer = l;
        mp.kindA = SYN_EX_DOWN;
        mp.lcolsA = Ie;
        TRY(add_mat(h, H, Ie, f8, 0, mp, &ly.m_exdown, E));
      }
    }
    {
      MatMap mp{};
      mp.kindA = SYN_LM_HEAD;
      mp.lcolsA = H;
      TRY(add_mat(h, d.vocab, H, 0, 0, mp, &h->model.m_lm));
    }
    // ---- RoPE table, double precision angles rounded to fp32 ----
    {
      const int rd = mla ? dr : hd;  // rotary dims
      const int half = rd / 2;
      std::vector<float2> tab((size_t)d.max_ctx * half);
      for (int p = 0; p < d.max_ctx; ++p)
        for (int i = 0; i < half; ++i) {
          const double inv = pow((double)d.rope_theta, -2.0 * i / (double)rd);
          const double ang = (double)p * inv;
          tab[(size_t)p * half + i] = make_float2((float)cos(ang), (float)sin(ang));
        }
      TRY(dalloc(h, (void**)&h->rope, tab.size() * sizeof(float2)));
      if (cudaMemcpy(h->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess) {
        s = MK_ERR_CUDA;
        goto fail_out;
      }
    }
    // ---- device model tables ----
    std::vector<Mat> mv;
    for (auto& m : h->mats) mv.push_back(m.m);
    TRY(dalloc(h, (void**)&h->d_mats, mv.size() * sizeof(Mat)));
    TRY(dalloc(h, (void**)&h->d_layers, (size_t)L * sizeof(Layer)));
    TRY(dalloc(h, (void**)&h->d_model, sizeof(Model)));
    Model& md = h->model;
    md.L = L;
    md.H = H;
    md.Hq = Hq;
    md.Hkv = G;
    md.d = hd;
    md.I = d.ffn;
    md.V = d.vocab;
    md.E = d.n_routed;
    md.NS = d.n_shared;
    md.K = d.top_k;
    md.Ie = d.expert_ffn;
    md.R = d.kv_lora_rank;
    md.dr = d.rope_dim;
    md.fp8 = d.expert_fp8;
    md.eps = d.rms_eps;
    md.embed = h->embed;
    md.final_norm = h->final_norm;
    md.rope = h->rope;
    md.rope_ctx = d.max_ctx;
    md.layers = h->d_layers;
    md.mats = h->d_mats;
    if (cudaMemcpy(h->d_mats, mv.data(), mv.size() * sizeof(Mat), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(h->d_layers, h->layers.data(), (size_t)L * sizeof(Layer), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(h->d_model, &md, sizeof(Model), cudaMemcpyHostToDevice) != cudaSuccess) {
      s = MK_ERR_CUDA;
      goto fail_out;
    }
    // ---- scratch ----
    const int MB = MAXM;
    // B_H: dense [M][ffn]; MoE [slot][M][expert_ffn] with slots = shared + the most
    // distinct routed experts one step can select
    const int hw = d.n_routed ? d.expert_ffn : d.ffn;
    const int hslots = d.n_routed ? d.n_shared + std::min(d.n_routed, MAXM * d.top_k) : 1;
    const int qkv_w = mla ? Hq * (hd + dr) + R + dr : (Hq + 2 * G) * hd;
    const int lat_w = mla ? Hq * R : 4;
    // B_QL holds the absorbed queries as bf16 hi / lo attention fragments:
    // 2 x (row tiles of 16 heads) x (R / 16) tiles x 512 B per query row
    const int ql_w = mla ? ((Hq + 15) / 16) * 16 * R : 4;
    const int xf16_w = (d.n_routed && d.expert_fp8) ? H : 4;
    const int widths[NBUF] = {H, qkv_w, Hq * hd, std::max(hw, 8), std::max(d.n_routed, 4), ql_w, lat_w, H, xf16_w};
    for (int b = 0; b < NBUF; ++b) {
      h->ld[b] = (widths[b] + 3) & ~3;
      const size_t rows = (b == B_H) ? (size_t)hslots * MB : (size_t)MB;
      TRY(dalloc(h, (void**)&h->buf[b], rows * h->ld[b] * sizeof(float)));
    }
    TRY(dalloc(h, (void**)&h->ss_part, (size_t)2 * h->ncta * MAXM * sizeof(float)));
    TRY(dalloc(h, (void**)&h->am_val, (size_t)h->ncta * MAXM * sizeof(float)));
    TRY(dalloc(h, (void**)&h->am_idx, (size_t)h->ncta * MAXM * sizeof(int32_t)));
    // attention pairs: (sequence, kv head) for GQA, one query row for latent attention
    h->max_pairs = mla ? d.max_batch : d.max_batch * G;
    h->n_items_max = std::max(h->ncta, h->max_pairs);
    h->att_rows_max = mla ? Hq : MAXM * (Hq / G);
    h->att_dpart = mla ? R : hd;
    TRY(dalloc(h, (void**)&h->att_part,
               (size_t)h->n_items_max * h->att_rows_max * (h->att_dpart + 4) * sizeof(float)));
    h->n_ctr = (L + 1) * NCTR_LAYER + L * h->max_pairs + 2;
    TRY(dalloc(h, (void**)&h->ctr, (size_t)h->n_ctr * sizeof(uint32_t)));
    TRY(dalloc(h, (void**)&h->status, 4 * sizeof(int32_t)));
    TRY(dalloc(h, (void**)&h->logits_tmp, 16));
    TRY(dalloc(h, (void**)&h->argmax_tmp, MAXM * sizeof(int32_t)));
    TRY(dalloc(h, (void**)&h->spec_dev, 32 * sizeof(int32_t)));
    if (cudaMemset(h->ctr, 0, (size_t)h->n_ctr * 4) != cudaSuccess || cudaMemset(h->status, 0, 16) != cudaSuccess) {
      s = MK_ERR_CUDA;
      goto fail_out;
    }
    h->kernel = plain::step_kernel_for(d.kv_lora_rank > 0, d.n_routed > 0, d.n_routed > 0 && d.expert_fp8 != 0);
    h->kernel_traced = traced::step_kernel_for(d.kv_lora_rank > 0, d.n_routed > 0, d.n_routed > 0 && d.expert_fp8 != 0);
    if (cudaFuncSetAttribute(h->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(h->kernel_traced, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess) {
      s = MK_ERR_CUDA;
      h->err = std::string("cannot reserve dynamic shared memory: ") + cudaGetErrorString(cudaGetLastError());
      goto fail_out;
    }
    int occ = 0;
    int occ_tr = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, h->kernel, NTHREADS, SMEM_BYTES) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_tr, h->kernel_traced, NTHREADS, SMEM_BYTES) != cudaSuccess ||
        occ < 1 || occ_tr < 1) {
      s = MK_ERR_CUDA;
      h->err = "kernel does not fit one CTA per SM (occupancy " + std::to_string(occ) + ", " +
               cudaGetErrorString(cudaGetLastError()) + ")";
      goto fail_out;
    }
  }
#undef TRY
  *out = h;
  return MK_OK;
fail_out:
  g_create_error = h->err.empty() ? std::string("mk_create failed (status ") + std::to_string((int)s) + ")" : h->err;
  for (void* p : h->allocs) cudaFree(p);
  delete h;
  return s;
}

void mk_destroy(mk_handle* h) {
  if (!h) return;
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  for (auto& kv : h->plans) {
    cudaFree(kv.second.d_tasks);
    cudaFree(kv.second.d_off);
    cudaFree(kv.second.d_pbeg);
    cudaFree(kv.second.d_pend);
  }
  for (auto& g : h->graphs) cudaGraphExecDestroy(g.second);
  if (h->mk_capture) cudaStreamDestroy(h->mk_capture);
  for (void* p : h->allocs) cudaFree(p);
  delete h;
}

const char* mk_last_error(const mk_handle* h) { return h ? h->err.c_str() : g_create_error.c_str(); }
int64_t mk_weight_bytes(const mk_handle* h) { return h ? h->weight_bytes : 0; }

mk_status mk_launch_info(mk_handle* h, int32_t* ctas, int32_t* smem_bytes, int32_t* threads) {
  if (!h) return MK_ERR_INVALID;
  if (ctas) *ctas = h->ncta;
  if (smem_bytes) *smem_bytes = SMEM_BYTES;
  if (threads) *threads = NTHREADS;
  return MK_OK;
}

// ---------------------------------------------------------------------------
// weights
// ---------------------------------------------------------------------------
static void launch_fill(const MatHost& mh, uint64_t seed, float sigA, float sigB, float fp8_base) {
  const int64_t n = (int64_t)mh.m.RT * mh.m.KT * 32;
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
  for (int e = 0; e < mh.m.ne; ++e) {
    MatMap mp = mh.map;
    if (mh.m.ne > 1 || mp.kindA == SYN_EX_GATE || mp.kindA == SYN_EX_DOWN || mp.kindA == SYN_SH_GATE ||
        mp.kindA == SYN_SH_DOWN)
      mp.expert = e;
    const uint64_t kA = syn_key(seed, syn_stream((uint32_t)mp.kindA, (uint32_t)mp.layer, (uint32_t)mp.expert));
    const uint64_t kB = syn_key(seed, syn_stream((uint32_t)mp.kindB, (uint32_t)mp.layer, (uint32_t)mp.expert));
    const float sA = mh.m.fp8 ? syn_normal_scale(16.0) : syn_normal_scale(sigA);
    const float sB = mh.m.fp8 ? syn_normal_scale(16.0) : syn_normal_scale(sigB);
    uint8_t* w = const_cast<uint8_t*>(mh.m.w) + (size_t)e * mh.m.estride;
    fill_tiles_kernel<<<blocks, 256>>>(w, mh.m.RT, mh.m.KT, mh.m.rows, mh.m.cols, mh.m.fp8, mp, kA, kB, sA, sB);
    if (mh.m.fp8) {
      const int64_t per = (int64_t)mh.m.nbr * mh.m.nbc;
      float* sc = const_cast<float*>(mh.m.scales) + (size_t)e * mh.m.sstride;
      const uint64_t sk = syn_key(seed, syn_stream(SYN_FP8_SCALE, (uint32_t)mp.layer, ((uint32_t)mp.kindA << 12) | (uint32_t)mp.expert));
      fill_scales_kernel<<<64, 256>>>(sc, per, sk, fp8_base);
      if (mh.m.gu) {
        const uint64_t sk2 = syn_key(seed, syn_stream(SYN_FP8_SCALE, (uint32_t)mp.layer, ((uint32_t)mp.kindB << 12) | (uint32_t)mp.expert));
        fill_scales_kernel<<<64, 256>>>(sc + per, per, sk2, fp8_base);
      }
    }
  }
}

static void launch_fill_vec(uint16_t* dst, int64_t n, uint64_t key, float sc, int gain) {
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
  fill_bf16_kernel<<<blocks, 256>>>(dst, n, key, sc, gain);
}

mk_status mk_init_random(mk_handle* h, const mk_synth_params* p) {
  if (!h || !p) return fail(h, MK_ERR_INVALID, "null argument");
  cudaSetDevice(h->device);
  const mk_model_desc& d = h->desc;
  const uint64_t seed = p->seed;
  launch_fill_vec(h->embed, (int64_t)d.vocab * d.hidden, syn_key(seed, syn_stream(SYN_EMBED, 0, 0)),
                  syn_normal_scale(p->w_sigma), 0);
  launch_fill_vec(h->final_norm, d.hidden, syn_key(seed, syn_stream(SYN_FINAL_NORM, 0, 0)),
                  syn_normal_scale(p->gain_sigma), 1);
  for (int l = 0; l < d.layers; ++l) {
    launch_fill_vec(h->attn_norm[l], d.hidden, syn_key(seed, syn_stream(SYN_ATTN_NORM, (uint32_t)l, 0)),
                    syn_normal_scale(p->gain_sigma), 1);
    launch_fill_vec(h->ffn_norm[l], d.hidden, syn_key(seed, syn_stream(SYN_FFN_NORM, (uint32_t)l, 0)),
                    syn_normal_scale(p->gain_sigma), 1);
  }
  for (auto& mh : h->mats) {
    const float sig = (mh.map.kindA == SYN_ROUTER) ? p->router_sigma : p->w_sigma;
    launch_fill(mh, seed, sig, p->w_sigma, p->fp8_block_base);
  }
  CK(cudaGetLastError());
  CK(cudaDeviceSynchronize());
  h->initialised = true;
  return MK_OK;
}

static int find_mat(mk_handle* h, int kind, int layer, int expert, int* which) {
  for (size_t i = 0; i < h->mats.size(); ++i) {
    const MatMap& mp = h->mats[i].map;
    if (mp.layer != layer) continue;
    if (h->mats[i].m.ne > 1 || kind == SYN_EX_GATE || kind == SYN_EX_UP || kind == SYN_EX_DOWN ||
        kind == SYN_SH_GATE || kind == SYN_SH_UP || kind == SYN_SH_DOWN) {
      if (expert < 0 || expert >= h->mats[i].m.ne) continue;
    } else if (mp.expert != expert) {
      continue;
    }
    if (mp.kindA == kind) { *which = 0; return (int)i; }
    if ((mp.type == MAP_GU || mp.type == MAP_CONCAT) && mp.kindB == kind) { *which = 1; return (int)i; }
  }
  return -1;
}

mk_status mk_load_weights(mk_handle* h, const mk_tensor_src* ts, int n) {
  if (!h || (!ts && n > 0)) return fail(h, MK_ERR_INVALID, "null argument");
  cudaSetDevice(h->device);
  const mk_model_desc& d = h->desc;
  for (int i = 0; i < n; ++i) {
    const mk_tensor_src& t = ts[i];
    if (!t.data) return fail(h, MK_ERR_INVALID, "tensor " + std::to_string(i) + ": null data");
    const cudaMemcpyKind kind = t.on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    // vectors
    uint16_t* vec = nullptr;
    int64_t vlen = 0;
    if (t.kind == SYN_EMBED) { vec = h->embed; vlen = (int64_t)d.vocab * d.hidden; }
    else if (t.kind == SYN_FINAL_NORM) { vec = h->final_norm; vlen = d.hidden; }
    else if (t.kind == SYN_ATTN_NORM || t.kind == SYN_FFN_NORM) {
      if (t.layer < 0 || t.layer >= d.layers) return fail(h, MK_ERR_INVALID, "layer out of range");
      vec = (t.kind == SYN_ATTN_NORM ? h->attn_norm : h->ffn_norm)[t.layer];
      vlen = d.hidden;
    }
    if (vec) {
      if (t.rows * t.cols != vlen) return fail(h, MK_ERR_INVALID, "tensor " + std::to_string(i) + ": wrong size");
      CK(cudaMemcpy(vec, t.data, (size_t)vlen * 2, kind));
      continue;
    }
    int which = 0;
    const int mi = find_mat(h, t.kind, t.layer, t.expert, &which);
    if (mi < 0) return fail(h, MK_ERR_INVALID, "tensor " + std::to_string(i) + ": unknown kind/layer/expert");
    MatHost& mh = h->mats[mi];
    int64_t lrows = mh.m.rows, lcols = mh.m.cols;
    if (mh.map.type == MAP_GU) lrows = mh.m.rows / 2;
    if (mh.map.type == MAP_CONCAT) lrows = which ? mh.m.rows - mh.map.rowsA : mh.map.rowsA;
    if (mh.map.type == MAP_UKT) {  // the source is W_uk [Hq dn, R]; the tiles hold its per-head transpose
      lrows = (int64_t)mh.map.Hq * mh.map.dn;
      lcols = mh.map.R;
    }
    if (t.rows != lrows || t.cols != lcols)
      return fail(h, MK_ERR_INVALID, "tensor " + std::to_string(i) + ": shape mismatch");
    const size_t eb = mh.m.fp8 ? 1 : 2;
    const size_t nbytes = (size_t)lrows * lcols * eb;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(t.data);
    void* staging = nullptr;
    if (!t.on_device) {
      CK(cudaMalloc(&staging, nbytes));
      cudaError_t e = cudaMemcpy(staging, t.data, nbytes, cudaMemcpyHostToDevice);
      if (e != cudaSuccess) { cudaFree(staging); return fail(h, MK_ERR_CUDA, "weight upload failed"); }
      src = reinterpret_cast<const uint8_t*>(staging);
    }
    const int64_t nthr = (int64_t)mh.m.RT * mh.m.KT * 32;
    const int blocks = (int)std::min<int64_t>((nthr + 255) / 256, 148 * 16);
    retile_kernel<<<blocks, 256>>>(const_cast<uint8_t*>(mh.m.w) + (size_t)(mh.m.ne > 1 || t.expert > 0 ? t.expert : 0) * mh.m.estride,
                                   mh.m.RT, mh.m.KT, mh.m.rows, mh.m.cols, mh.m.fp8, mh.map, which, src, lcols);
    cudaError_t e = cudaDeviceSynchronize();
    if (staging) cudaFree(staging);
    if (e != cudaSuccess) return fail(h, MK_ERR_CUDA, std::string("retile: ") + cudaGetErrorString(e));
    if (mh.m.fp8) {
      if (!t.scales) return fail(h, MK_ERR_INVALID, "fp8 tensor without scales");
      const size_t sn = (size_t)mh.m.nbr * mh.m.nbc;
      float* dst = const_cast<float*>(mh.m.scales) + (size_t)t.expert * mh.m.sstride + (mh.m.gu && which ? sn : 0);
      CK(cudaMemcpy(dst, t.scales, sn * sizeof(float), kind));
    }
  }
  h->initialised = true;
  return MK_OK;
}

// ---------------------------------------------------------------------------
// KV caches
// ---------------------------------------------------------------------------
mk_status mk_kv_create(mk_handle* h, int max_seqs, int max_ctx, mk_kv** out) {
  if (!h || !out) return fail(h, MK_ERR_INVALID, "null argument");
  *out = nullptr;
  if (max_seqs < 1 || max_seqs > MAXM || max_ctx < 2 || max_ctx > h->desc.max_ctx)
    return fail(h, MK_ERR_INVALID, "kv: max_seqs in [1, 8] and max_ctx in [2, model max_ctx] required");
  cudaSetDevice(h->device);
  const mk_model_desc& d = h->desc;
  mk_kv* kv = new mk_kv();
  kv->h = h;
  kv->max_seqs = max_seqs;
  kv->max_ctx = max_ctx;
  if (d.kv_lora_rank > 0) {
    // latent rows [c | k_rope] per (layer, sequence, position); no separate values
    const size_t n = (size_t)d.layers * max_seqs * max_ctx * (d.kv_lora_rank + d.rope_dim);
    if (cudaMalloc(&kv->k, n * 2) != cudaSuccess) {
      cudaGetLastError();
      delete kv;
      return fail(h, MK_ERR_OOM, "kv cache allocation failed");
    }
    kv->bytes = (int64_t)n * 2;
    cudaMemset(kv->k, 0, n * 2);
    CK(cudaDeviceSynchronize());
    *out = kv;
    return MK_OK;
  }
  const size_t n = (size_t)d.layers * max_seqs * d.n_kv_heads * max_ctx * d.head_dim;
  if (cudaMalloc(&kv->k, n * 2) != cudaSuccess || cudaMalloc(&kv->v, n * 2) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(kv->k);
    cudaFree(kv->v);
    delete kv;
    return fail(h, MK_ERR_OOM, "kv cache allocation failed");
  }
  kv->bytes = (int64_t)n * 4;
  cudaMemset(kv->k, 0, n * 2);
  cudaMemset(kv->v, 0, n * 2);
  CK(cudaDeviceSynchronize());
  *out = kv;
  return MK_OK;
}

void mk_kv_destroy(mk_kv* kv) {
  if (!kv) return;
  cudaSetDevice(kv->h->device);
  cudaDeviceSynchronize();
  cudaFree(kv->k);
  cudaFree(kv->v);
  delete kv;
}

int64_t mk_kv_bytes(const mk_kv* kv) { return kv ? kv->bytes : 0; }

mk_status mk_kv_fill_random(mk_kv* kv, uint64_t seed, float sigma, int32_t length) {
  if (!kv) return MK_ERR_INVALID;
  mk_handle* h = kv->h;
  if (length < 0 || length > kv->max_ctx) return fail(h, MK_ERR_INVALID, "kv fill length out of range");
  if (length == 0) return MK_OK;
  cudaSetDevice(h->device);
  const mk_model_desc& d = h->desc;
  const int blocks = 148 * 16;
  const float sc = syn_normal_scale(sigma);
  if (d.kv_lora_rank > 0) {
    // latent rows: element i of (sequence s, position t) has index (s << 32) + t * W + i
    fill_kv_kernel<<<blocks, 256>>>(kv->k, d.layers, kv->max_seqs, 1, kv->max_ctx, d.kv_lora_rank + d.rope_dim,
                                    length, seed, SYN_KV_LAT, sc, 0);
    CK(cudaGetLastError());
    CK(cudaDeviceSynchronize());
    return MK_OK;
  }
  fill_kv_kernel<<<blocks, 256>>>(kv->k, d.layers, kv->max_seqs, d.n_kv_heads, kv->max_ctx, d.head_dim, length, seed,
                                  SYN_KV_K, sc, 1);
  fill_kv_kernel<<<blocks, 256>>>(kv->v, d.layers, kv->max_seqs, d.n_kv_heads, kv->max_ctx, d.head_dim, length, seed,
                                  SYN_KV_V, sc, 1);
  CK(cudaGetLastError());
  CK(cudaDeviceSynchronize());
  return MK_OK;
}

mk_status mk_kv_copy_out(mk_kv* kv, void* dst) {
  if (!kv || !dst) return MK_ERR_INVALID;
  mk_handle* h = kv->h;
  cudaSetDevice(h->device);
  if (!kv->v) {  // latent cache: one array
    CK(cudaMemcpy(dst, kv->k, (size_t)kv->bytes, cudaMemcpyDeviceToDevice));
    return MK_OK;
  }
  const size_t half = (size_t)kv->bytes / 2;
  const int d = h->desc.head_dim;
  const int64_t rows = (int64_t)(half / 2) / d;
  unpermute_kv_kernel<<<148 * 16, 256>>>(reinterpret_cast<uint16_t*>(dst), kv->k, rows, kv->max_ctx, d);
  unpermute_kv_kernel<<<148 * 16, 256>>>(reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(dst) + half), kv->v,
                                         rows, kv->max_ctx, d);
  CK(cudaGetLastError());
  CK(cudaDeviceSynchronize());
  return MK_OK;
}

mk_status mk_kv_copy_in(mk_kv* kv, const void* src) {
  if (!kv || !src) return MK_ERR_INVALID;
  mk_handle* h = kv->h;
  cudaSetDevice(h->device);
  if (!kv->v) {
    CK(cudaMemcpy(kv->k, src, (size_t)kv->bytes, cudaMemcpyDeviceToDevice));
    return MK_OK;
  }
  const size_t half = (size_t)kv->bytes / 2;
  const int d = h->desc.head_dim;
  const int64_t rows = (int64_t)(half / 2) / d;
  permute_kv_kernel<<<148 * 16, 256>>>(kv->k, reinterpret_cast<const uint16_t*>(src), rows, kv->max_ctx, d);
  permute_kv_kernel<<<148 * 16, 256>>>(kv->v, reinterpret_cast<const uint16_t*>(reinterpret_cast<const uint8_t*>(src) + half),
                                       rows, kv->max_ctx, d);
  CK(cudaGetLastError());
  CK(cudaDeviceSynchronize());
  return MK_OK;
}

// ---------------------------------------------------------------------------
// planner: per-CTA task lists for a step of S sequences x Q positions
// ---------------------------------------------------------------------------
// Row tiles of one matrix over the CTAs: contiguous ranges, the remainder
// tiles placed starting at a rotating CTA so that cumulative bytes balance.
static std::vector<std::pair<int, int>> split_rows(int RT, int ncta, int& rot) {
  std::vector<std::pair<int, int>> r(ncta);
  const int base = RT / ncta, rem = RT % ncta;
  int cur = 0;
  for (int c = 0; c < ncta; ++c) {
    const int extra = (((c - rot) % ncta + ncta) % ncta) < rem ? 1 : 0;
    r[c] = {cur, cur + base + extra};
    cur += base + extra;
  }
  rot = (rot + rem) % ncta;
  return r;
}

// As split_rows, over the CTAs whose `busy` entry is false only (the others
// get empty ranges); all CTAs when every one is busy.
static std::vector<std::pair<int, int>> split_rows_free(int RT, int ncta, int& rot, const std::vector<bool>& busy) {
  std::vector<int> freec;
  for (int c = 0; c < ncta; ++c)
    if (!busy[c]) freec.push_back(c);
  if (freec.empty()) return split_rows(RT, ncta, rot);
  const int n = (int)freec.size();
  std::vector<std::pair<int, int>> r(ncta, {0, 0});
  const int base = RT / n, rem = RT % n;
  int cur = 0;
  for (int i = 0; i < n; ++i) {
    const int extra = (((i - rot) % n + n) % n) < rem ? 1 : 0;
    r[freec[i]] = {cur, cur + base + extra};
    cur += base + extra;
  }
  rot = (rot + rem) % n;
  return r;
}

static Task gemv(int layer, int mat, int rt0, int rt1, int in_kind, int in_buf, int epi, int out_buf, int gain,
                 int wait_ctr, int wait_tgt, int sig) {
  Task t{};
  t.type = T_GEMV;
  t.layer = (int16_t)layer;
  t.mat = mat;
  t.rt0 = rt0;
  t.rt1 = rt1;
  t.in_kind = (int16_t)in_kind;
  t.in_buf = (int16_t)in_buf;
  t.epi = (int16_t)epi;
  t.out_buf = (int16_t)out_buf;
  t.gain = (int16_t)gain;
  t.wait_ctr = wait_ctr;
  t.wait_tgt = wait_tgt;
  t.sig_ctr = sig;
  return t;
}

// The task list of one step shape, built on the host: per-CTA task lists
// flattened into `flat`, CTA c owning flat[off[c], off[c + 1]).
static void build_plan_host(const mk_handle* h, int S, int Q, std::vector<Task>& flat, std::vector<int32_t>& off,
                            int& n_items_out, int& n_pairs_out, int& n_phases_out) {
  (void)Q;
  const mk_model_desc& d = h->desc;
  const int ncta = h->ncta, L = d.layers;
  const bool mla = d.kv_lora_rank > 0;
  const int n_pairs = mla ? S * Q : S * d.n_kv_heads;
  const int n_items = std::max(n_pairs, ncta);
  auto C = [&](int l, int slot) { return l * NCTR_LAYER + slot; };
  std::vector<std::vector<Task>> per(ncta);
  int rot = 0;
  // Phase of every task: the tasks pushed between two calls of next_phase()
  // (one projection's row split over the CTAs, one layer's attention items,
  // ...) form one kernel of the multi-kernel comparison path.
  int phase = -1;
  std::vector<size_t> mark(ncta, 0);
  auto next_phase = [&]() {
    for (int c = 0; c < ncta; ++c) {
      for (size_t i = mark[c]; i < per[c].size(); ++i) per[c][i].phase = (int16_t)phase;
      mark[c] = per[c].size();
    }
    ++phase;
  };
  // embedding gather: every CTA writes its slice of the fp32 residual x and
  // the per-CTA sums of squares the first RMSNorm needs
  next_phase();
  for (int c = 0; c < ncta; ++c) {
    Task t{};
    t.type = T_EMBED;
    t.rt0 = (int)((int64_t)c * d.hidden / ncta);
    t.rt1 = (int)((int64_t)(c + 1) * d.hidden / ncta);
    t.wait_ctr = -1;
    t.sig_ctr = C(L, C_QKV);
    t.ss_dst = 1;
    per[c].push_back(t);
  }
  for (int l = 0; l < L; ++l) {
    const Layer& ly = h->layers[l];
    if (mla) {
      // latent attention: [q | c | k_rope] = W h, absorbed queries per head,
      // attention over the latent rows, per-head value up-projection, W_o
      const int hd = d.head_dim, dr = d.rope_dim, R = d.kv_lora_rank;
      auto rr = split_rows(h->mats[ly.m_qkv].m.RT, ncta, rot);
      next_phase();
      for (int c = 0; c < ncta; ++c) {
        Task t = gemv(l, ly.m_qkv, rr[c].first, rr[c].second, IN_X_NORM, 0, EPI_STORE, B_QKV, 0,
                      l == 0 ? C(L, C_QKV) : C(l - 1, C_DOWN), ncta, C(l, C_QKV));
        t.ss_src = 1;
        per[c].push_back(t);
      }
      rr = split_rows(h->mats[ly.m_ukt].m.RT, ncta, rot);
      next_phase();
      for (int c = 0; c < ncta; ++c) {
        // head g's rows read q_nope of head g: columns g * (dn + dr) of the QKV output
        Task t = gemv(l, ly.m_ukt, rr[c].first, rr[c].second, IN_BUF, B_QKV, EPI_STORE, B_QL, 0, C(l, C_QKV), ncta,
                      C(l, C_UKT));
        t.xg_rt = (int16_t)(R / 16);
        t.xg_stride = hd + dr;
        per[c].push_back(t);
      }
      next_phase();
      for (int i = 0; i < n_items; ++i) {
        // every item writes its partial (M, L, O) and counts itself done
        Task t{};
        t.type = T_MLA;
        t.layer = (int16_t)l;
        t.rt0 = i;
        t.wait_ctr = C(l, C_UKT);
        t.wait_tgt = ncta;
        t.sig_ctr = C(l, C_ATTN);
        per[i % ncta].push_back(t);
      }
      next_phase();
      for (int c = 0; c < ncta; ++c) {
        // the split combine, a slice per CTA
        Task t{};
        t.type = T_MLA_COMB;
        t.layer = (int16_t)l;
        t.wait_ctr = C(l, C_ATTN);
        t.wait_tgt = n_items;
        t.sig_ctr = C(l, C_COMB);
        per[c].push_back(t);
      }
      rr = split_rows(h->mats[ly.m_uv].m.RT, ncta, rot);
      next_phase();
      for (int c = 0; c < ncta; ++c) {
        // head g's rows read the attention output of head g: columns g * R
        Task t = gemv(l, ly.m_uv, rr[c].first, rr[c].second, IN_BUF, B_OL, EPI_STORE, B_ATTN, 0, C(l, C_COMB),
                      ncta, C(l, C_UV));
        t.xg_rt = (int16_t)(hd / 16);
        t.xg_stride = R;
        per[c].push_back(t);
      }
      rr = split_rows(h->mats[ly.m_o].m.RT, ncta, rot);
      next_phase();
      for (int c = 0; c < ncta; ++c) {
        Task t = gemv(l, ly.m_o, rr[c].first, rr[c].second, IN_BUF, B_ATTN, EPI_RESID, 0, 0, C(l, C_UV), ncta,
                      C(l, C_O));
        t.ss_dst = 0;
        per[c].push_back(t);
      }
    }
    // QKV projection (layer 0 reads the embedding rows directly)
    if (!mla) {
      auto rr = split_rows(h->mats[ly.m_qkv].m.RT, ncta, rot);
      next_phase();
      for (int c = 0; c < ncta; ++c) {
        Task t = gemv(l, ly.m_qkv, rr[c].first, rr[c].second, IN_X_NORM, 0, EPI_STORE, B_QKV, 0,
                      l == 0 ? C(L, C_QKV) : C(l - 1, C_DOWN), ncta, C(l, C_QKV));
        t.ss_src = 1;
        per[c].push_back(t);
      }
    }
    // attention items
    next_phase();
    for (int i = 0; i < (mla ? 0 : n_items); ++i) {
      Task t{};
      t.type = T_ATTN;
      t.layer = (int16_t)l;
      t.rt0 = i;
      t.wait_ctr = C(l, C_QKV);
      t.wait_tgt = ncta;
      t.sig_ctr = -1;
      per[i % ncta].push_back(t);
    }
    // output projection + residual
    if (!mla) {
      auto rr = split_rows(h->mats[ly.m_o].m.RT, ncta, rot);
      next_phase();
      for (int c = 0; c < ncta; ++c) {
        Task t = gemv(l, ly.m_o, rr[c].first, rr[c].second, IN_BUF, B_ATTN, EPI_RESID, 0, 0, C(l, C_ATTN), n_items,
                      C(l, C_O));
        t.ss_dst = 0;
        per[c].push_back(t);
      }
    }
    if (d.n_routed == 0) {
      // gate/up + SwiGLU
      {
        auto rr = split_rows(h->mats[ly.m_gu].m.RT, ncta, rot);
        next_phase();
        for (int c = 0; c < ncta; ++c) {
          Task t = gemv(l, ly.m_gu, rr[c].first, rr[c].second, IN_X_NORM, 0, EPI_SWIGLU, B_H, 1, C(l, C_O), ncta,
                        C(l, C_GU));
          t.ss_src = 0;
          per[c].push_back(t);
        }
      }
      // down projection + residual
      {
        auto rr = split_rows(h->mats[ly.m_down].m.RT, ncta, rot);
        next_phase();
        for (int c = 0; c < ncta; ++c) {
          Task t = gemv(l, ly.m_down, rr[c].first, rr[c].second, IN_BUF, B_H, EPI_RESID, 0, 0, C(l, C_GU), ncta,
                        C(l, C_DOWN));
          t.ss_dst = 1;
          per[c].push_back(t);
        }
      }
    } else {
      // Phase order of one MoE layer: router -> shared expert -> routed experts
      // -> down projection over all of them.  The shared expert's weights are
      // streamed while the router's choice is being made; only the routed
      // experts' (and the down) tiles wait for it.
      // The few CTAs that compute the router's rows get no shared-expert rows:
      // they start on the routed experts as soon as the route is known
      // instead of after a shared-expert task as well.
      std::vector<bool> routing(ncta, false);
      {
        auto rr = split_rows(h->mats[ly.m_router].m.RT, ncta, rot);
        for (int c = 0; c < ncta; ++c) routing[c] = rr[c].second > rr[c].first;
        next_phase();
        for (int c = 0; c < ncta; ++c) {
          Task t = gemv(l, ly.m_router, rr[c].first, rr[c].second, IN_X_NORM, 0, EPI_STORE, B_RLOG, 1, C(l, C_O),
                        ncta, C(l, C_ROUTER));
          t.ss_src = 0;
          per[c].push_back(t);
        }
      }
      if (d.n_shared > 0) {
        const MatHost& sh = h->mats[ly.m_shgu];
        auto rr = split_rows_free(sh.m.RT * sh.m.ne, ncta, rot, routing);
        next_phase();
        for (int c = 0; c < ncta; ++c) {
          Task t = gemv(l, ly.m_shgu, rr[c].first, rr[c].second, IN_X_NORM, 0, EPI_SWIGLU_MOE, B_H, 1, C(l, C_O),
                        ncta, C(l, C_GU));
          t.type = T_MOE_GU;
          t.moe = 1;
          t.ss_src = 0;
          per[c].push_back(t);
        }
      }
      next_phase();
      for (int c = 0; c < ncta; ++c) {
        // rows decided on the device from the router's union of experts
        Task t = gemv(l, ly.m_exgu, 0, 0, IN_X_NORM, 0, EPI_SWIGLU_MOE, B_H, 1, C(l, C_ROUTER), ncta, C(l, C_GU));
        t.type = T_MOE_GU;
        t.moe = 2;
        t.ss_src = 0;
        per[c].push_back(t);
      }
      {
        auto rr = split_rows(h->mats[ly.m_exdown].m.RT, ncta, rot);
        const int ngu = (d.n_shared > 0 ? 2 : 1) * ncta;
        next_phase();
        for (int c = 0; c < ncta; ++c) {
          Task t = gemv(l, ly.m_exdown, rr[c].first, rr[c].second, IN_BUF, B_H, EPI_RESID, 0, 0, C(l, C_GU), ngu,
                        C(l, C_DOWN));
          t.type = T_MOE_DOWN;
          t.mat2 = ly.m_shdown;
          t.ss_dst = 1;
          per[c].push_back(t);
        }
      }
    }
  }
  // final norm + LM head + argmax
  {
    auto rr = split_rows(h->mats[h->model.m_lm].m.RT, ncta, rot);
    next_phase();
    for (int c = 0; c < ncta; ++c) {
      Task t = gemv(L - 1, h->model.m_lm, rr[c].first, rr[c].second, IN_X_NORM, 0, EPI_LOGITS, 0, 2,
                    C(L - 1, C_DOWN), ncta, -1);
      t.ss_src = 1;
      per[c].push_back(t);
    }
  }
  flat.clear();
  off.assign(ncta + 1, 0);
  next_phase();  // tags the last phase's tasks
  n_phases_out = phase;
#ifndef MK_TAIL_PREFETCH
#define MK_TAIL_PREFETCH 1
#endif
  // L2 requests one task ahead, issued by the weight producer when it starts
  // the CTA's previous task:
  //  - a CTA that streams one row tile more than the phase's even share ends
  //    the phase late by that row's HBM time: that row is requested, so it
  //    streams from L2;
  //  - (mode 2) a projection that follows attention gets all of the CTA's rows
  //    requested, since attention leaves HBM nearly idle.
  if (MK_TAIL_PREFETCH) {
    for (int c = 0; c < ncta; ++c) {
      std::vector<Task>& v = per[c];
      for (size_t i = 1; i < v.size(); ++i) {
        const Task& t = v[i];
        if (t.type != T_GEMV || t.rt1 <= t.rt0) continue;
        const Mat& m = h->mats[t.mat].m;
        const int16_t prev = v[i - 1].type;
        const bool after_att = prev == T_ATTN || prev == T_MLA || prev == T_MLA_COMB;
        int r0 = -1;
        if (MK_TAIL_PREFETCH >= 2 && after_att) r0 = t.rt0;
        else if (t.rt1 - t.rt0 > m.RT / ncta) r0 = t.rt1 - 1;
        if (r0 < 0) continue;
        Task pf{};
        pf.type = T_PREFETCH;
        pf.layer = t.layer;
        pf.phase = v[i - 1].phase;
        pf.mat = t.mat;
        pf.rt0 = r0;
        pf.rt1 = t.rt1;
        pf.wait_ctr = -1;
        pf.sig_ctr = -1;
        v.insert(v.begin() + (i - 1), pf);
        ++i;  // skip over the task just handled
      }
    }
  }
  for (int c = 0; c < ncta; ++c) {
    off[c] = (int32_t)flat.size();
    flat.insert(flat.end(), per[c].begin(), per[c].end());
  }
  off[ncta] = (int32_t)flat.size();
  // copies the kernel would otherwise load, dependently, at every task start
  for (Task& t : flat) {
    t.m = h->mats[t.mat].m;
    t.gvec = nullptr;
    if (t.in_kind == IN_X_NORM)
      t.gvec = t.gain == 0 ? h->attn_norm[t.layer] : (t.gain == 1 ? h->ffn_norm[t.layer] : h->final_norm);
    // producers of x write x * (the gain of the norm that reads it next) as GEMV fragments
    t.gnext = nullptr;
    t.xf16 = 0;
    if (t.type == T_EMBED) {
      t.gnext = h->attn_norm[0];
    } else if (t.epi == EPI_RESID) {
      if (t.ss_dst == 0) {  // after attention: the FFN (router, shared and routed experts)
        t.gnext = h->ffn_norm[t.layer];
        t.xf16 = (d.n_routed && d.expert_fp8) ? 1 : 0;
      } else {  // after the FFN: the next layer's attention, or the final norm
        t.gnext = t.layer + 1 < L ? h->attn_norm[t.layer + 1] : h->final_norm;
      }
    }
  }
  n_items_out = n_items;
  n_pairs_out = n_pairs;
}

static mk_status get_plan(mk_handle* h, int S, int Q, Plan** out) {
  auto it = h->plans.find(PlanKey{S, Q});
  if (it != h->plans.end()) {
    *out = &it->second;
    return MK_OK;
  }
  std::vector<Task> flat;
  std::vector<int32_t> off;
  int n_items = 0, n_pairs = 0;
  int n_phases = 0;
  build_plan_host(h, S, Q, flat, off, n_items, n_pairs, n_phases);
  Plan p;
  p.n_items = n_items;
  p.n_pairs = n_pairs;
  p.n_tasks = (int)flat.size();
  p.n_phases = n_phases;
  p.host_tasks = flat;
  p.host_off = off;
  CK(cudaMalloc(&p.d_tasks, flat.size() * sizeof(Task)));
  CK(cudaMalloc(&p.d_off, off.size() * sizeof(int32_t)));
  CK(cudaMemcpy(p.d_tasks, flat.data(), flat.size() * sizeof(Task), cudaMemcpyHostToDevice));
  CK(cudaMemcpy(p.d_off, off.data(), off.size() * sizeof(int32_t), cudaMemcpyHostToDevice));
  auto res = h->plans.emplace(PlanKey{S, Q}, p);
  *out = &res.first->second;
  return MK_OK;
}

// ---------------------------------------------------------------------------
// compute entry points
// ---------------------------------------------------------------------------
// The launch arguments of one step.  seq0: the cache sequence that step
// sequence 0 maps to (sequences seq0 .. seq0 + S - 1 are used; the cache base
// is offset, its strides are kept).
static mk_status make_launch(mk_handle* h, mk_kv* kv, int S, int Q, const int32_t* tokens, const int32_t* positions,
                             int32_t pos_const, float* logits, int32_t* argmax, int32_t* accepted, int seq0, Plan** plan_out,
                             Launch* out) {
  if (h->sticky) return fail(h, MK_ERR_STATE, "a previous device error is pending; call mk_reset");
  if (!h->initialised) return fail(h, MK_ERR_STATE, "weights not initialised");
  cudaSetDevice(h->device);
  Plan* plan = nullptr;
  mk_status s = get_plan(h, S, Q, &plan);
  if (s != MK_OK) return s;
  Launch P{};
  P.model = h->d_model;
  P.tasks = plan->d_tasks;
  P.task_off = plan->d_off;
  P.tokens = tokens;
  P.positions = positions;
  P.pos_const = pos_const;
  P.S = S;
  P.Q = Q;
  P.M = S * Q;
  const mk_model_desc& dd = h->desc;
  const size_t seq_elems = dd.kv_lora_rank > 0 ? (size_t)kv->max_ctx * (dd.kv_lora_rank + dd.rope_dim)
                                               : (size_t)dd.n_kv_heads * kv->max_ctx * dd.head_dim;
  P.kv_k = kv->k + (size_t)seq0 * seq_elems;
  P.kv_v = kv->v ? kv->v + (size_t)seq0 * seq_elems : nullptr;
  P.kv_seqs = kv->max_seqs;
  P.kv_ctx = kv->max_ctx;
  P.logits = logits;
  P.argmax = argmax ? argmax : h->argmax_tmp;
  P.accepted = accepted;
  P.router_idx = h->trace_idx;
  P.router_w = h->trace_w;
  for (int b = 0; b < NBUF; ++b) {
    P.buf[b] = h->buf[b];
    P.ld[b] = h->ld[b];
  }
  P.ss_part = h->ss_part;
  P.am_val = h->am_val;
  P.am_idx = h->am_idx;
  P.att_part = h->att_part;
  P.att_rows_max = h->att_rows_max;
  P.ctr = h->ctr;
  P.ctr_layer_stride = NCTR_LAYER;
  P.ctr_pair_base = (h->desc.layers + 1) * NCTR_LAYER;
  P.ctr_lm = P.ctr_pair_base + h->desc.layers * h->max_pairs;
  P.ctr_done = P.ctr_lm + 1;
  P.n_ctr = h->n_ctr;
  P.status = h->status;
  P.timeout_ns = h->stall_ns > 0 ? h->stall_ns : h->timeout_ns;
  P.stall_ctr = h->stall_ns > 0 ? (h->desc.layers * NCTR_LAYER + C_STALL) : -1;
  P.n_items = plan->n_items;
  P.n_pairs = plan->n_pairs;
  P.trace = h->task_trace;
  P.trace_cap = h->task_trace_cap;
  P.task_end = nullptr;
  P.phase_mode = 0;
  h->stall_ns = 0;
  *out = P;
  if (plan_out) *plan_out = plan;
  return MK_OK;
}

static mk_status launch_step(mk_handle* h, mk_kv* kv, int S, int Q, const int32_t* tokens, const int32_t* positions,
                             int32_t pos_const, float* logits, int32_t* argmax, int32_t* accepted, void* stream,
                             int seq0 = 0) {
  Launch P;
  mk_status s = make_launch(h, kv, S, Q, tokens, positions, pos_const, logits, argmax, accepted, seq0, nullptr, &P);
  if (s != MK_OK) return s;
  void* args[] = {&P};
  cudaError_t e = cudaLaunchCooperativeKernel(P.trace ? h->kernel_traced : h->kernel, dim3(h->ncta), dim3(NTHREADS), args,
                                              SMEM_BYTES, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(h, MK_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return MK_OK;
}

mk_status mk_decode_step(mk_handle* h, const int32_t* tokens, const int32_t* positions, int B, mk_kv* kv,
                         float* logits_out, int32_t* argmax_out, void* stream) {
  if (!h) return MK_ERR_INVALID;
  if (!tokens || !positions || !kv || !argmax_out) return fail(h, MK_ERR_INVALID, "null argument");
  if (kv->h != h) return fail(h, MK_ERR_INVALID, "kv cache belongs to another model");
  if (B < 1 || B > h->desc.max_batch || B > kv->max_seqs) return fail(h, MK_ERR_INVALID, "B out of range");
  return launch_step(h, kv, B, 1, tokens, positions, 0, logits_out, argmax_out, nullptr, stream);
}

// Per-phase task ranges of a plan, for the multi-kernel path (empty phases
// are dropped).
static mk_status ensure_phases(mk_handle* h, Plan* p) {
  if (p->d_pbeg) return MK_OK;
  const int ncta = h->ncta;
  std::vector<int32_t> beg, end;
  for (int ph = 0; ph < p->n_phases; ++ph) {
    std::vector<int32_t> b(ncta), e(ncta);
    bool any = false;
    for (int c = 0; c < ncta; ++c) {
      const int lo = p->host_off[c], hi = p->host_off[c + 1];
      int i = lo;
      while (i < hi && p->host_tasks[i].phase < ph) ++i;
      int j = i;
      while (j < hi && p->host_tasks[j].phase == ph) ++j;
      b[c] = i;
      e[c] = j;
      any = any || j > i;
    }
    if (!any) continue;
    beg.insert(beg.end(), b.begin(), b.end());
    end.insert(end.end(), e.begin(), e.end());
  }
  p->n_kphases = (int)(beg.size() / ncta);
  CK(cudaMalloc(&p->d_pbeg, beg.size() * sizeof(int32_t)));
  CK(cudaMalloc(&p->d_pend, end.size() * sizeof(int32_t)));
  CK(cudaMemcpy(p->d_pbeg, beg.data(), beg.size() * sizeof(int32_t), cudaMemcpyHostToDevice));
  CK(cudaMemcpy(p->d_pend, end.data(), end.size() * sizeof(int32_t), cudaMemcpyHostToDevice));
  return MK_OK;
}

mk_status mk_decode_step_multikernel(mk_handle* h, const int32_t* tokens, const int32_t* positions, int B, mk_kv* kv,
                                     float* logits_out, int32_t* argmax_out, void* stream) {
  if (!h) return MK_ERR_INVALID;
  if (!tokens || !positions || !kv || !argmax_out) return fail(h, MK_ERR_INVALID, "null argument");
  if (kv->h != h) return fail(h, MK_ERR_INVALID, "kv cache belongs to another model");
  if (B < 1 || B > h->desc.max_batch || B > kv->max_seqs) return fail(h, MK_ERR_INVALID, "B out of range");
  if (h->task_trace || h->stall_ns > 0)
    return fail(h, MK_ERR_STATE, "the task trace and the stall hook apply to the single-kernel step only");
  CK(cudaSetDevice(h->device));
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const mk_model_desc& d = h->desc;
  if (!h->mk_tokens) {
    mk_status s;
    if ((s = dalloc(h, (void**)&h->mk_tokens, MAXM * sizeof(int32_t))) != MK_OK) return s;
    if ((s = dalloc(h, (void**)&h->mk_pos, MAXM * sizeof(int32_t))) != MK_OK) return s;
    if ((s = dalloc(h, (void**)&h->mk_argmax, MAXM * sizeof(int32_t))) != MK_OK) return s;
    if ((s = dalloc(h, (void**)&h->mk_logits, (size_t)MAXM * d.vocab * sizeof(float))) != MK_OK) return s;
    CK(cudaStreamCreateWithFlags(&h->mk_capture, cudaStreamNonBlocking));
  }
  const GraphKey key{B, kv, logits_out != nullptr, h->trace_idx};
  auto gi = h->graphs.find(key);
  if (gi == h->graphs.end()) {
    Launch P;
    Plan* plan = nullptr;
    mk_status s = make_launch(h, kv, B, 1, h->mk_tokens, h->mk_pos, 0, logits_out ? h->mk_logits : nullptr, h->mk_argmax,
                              nullptr, 0, &plan, &P);
    if (s != MK_OK) return s;
    if ((s = ensure_phases(h, plan)) != MK_OK) return s;
    // one kernel per phase, each allowed to start (programmatic dependent
    // launch) while the previous one drains; recorded once as a graph
    CK(cudaStreamBeginCapture(h->mk_capture, cudaStreamCaptureModeThreadLocal));
    cudaError_t le = cudaSuccess;
    for (int k = 0; k < plan->n_kphases && le == cudaSuccess; ++k) {
      Launch Pk = P;
      Pk.task_off = plan->d_pbeg + (size_t)k * h->ncta;
      Pk.task_end = plan->d_pend + (size_t)k * h->ncta;
      Pk.phase_mode = k + 1 == plan->n_kphases ? 2 : 1;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(h->ncta);
      cfg.blockDim = dim3(NTHREADS);
      cfg.dynamicSmemBytes = SMEM_BYTES;
      cfg.stream = h->mk_capture;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = k > 0 ? 1 : 0;
      void* args[] = {&Pk};
      le = cudaLaunchKernelExC(&cfg, h->kernel, args);
    }
    cudaGraph_t graph = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(h->mk_capture, &graph);
    if (le != cudaSuccess || ce != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      return fail(h, MK_ERR_CUDA, std::string("capture of the phase kernels: ") +
                                      cudaGetErrorString(le != cudaSuccess ? le : ce));
    }
    cudaGraphExec_t exec = nullptr;
    const cudaError_t ie = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ie != cudaSuccess) return fail(h, MK_ERR_CUDA, std::string("graph instantiate: ") + cudaGetErrorString(ie));
    gi = h->graphs.emplace(key, exec).first;
  } else if (h->sticky) {
    return fail(h, MK_ERR_STATE, "a previous device error is pending; call mk_reset");
  }
  CK(cudaMemcpyAsync(h->mk_tokens, tokens, (size_t)B * sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  CK(cudaMemcpyAsync(h->mk_pos, positions, (size_t)B * sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  CK(cudaGraphLaunch(gi->second, st));
  CK(cudaMemcpyAsync(argmax_out, h->mk_argmax, (size_t)B * sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  if (logits_out)
    CK(cudaMemcpyAsync(logits_out, h->mk_logits, (size_t)B * d.vocab * sizeof(float), cudaMemcpyDeviceToDevice, st));
  return MK_OK;
}

mk_status mk_verify(mk_handle* h, const int32_t* tokens8, int n_prop, int32_t position, mk_kv* kv, float* logits_out,
                    int32_t* argmax_out, int32_t* accepted_out, void* stream) {
  if (!h) return MK_ERR_INVALID;
  if (!tokens8 || !kv || !argmax_out || !accepted_out) return fail(h, MK_ERR_INVALID, "null argument");
  if (kv->h != h) return fail(h, MK_ERR_INVALID, "kv cache belongs to another model");
  if (n_prop < 0 || n_prop + 1 > h->desc.max_batch || n_prop + 1 > MAXM)
    return fail(h, MK_ERR_INVALID, "n_prop out of range");
  if (position < 0 || position + n_prop + 1 > kv->max_ctx) return fail(h, MK_ERR_INVALID, "position out of range");
  return launch_step(h, kv, 1, n_prop + 1, tokens8, nullptr, position, logits_out, argmax_out, accepted_out, stream);
}

mk_status mk_prefill(mk_handle* h, const int32_t* tokens, int n, int seq, int32_t start, mk_kv* kv,
                     int32_t* argmax_last, void* stream) {
  if (!h) return MK_ERR_INVALID;
  if (!tokens || !kv) return fail(h, MK_ERR_INVALID, "null argument");
  if (kv->h != h) return fail(h, MK_ERR_INVALID, "kv cache belongs to another model");
  if (n < 1 || seq < 0 || seq >= kv->max_seqs) return fail(h, MK_ERR_INVALID, "n or seq out of range");
  if (start < 0 || (int64_t)start + n > kv->max_ctx) return fail(h, MK_ERR_INVALID, "positions out of range");
  const int chunk = std::min(h->desc.max_batch, MAXM);
  for (int i = 0; i < n; i += chunk) {
    const int q = std::min(chunk, n - i);
    mk_status s = launch_step(h, kv, 1, q, tokens + i, nullptr, start + i, nullptr, h->argmax_tmp, nullptr, stream, seq);
    if (s != MK_OK) return s;
    if (i + q == n && argmax_last)
      CK(cudaMemcpyAsync(argmax_last, h->argmax_tmp + (q - 1), sizeof(int32_t), cudaMemcpyDeviceToDevice,
                         reinterpret_cast<cudaStream_t>(stream)));
  }
  return MK_OK;
}

mk_status mk_spec_generate(mk_handle* h, mk_kv* kv, int32_t anchor, int32_t position, int32_t n_out,
                           mk_draft_fn draft, void* user, int32_t* out_tokens, mk_spec_stats* stats, void* stream) {
  if (!h) return MK_ERR_INVALID;
  if (!kv || !draft || !out_tokens) return fail(h, MK_ERR_INVALID, "null argument");
  if (kv->h != h) return fail(h, MK_ERR_INVALID, "kv cache belongs to another model");
  if (n_out < 1 || position < 0 || anchor < 0 || anchor >= h->desc.vocab)
    return fail(h, MK_ERR_INVALID, "n_out, position or anchor out of range");
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int kcap = std::min(std::min(7, h->desc.max_batch - 1), MAXM - 1);
  std::vector<int32_t> hist;
  hist.reserve((size_t)n_out + 1);
  hist.push_back(anchor);
  mk_spec_stats sst{0, 0, 0, 0};
  int32_t pos = position, emitted = 0;
  int32_t props[8], toks[8], back[17];
  while (emitted < n_out) {
    const int kmax = std::min(kcap, kv->max_ctx - pos - 1);
    if (kmax < 0) return fail(h, MK_ERR_INVALID, "mk_spec_generate: the cache is full");
    int k = draft(user, hist.data(), (int32_t)hist.size(), props, kmax);
    k = std::max(0, std::min(k, kmax));
    toks[0] = anchor;
    for (int j = 0; j < k; ++j) toks[j + 1] = props[j];
    CK(cudaMemcpyAsync(h->spec_dev, toks, (size_t)(k + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, st));
    mk_status s = launch_step(h, kv, 1, k + 1, h->spec_dev, nullptr, pos, nullptr, h->spec_dev + 8, h->spec_dev + 16,
                              stream);
    if (s != MK_OK) return s;
    CK(cudaMemcpyAsync(back, h->spec_dev + 8, 9 * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
    CK(cudaStreamSynchronize(st));
    s = mk_sync_status(h);
    if (s != MK_OK) return s;
    const int a = std::max(0, std::min(back[8], k));
    for (int j = 0; j <= a && emitted < n_out; ++j) {
      const int32_t tkn = j < a ? props[j] : back[a];
      out_tokens[emitted++] = tkn;
      hist.push_back(tkn);
    }
    sst.launches += 1;
    sst.proposed += k;
    sst.accepted += a;
    sst.emitted += a + 1;
    anchor = back[a];
    pos += a + 1;
  }
  if (stats) *stats = sst;
  return MK_OK;
}

mk_status mk_set_router_trace(mk_handle* h, int32_t* idx_dev, float* w_dev) {
  if (!h) return MK_ERR_INVALID;
  h->trace_idx = idx_dev;
  h->trace_w = w_dev;
  return MK_OK;
}

mk_status mk_set_trace(mk_handle* h, int64_t* trace_dev, int32_t max_tasks_per_cta) {
  if (!h || max_tasks_per_cta < 0) return MK_ERR_INVALID;
  h->task_trace = trace_dev;
  h->task_trace_cap = trace_dev ? max_tasks_per_cta : 0;
  return MK_OK;
}

mk_status mk_sync_status(mk_handle* h) {
  if (!h) return MK_ERR_INVALID;
  cudaSetDevice(h->device);
  int32_t st[4] = {0, 0, 0, 0};
  CK(cudaMemcpy(st, h->status, sizeof st, cudaMemcpyDeviceToHost));
  if (st[0] != 0) {
    h->sticky = true;
    h->err = std::string(st[0] == DERR_TIMEOUT ? "device dependency wait timed out" : "device bounds error") +
             " (detail " + std::to_string(st[2]) + ")";
    return (mk_status)st[0];
  }
  return MK_OK;
}

mk_status mk_reset(mk_handle* h) {
  if (!h) return MK_ERR_INVALID;
  cudaSetDevice(h->device);
  CK(cudaDeviceSynchronize());
  CK(cudaMemset(h->status, 0, 16));
  CK(cudaMemset(h->ctr, 0, (size_t)h->n_ctr * 4));
  CK(cudaDeviceSynchronize());
  h->sticky = false;
  return MK_OK;
}

mk_status mk_debug_inject_stall(mk_handle* h, int64_t timeout_ns) {
  if (!h || timeout_ns < 0) return MK_ERR_INVALID;
  h->stall_ns = timeout_ns;
  return MK_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// mk_decode_step_noalloc: the decode step with its scratch in a static array
// ---------------------------------------------------------------------------
// Who needs it: a caller that has handed its whole device-memory budget to its
// own allocator (a framework's caching allocator, a serving engine that sizes
// its KV pool to fill the GPU after warm-up) has nothing left for cudaMalloc,
// and a caller that steps the model from a latency-critical loop cannot let a
// cudaMalloc or cudaFree synchronise the device in the middle of it.
// mk_decode_step itself allocates the device task list of a batch size on the
// first call with that size; this variant keeps the task list and every
// per-step scratch buffer (activations, per-CTA partial sums, split-KV
// partials, inter-CTA counters) in the one array below instead.

static __device__ __align__(256) unsigned char g_noalloc_scratch[MK_NOALLOC_SCRATCH_BYTES];

namespace {
struct NoallocDevice {
  unsigned char* base = nullptr;  // device address of g_noalloc_scratch on this device
  uint64_t plan_owner = 0;        // handle whose task list is in the array (0: none)
  int plan_S = 0;                 // ... and its batch size
  size_t plan_tasks = 0;
  int plan_items = 0, plan_pairs = 0;
};
constexpr int NOALLOC_MAX_DEVICES = 64;
std::mutex g_noalloc_mu;
NoallocDevice g_noalloc_dev[NOALLOC_MAX_DEVICES];
std::atomic<uint64_t> g_noalloc_next_id{1};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
}  // namespace

extern "C" mk_status mk_decode_step_noalloc(mk_handle* h, const int32_t* tokens, const int32_t* positions, int B,
                                            mk_kv* kv, float* logits_out, int32_t* argmax_out, void* stream) {
  if (!h) return MK_ERR_INVALID;
  if (!tokens || !positions || !kv || !argmax_out) return fail(h, MK_ERR_INVALID, "null argument");
  if (kv->h != h) return fail(h, MK_ERR_INVALID, "kv cache belongs to another model");
  if (B < 1 || B > h->desc.max_batch || B > kv->max_seqs) return fail(h, MK_ERR_INVALID, "B out of range");
  if (h->sticky) return fail(h, MK_ERR_STATE, "a previous device error is pending; call mk_reset");
  if (!h->initialised) return fail(h, MK_ERR_STATE, "weights not initialised");
  if (h->device < 0 || h->device >= NOALLOC_MAX_DEVICES) return fail(h, MK_ERR_INVALID, "device ordinal too large");
  CK(cudaSetDevice(h->device));
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const mk_model_desc& d = h->desc;

  // The task list is rebuilt only when another handle or batch size used the
  // array last; it is built on the host (no device memory involved).
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocDevice& nd = g_noalloc_dev[h->device];
  if (!nd.base) {
    // one-time set-up on this device (the device is current): the host-side
    // name of the array is not a device address, so ask the runtime for it
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(h, MK_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch: ") + cudaGetErrorString(e));
    nd.base = static_cast<unsigned char*>(p);
  }
  if (h->noalloc_id == 0) h->noalloc_id = g_noalloc_next_id.fetch_add(1);

  std::vector<Task> flat;
  std::vector<int32_t> off;
  const bool installed = nd.plan_owner == h->noalloc_id && nd.plan_S == B;
  int n_items = nd.plan_items, n_pairs = nd.plan_pairs;
  size_t n_tasks = nd.plan_tasks;
  if (!installed) {
    // Installing copies the task list from pageable host memory that is
    // freed when this call returns; that copy must run now, not be recorded.
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    CK(cudaStreamIsCapturing(st, &cs));
    if (cs != cudaStreamCaptureStatusNone)
      return fail(h, MK_ERR_STATE,
                  "mk_decode_step_noalloc: this handle and batch size must be installed by a call outside stream "
                  "capture first");
    int n_phases = 0;
    build_plan_host(h, B, 1, flat, off, n_items, n_pairs, n_phases);
    n_tasks = flat.size();
  }

  // carve the array: task list, offsets, activation buffers, partials, counters
  const int hw_rows_h = d.n_routed ? d.n_shared + std::min(d.n_routed, MAXM * d.top_k) : 1;
  size_t at = 0;
  const size_t o_tasks = at;
  at = align256(at + n_tasks * sizeof(Task));
  const size_t o_off = at;
  at = align256(at + (size_t)(h->ncta + 1) * sizeof(int32_t));
  size_t o_buf[NBUF];
  for (int b = 0; b < NBUF; ++b) {
    o_buf[b] = at;
    const size_t rows = (b == B_H) ? (size_t)hw_rows_h * MAXM : (size_t)MAXM;
    at = align256(at + rows * h->ld[b] * sizeof(float));
  }
  const size_t o_ss = at;
  at = align256(at + (size_t)2 * h->ncta * MAXM * sizeof(float));
  const size_t o_amv = at;
  at = align256(at + (size_t)h->ncta * MAXM * sizeof(float));
  const size_t o_ami = at;
  at = align256(at + (size_t)h->ncta * MAXM * sizeof(int32_t));
  const size_t o_att = at;
  at = align256(at + (size_t)n_items * h->att_rows_max * (h->att_dpart + 4) * sizeof(float));
  const size_t o_ctr = at;
  at = align256(at + (size_t)h->n_ctr * sizeof(uint32_t));
  if (at > (size_t)MK_NOALLOC_SCRATCH_BYTES)
    return fail(h, MK_ERR_INVALID,
                "mk_decode_step_noalloc: this model and batch need " + std::to_string(at) +
                    " bytes of scratch; the static array holds " + std::to_string((size_t)MK_NOALLOC_SCRATCH_BYTES));
  unsigned char* base = nd.base;

  if (!installed) {
    // pageable host source: the call returns once the source has been read
    nd.plan_owner = 0;
    CK(cudaMemcpyAsync(base + o_tasks, flat.data(), n_tasks * sizeof(Task), cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(base + o_off, off.data(), off.size() * sizeof(int32_t), cudaMemcpyHostToDevice, st));
    nd.plan_owner = h->noalloc_id;
    nd.plan_S = B;
    nd.plan_tasks = n_tasks;
    nd.plan_items = n_items;
    nd.plan_pairs = n_pairs;
  }
  // The inter-CTA counters must start at zero.  A completed step leaves them
  // zero, but one that stopped on a device error does not, and the array is
  // shared by every handle on the device: clear them before every step.
  // Nothing else needs clearing: every other region is written before it is read.
  CK(cudaMemsetAsync(base + o_ctr, 0, (size_t)h->n_ctr * sizeof(uint32_t), st));

  Launch P{};
  P.model = h->d_model;
  P.tasks = reinterpret_cast<const Task*>(base + o_tasks);
  P.task_off = reinterpret_cast<const int32_t*>(base + o_off);
  P.tokens = tokens;
  P.positions = positions;
  P.pos_const = 0;
  P.S = B;
  P.Q = 1;
  P.M = B;
  P.kv_k = kv->k;
  P.kv_v = kv->v;
  P.kv_seqs = kv->max_seqs;
  P.kv_ctx = kv->max_ctx;
  P.logits = logits_out;
  P.argmax = argmax_out;
  P.accepted = nullptr;
  P.router_idx = h->trace_idx;
  P.router_w = h->trace_w;
  for (int b = 0; b < NBUF; ++b) {
    P.buf[b] = reinterpret_cast<float*>(base + o_buf[b]);
    P.ld[b] = h->ld[b];
  }
  P.ss_part = reinterpret_cast<float*>(base + o_ss);
  P.am_val = reinterpret_cast<float*>(base + o_amv);
  P.am_idx = reinterpret_cast<int32_t*>(base + o_ami);
  P.att_part = reinterpret_cast<float*>(base + o_att);
  P.att_rows_max = h->att_rows_max;
  P.ctr = reinterpret_cast<uint32_t*>(base + o_ctr);
  P.ctr_layer_stride = NCTR_LAYER;
  P.ctr_pair_base = (d.layers + 1) * NCTR_LAYER;
  P.ctr_lm = P.ctr_pair_base + d.layers * h->max_pairs;
  P.ctr_done = P.ctr_lm + 1;
  P.n_ctr = h->n_ctr;
  P.status = h->status;  // device errors are read with mk_sync_status, as for mk_decode_step
  P.timeout_ns = h->timeout_ns;
  P.stall_ctr = -1;
  P.n_items = n_items;
  P.n_pairs = n_pairs;
  P.trace = h->task_trace;
  P.trace_cap = h->task_trace_cap;
  void* args[] = {&P};
  const cudaError_t e = cudaLaunchCooperativeKernel(P.trace ? h->kernel_traced : h->kernel, dim3(h->ncta), dim3(NTHREADS), args,
                                                    SMEM_BYTES, st);
  if (e != cudaSuccess) return fail(h, MK_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return MK_OK;
}

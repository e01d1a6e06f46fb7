// mk_kernel.cu - the persistent decode-step kernel for sm_100a.
//
// One launch evaluates a whole decoder step ("700 TPS on Kimi K3: A Case for
// TPU Megakernels", section "Why megakernels?": the whole decoder step is one
// program, so a weight load is not tied to the kernel that consumes it).
//
// B200 mapping:
//   - grid = one CTA per SM (cooperative launch guarantees co-residency);
//   - each CTA runs a host-planned task list (GEMV row tiles, attention items);
//   - warp 8 is a producer: it walks the same task list and streams every
//     weight tile and KV-cache row the CTA will consume into a 2-stage shared
//     memory ring with cp.async.bulk (TMA) + mbarrier complete_tx.  Weights do
//     not depend on activations, so the producer never waits on another CTA:
//     it runs ahead across task and layer boundaries (the cross-layer
//     prefetch of section "Our Kimi K3 megakernel");
//   - warps 0..7 consume: they wait on a global dependency counter (acquire),
//     compute with mma.sync m16n8k16 on the tile in shared memory, write
//     their outputs and release-increment the next counter.  Activations are
//     fp32; tensor-core operands carry them as a bf16 hi + lo pair (about 16
//     significant bits), so accumulation matches fp32 GEMV to ~1e-5.
//   - every wait is bounded by %globaltimer; on expiry a CTA records the
//     error, raises a global abort flag that all CTAs poll, drains its own
//     in-flight bulk copies and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "mk_internal.h"

// Tracing (per-task records and per-region cycle counts for the trace tool)
// lives in separate instances of every kernel: mk_kernel_traced.cu compiles
// this file again with MK_TRACE 1, into its own namespace.  The untraced
// instances, which serve every ordinary step, carry none of its code: the
// checks and counters cost about 4 % of the step time when compiled in.
#ifndef MK_TRACE
#define MK_TRACE 0
#endif
#if MK_TRACE
#define MK_KNS traced
#else
#define MK_KNS plain
#endif

namespace mk {
namespace MK_KNS {

constexpr int NTSD = NTS > 0 ? NTS : 1;  // TMEM slot count as a divisor (the slot code is dead when NTS == 0)

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bulk (non-tensor) TMA copy global -> shared, completion on an mbarrier,
// with an L2 policy (weights and cache rows are streamed once per step).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
// Bring `bytes` (a multiple of 16) at `src` into L2, with no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void bar_consumers() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_volatile_i32(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t atom_add_acqrel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ uint2 lds64(const void* p) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ uint32_t lds32(const void* p) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
  return v;
}
// Two 8x8 bf16 matrices, transposed: with rows = positions of a row-major
// [position][dim] tile, thread (g, tq) receives the mma B fragment
// {V[2tq][g], V[2tq+1][g]} of matrix 0 (rows 0-7) and of matrix 1 (rows 8-15).
// Lanes 0-15 give the row addresses (16-byte aligned).
__device__ __forceinline__ void ldsm_x2_trans(const void* row_addr, uint32_t& b0, uint32_t& b1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(b0), "=r"(b1)
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ uint32_t lds16(const void* p) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t cnt) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)), "r"(cnt)
               : "memory");
}

// Tensor memory (tcgen05).  One warp allocates the CTA's columns at start and
// frees them at exit.  Addresses are (lane << 16) | column.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Shared-memory matrix descriptor of 128 rows x 16 bytes stored contiguously
// (no swizzle; 8-row core matrices 128 B apart).
__device__ __forceinline__ uint64_t sdesc_rows16(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
         (1ull << 46);
}
// Copy 128 rows x 16 bytes of shared memory into TMEM lanes 0..127, 4 columns.
__device__ __forceinline__ void tmem_cp_rows16(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}
// Arrive (once) on `bar` when every earlier tcgen05 operation of this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// This warp's 32 lanes x 4 columns: lane l receives the 16 bytes of TMEM lane (quarter base + l).
__device__ __forceinline__ uint4 tmem_ld16(uint32_t taddr) {
  uint4 v;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(taddr)
               : "memory");
  return v;
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint4 a, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&d)[4], uint4 a, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<uint32_t*>(&h);
}
// fp32 pair -> bf16 hi pair + bf16 residual pair.
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  float2 hf = __bfloat1622float2(h);
  __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = *reinterpret_cast<uint32_t*>(&l);
}
__device__ __forceinline__ void split_f16(float a, float b, uint32_t& hi, uint32_t& lo) {
  __half2 h = __floats2half2_rn(a, b);
  float2 hf = __half22float2(h);
  __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = *reinterpret_cast<uint32_t*>(&l);
}

// Activation buffers that feed only GEMVs and no other phase (the attention
// output, the SwiGLU hidden units, the latent attention output) are written
// by their producers directly in the GEMV's B-operand layout: per 16-value
// col tile 64 bytes = for each quad lane tq, {hi(k 2tq, 2tq+1), hi(k 2tq+8,
// 2tq+9), lo(..), lo(..)} (bf16 split, or f16 for fp8 weights), so that the
// consuming GEMV copies them in and skips the conversion.
__device__ __forceinline__ int frag_off(int r, int k, int KTn) {
  // byte offset of element (row r, col k) in an A-fragment tile array [mt][KTn][32][8 x 2B]
  const int mi = r >> 4, rr = r & 15, kt = k >> 4, kk = k & 15;
  const int ln = (rr & 7) * 4 + ((kk & 7) >> 1);
  const int e = (kk & 1) + 2 * (rr >> 3) + 4 * (kk >> 3);
  return (((mi * KTn + kt) * 32 + ln) * 8 + e) * 2;
}

__device__ __forceinline__ bool frag_buf(int b) { return b == B_ATTN || b == B_H || b == B_OL; }
__device__ __forceinline__ void st_frag(float* row, int k, float v, bool f16) {
  uint8_t* p = reinterpret_cast<uint8_t*>(row) + (size_t)(k >> 4) * 64 + ((k & 7) >> 1) * 16 + ((k >> 3) & 1) * 4 +
               (k & 1) * 2;
  uint16_t hb, lb;
  if (!f16) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
    hb = *reinterpret_cast<const uint16_t*>(&h);
    lb = *reinterpret_cast<const uint16_t*>(&l);
  } else {
    const __half h = __float2half_rn(v);
    const __half l = __float2half_rn(v - __half2float(h));
    hb = *reinterpret_cast<const uint16_t*>(&h);
    lb = *reinterpret_cast<const uint16_t*>(&l);
  }
  *reinterpret_cast<uint16_t*>(p) = hb;
  *reinterpret_cast<uint16_t*>(p + 8) = lb;
}
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t fp8x2_to_f16x2(uint32_t two) {
  __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xFFFFu), __NV_E4M3);
  return (uint32_t)r.x | ((uint32_t)r.y << 16);
}
__device__ __forceinline__ uint4 fp8_frag_to_f16(uint2 v) {
  uint4 a;
  a.x = fp8x2_to_f16x2(v.x);
  a.y = fp8x2_to_f16x2(v.x >> 16);
  a.z = fp8x2_to_f16x2(v.y);
  a.w = fp8x2_to_f16x2(v.y >> 16);
  return a;
}

// ---------------------------------------------------------------------------
// shared state
// ---------------------------------------------------------------------------
struct Misc {
  uint64_t full[NSTAGE];
  uint64_t empty[NSTAGE];   // consumers (NCW) + the mover (1); for TMEM chunks the mover's NCW + its copy commit
  uint64_t tfull[NTS > 0 ? NTS : 1];   // TMEM slot written (copy commit)
  uint64_t tempty[NTS > 0 ? NTS : 1];  // TMEM slot read by every consumer warp
  uint32_t tmem_base;
  int32_t cdesc[NSTAGE];    // per ring stage: 2 KB groups to move to TMEM (0: stays in shared memory; -1: end)
  uint64_t xfull[XSLOTS];   // activation slice landed (bulk copy)
  uint64_t xempty[XSLOTS];
  float scale[MAXM];
  float xscale[XSLOTS][MAXM];  // RMSNorm scale of the rows of the window in each activation slot
  float gscale[MAXM];          // ... of the row group the consumers are on
  volatile int abort;
  int flag;
  int pad[2];
  // MoE routing tables, one per role (each role computes its own copy)
  int rt_u[3];
  int route_layer;  // layer + 1 of the route the activation producer last published
  int16_t rt_ex[3][64];
  int16_t rt_sel[3][MAXM * 8];  // each row's picks in top-k order, per role
  float rt_selw[MAXM][8];       // consumers: their renormalised weights
  float rt_w[64][MAXM];      // consumers: weight of (union slot, row)
  // per-task trace accumulators (consumer thread 0)
  long long tr_wf, tr_wx, tr_bytes, tr_route;
  long long tr_frag, tr_mma, tr_epi, tr_rel, tr_loop, tr_pre, tr_post, tr_sig;
  int tr_chunks;
  // shared-memory copies, so that reading them costs no global (or spilled
  // local) round trip: the model description (every role), and the task the
  // consumer warps are on
  Model cmodel;
  Task ctask;
  // latent attention: bulk copy of the absorbed queries (completion, uses so far)
  uint64_t qbar;
  uint32_t qpar;
};

static_assert(sizeof(Misc) <= MISC_BYTES, "Misc must fit its shared-memory region");

// The GEMV's cross-warp reduction uses the first RED_BYTES of the attention
// scratch; fp8 block-scale tables (two alternating, FP8_SCALE_TAB floats each)
// follow it.
constexpr int RED_BYTES = NCW * RMAX * 32 * 16;
constexpr int FP8_SCALE_OFF = RED_BYTES;
constexpr int FP8_SCALE_TAB = 512;  // floats: 2 halves x 2 row blocks x 128 column blocks
static_assert(FP8_SCALE_OFF + 2 * FP8_SCALE_TAB * 4 <= ATT_BYTES, "fp8 scale tables fit the attention scratch");

struct Ctx {
  const Launch* P;
  const Model* md;
  Misc* ms;
  uint8_t* ring;
  uint8_t* xring;
  uint8_t* att;
  uint8_t* newkv;
  int ncta;
  uint32_t tmem;  // TMEM base address of the weight slots
};

__device__ __forceinline__ bool global_abort(const Launch& P) { return ld_volatile_i32(P.status + 1) != 0; }

__device__ __forceinline__ int task_end_of(const Launch& P) {
  return P.phase_mode ? P.task_end[blockIdx.x] : P.task_off[blockIdx.x + 1];
}
// Multi-kernel path: the activations and counters a phase reads were written
// by earlier phase kernels; with programmatic dependent launch this kernel
// may start before they finish, so every role that reads them waits here for
// the preceding grid (the weight producer does not: weights are constant).
__device__ __forceinline__ void phase_dependency_wait(const Launch& P) {
  if (P.phase_mode) asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ void raise_error(const Launch& P, Misc* ms, int code, int detail) {
  atomicCAS(P.status, 0, code);
  atomicExch(P.status + 2, detail);
  atomicExch(P.status + 1, 1);
  ms->abort = 1;
}

// ---------------------------------------------------------------------------
// chunk iteration (identical in producer and consumers)
// ---------------------------------------------------------------------------
struct ChunkIt {
  int rt1, KT, tb, gsz, xcap;
  int g0, nr, KC, WC, c0, nc, wb;  // wb: first col tile of the current activation window
  bool tm;                         // the group's chunks go through the TMEM stage
  __device__ __forceinline__ void set_group() {
    nr = min(RMAX, rt1 - g0);
    if (gsz > 0) {
      int nb = (g0 / gsz + 1) * gsz;
      nr = min(nr, nb - g0);
    }
    KC = min(min(KT, TILE_CAP / (nr * tb)), min(NCW * CPW, xcap));
    if (NTS > 0 && KC < KT && KC >= 4) KC &= ~3;  // chunk widths in whole 4-tile groups (TMEM stage)
    WC = (xcap / KC) * KC;  // activation window: a whole number of chunks
    // a chunk moves to TMEM in 2 KB groups of 4 consecutive tiles; with a
    // width that is a multiple of 4, the tiles of col j (j = warp mod 8) sit
    // in lane quarter warp mod 4, the only one the warp can read
    tm = NTS > 0 && tb == TILE_BF16 && (KT & 3) == 0 && (KC & 3) == 0;
  }
  // xcap: most col tiles whose activation slice (M rows) fits one x slot
  __device__ __forceinline__ bool init(int rt0_, int rt1_, int KT_, int tb_, int gsz_, int xcap_) {
    rt1 = rt1_;
    KT = KT_;
    tb = tb_;
    gsz = gsz_;
    xcap = xcap_;
    g0 = rt0_;
    if (g0 >= rt1) return false;
    set_group();
    c0 = 0;
    wb = 0;
    nc = min(KC, KT);
    return true;
  }
  __device__ __forceinline__ bool next() {
    c0 += KC;
    if (c0 >= KT) {
      g0 += nr;
      if (g0 >= rt1) return false;
      set_group();
      c0 = 0;
      wb = 0;
    } else if (c0 - wb >= WC) {
      wb = c0;
    }
    nc = min(KC, KT - c0);
    return true;
  }
  __device__ __forceinline__ bool group_done() const { return c0 + KC >= KT; }
  __device__ __forceinline__ uint32_t bytes() const { return (uint32_t)(nr * nc * tb); }
  // activation windows (no division: tracked incrementally)
  __device__ __forceinline__ int w0() const { return wb; }
  __device__ __forceinline__ int wn() const { return min(WC, KT - wb); }
  __device__ __forceinline__ bool win_first() const { return c0 == wb; }
  __device__ __forceinline__ bool win_last() const { return c0 + KC >= KT || c0 + KC - wb >= WC; }
};

// Activation element size and the x-slot column cap of a GEMV task.
__device__ __forceinline__ int x_esize(const Task& t) { return 4; }
__device__ __forceinline__ int x_cap(const Task& t, int M) {
  return (XSLOT_BYTES / M - XROW_PAD) / (16 * x_esize(t));
}
// row stride of an activation window in the x slot
__device__ __forceinline__ int x_rowbytes(const Task& t, int wc) { return wc * 16 * x_esize(t) + XROW_PAD; }

// Attention item -> (pair, split index, number of splits, first item of pair).
struct Item {
  int pair, j, ns, first;
};
__device__ __forceinline__ int pair_first_item(int pair, int n_pairs, int n_items) {
  return n_pairs >= n_items ? pair : (int)(((int64_t)pair * n_items + n_pairs - 1) / n_pairs);
}
__device__ __forceinline__ Item decode_item(int item, int n_pairs, int n_items) {
  Item it;
  if (n_pairs >= n_items) {
    it.pair = item;
    it.j = 0;
    it.ns = 1;
    it.first = item;
  } else {
    it.pair = (int)(((int64_t)item * n_pairs) / n_items);
    it.first = (int)(((int64_t)it.pair * n_items + n_pairs - 1) / n_pairs);
    int nxt = (int)(((int64_t)(it.pair + 1) * n_items + n_pairs - 1) / n_pairs);
    it.ns = nxt - it.first;
    it.j = item - it.first;
  }
  return it;
}

__device__ __forceinline__ int seq_pos0(const Launch& P, int s) {
  return P.positions ? __ldg(P.positions + s) : P.pos_const;
}

// K / V rows in shared memory, unpadded: a chunk's rows are contiguous in the
// cache and arrive as one bulk copy each for K and V (per-row copies into
// padded rows avoid bank conflicts but cost more in copy issue than they save).
__device__ __forceinline__ int att_pitch(int d) { return d * 2; }

// ---------------------------------------------------------------------------
// MoE routing: softmax over the router logits of each activation row, top-k by
// logit (ties to the lower expert index), weights renormalised over the k
// picks; the union of the picked experts in ascending expert order.  One
// warp; every role that needs the result computes it itself from the same
// logits with the same code, so all roles agree.
// ---------------------------------------------------------------------------
enum RouteRole { RR_CONS = 0, RR_PROD = 1, RR_XPROD = 2 };  // RR_XPROD's tables also serve the consumers

__device__ __noinline__ int moe_route(const Launch& P, const Model& md, int layer, Misc* ms, int role, bool want_w,
                                      bool trace) {
  // Compact on purpose (a runtime loop over rows, one out-of-line copy for
  // the three roles): it runs once per layer, so its instruction fetch is
  // cold every time and dominates its cost.
  const int lane = threadIdx.x & 31;
  const int E = md.E, K = md.K, M = P.M;
  const float* rl = P.buf[B_RLOG];
  const int ld = P.ld[B_RLOG];
  int16_t* sel = ms->rt_sel[role];
  uint32_t ubits = 0;  // bit q: expert lane + 32 q picked by some row
#pragma unroll 1
  for (int mm = 0; mm < M; ++mm) {
    float v[8];
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      v[q] = e < E ? __ldcg(rl + (size_t)mm * ld + e) : -INFINITY;
      mx = fmaxf(mx, v[q]);
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) sum += expf(v[q] - mx);  // -inf lanes add 0
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    float psum = 0.f, my_p = 0.f;
#pragma unroll 1
    for (int j = 0; j < K; ++j) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int e = lane + 32 * q;
        if (v[q] > bv || (v[q] == bv && e < be)) {
          bv = v[q];
          be = e;
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      const float pj = expf(bv - mx) / sum;
      psum += pj;
      if (lane == j) {
        sel[mm * 8 + j] = (int16_t)be;
        my_p = pj;
      }
      if ((be & 31) == lane) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q == (be >> 5)) v[q] = -INFINITY;
        ubits |= 1u << (be >> 5);
      }
    }
    if (want_w && lane < K) ms->rt_selw[mm][lane] = my_p / psum;
  }
  // union in ascending expert order
  int U = 0;
  int16_t* ex = ms->rt_ex[role];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint32_t b = __ballot_sync(0xffffffffu, (ubits >> q) & 1u);
    if ((ubits >> q) & 1u) ex[U + __popc(b & ((1u << lane) - 1u))] = (int16_t)(lane + 32 * q);
    U += __popc(b);
  }
  if (lane == 0) ms->rt_u[role] = U;
  __syncwarp();
  if (want_w) {
    for (int i = lane; i < 64 * MAXM; i += 32) ms->rt_w[i / MAXM][i % MAXM] = 0.f;
    __syncwarp();
    for (int i = lane; i < M * K; i += 32) {
      const int mm = i / K, j = i - mm * K;
      const int e = sel[mm * 8 + j];
      const float w = ms->rt_selw[mm][j];
      int slot = 0;
      while (slot < U && ex[slot] != e) ++slot;
      ms->rt_w[slot][mm] = w;
      if (trace && P.router_idx) {
        P.router_idx[((size_t)layer * M + mm) * K + j] = e;
        P.router_w[((size_t)layer * M + mm) * K + j] = w;
      }
    }
    __syncwarp();
  }
  return U;
}

// The pieces of a GEMV-like task: row groups (<= RMAX row tiles, not crossing
// an expert boundary for virtual expert rows) x K segments (one per expert for
// the MoE down projection).
struct Pieces {
  int rt1, gsz, nseg;
  int g0, nr, seg;
  __device__ __forceinline__ void set_nr() {
    nr = min(RMAX, rt1 - g0);
    if (gsz > 0) nr = min(nr, (g0 / gsz + 1) * gsz - g0);
  }
  __device__ __forceinline__ bool init(int rt0_, int rt1_, int gsz_, int nseg_) {
    rt1 = rt1_;
    gsz = gsz_;
    nseg = nseg_;
    g0 = rt0_;
    seg = 0;
    if (g0 >= rt1 || nseg <= 0) return false;
    set_nr();
    return true;
  }
  __device__ __forceinline__ bool next() {
    if (++seg < nseg) return true;
    seg = 0;
    g0 += nr;
    if (g0 >= rt1) return false;
    set_nr();
    return true;
  }
};

// Matrix base, local row tile and activation source of the current piece.
struct PieceSrc {
  const uint8_t* w;
  const float* scales;
  int lg0;    // first row tile inside the piece's matrix
  int xbuf;   // activation buffer
  int xrow0;  // first activation row in it (expert slot * MAXM for the MoE down projection)
  int xcol0;  // first activation column (per-head groups of the latent-attention projections)
};

template <int MOE>
__device__ __forceinline__ PieceSrc piece_src(const Model& md, const Task& t, const Mat& m, const Mat& m2,
                                              const int16_t* ex, const Pieces& pc) {
  PieceSrc r;
  r.lg0 = pc.g0;
  r.xrow0 = 0;
  r.xcol0 = t.xg_rt > 0 ? (pc.g0 / t.xg_rt) * t.xg_stride : 0;
  // normed inputs: the fragment copy of x * gain (the RMS scale is applied after the GEMV)
  r.xbuf = t.in_kind == IN_X_NORM ? (m.fp8 ? (int)B_XF16 : (int)B_XF) : (int)t.in_buf;
  r.w = m.w;
  r.scales = m.scales;
  if (MOE && t.type == T_MOE_GU) {
    const int slot = pc.g0 / m.RT;
    const int e = t.moe == 1 ? slot : ex[slot];
    r.w = m.w + (size_t)e * m.estride;
    r.scales = m.scales ? m.scales + (size_t)e * m.sstride : nullptr;
    r.lg0 = pc.g0 - slot * m.RT;
  } else if (MOE && t.type == T_MOE_DOWN) {
    const int ns = md.NS;
    const Mat& mm = pc.seg < ns ? m2 : m;
    const int e = pc.seg < ns ? pc.seg : ex[pc.seg - ns];
    r.w = mm.w + (size_t)e * mm.estride;
    r.scales = mm.scales ? mm.scales + (size_t)e * mm.sstride : nullptr;
    r.xbuf = B_H;
    r.xrow0 = pc.seg * MAXM;
  }
  return r;
}

// Row range, expert-group size and K-segment count of a GEMV-like task.
template <int MOE>
__device__ __forceinline__ void task_rows(const Model& md, const Task& t, const Mat& m, int U, int& rt0, int& rt1,
                                          int& gsz, int& nseg) {
  rt0 = t.rt0;
  rt1 = t.rt1;
  gsz = t.xg_rt > 0 ? t.xg_rt : 0;
  nseg = 1;
  if (MOE && t.type == T_MOE_GU) {
    gsz = m.RT;
    if (t.moe == 2) {
      const int T = U * m.RT;
      rt0 = (int)(((int64_t)blockIdx.x * T) / gridDim.x);
      rt1 = (int)(((int64_t)(blockIdx.x + 1) * T) / gridDim.x);
    }
  } else if (MOE && t.type == T_MOE_DOWN) {
    nseg = md.NS + U;
  }
}

template <int MOE>
__device__ __forceinline__ bool task_needs_route(const Task& t) {
  return MOE && ((t.type == T_MOE_GU && t.moe == 2) || t.type == T_MOE_DOWN);
}
template <int MOE>
__device__ __forceinline__ bool gemv_like(const Task& t) {
  return t.type == T_GEMV || (MOE && (t.type == T_MOE_GU || t.type == T_MOE_DOWN));
}

// ---------------------------------------------------------------------------
// producer warp
// ---------------------------------------------------------------------------
// Reserve ring slot `it` for `bytes` (lane 0 waits for the consumers to free
// it, then arms the full barrier).  Returns false on abort.
__device__ bool prod_reserve(const Ctx& C, uint32_t it, uint32_t bytes, long long& blocked, int desc = 0,
                             bool end = false) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) {
    const int s = it % NSTAGE;
    const long long c0 = clock64();
    if (it >= (uint32_t)NSTAGE) {
      const uint32_t par = ((it / NSTAGE) + 1) & 1;
      uint64_t t0 = 0;
      uint32_t spins = 0;
      while (!mbar_try_wait(&C.ms->empty[s], par)) {
        __nanosleep(64);
        if (++spins >= 64) {
          spins = 0;
          if (C.ms->abort || global_abort(*C.P)) { ok = 0; break; }
          uint64_t now = globaltimer();
          if (t0 == 0) t0 = now;
          else if (now - t0 > (uint64_t)C.P->timeout_ns * 2) {
            raise_error(*C.P, C.ms, DERR_TIMEOUT, 0x10000 | s);
            ok = 0;
            break;
          }
        }
      }
    }
    blocked += clock64() - c0;
    if (ok) {
      // the mover reads the stage's descriptor once the stage's phase completes
      if (NTS > 0) C.ms->cdesc[s] = end ? -1 : desc;
      if (end) mbar_arrive(&C.ms->full[s]);
      else mbar_arrive_expect_tx(&C.ms->full[s], bytes);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

// Bounded wait of one warp on a dependency counter (lane 0 polls with
// acquire); later bulk (async-proxy) reads must observe the generic-proxy
// writes the acquire made visible, hence the proxy fence.
__device__ bool warp_wait_counter(const Ctx& C, int idx, uint32_t target, int code) {
  const Launch& P = *C.P;
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) {
    const uint32_t* p = P.ctr + idx;
    uint64_t t0 = 0;
    uint32_t spins = 0;
    while ((int)(ld_acquire(p) - target) < 0) {
      if (C.ms->abort) { ok = 0; break; }
      __nanosleep(64);
      if (++spins >= 16) {
        spins = 0;
        if (global_abort(P)) { C.ms->abort = 1; ok = 0; break; }
        uint64_t now = globaltimer();
        if (t0 == 0) t0 = now;
        else if (now - t0 > (uint64_t)P.timeout_ns * 2) {
          raise_error(P, C.ms, DERR_TIMEOUT, code | idx);
          ok = 0;
          break;
        }
      }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

// One unit of streamed data, in the order the consumers take it.
struct Chunk {
  int kind;  // 1: GEMV tiles, 2: attention K/V rows, 3: latent cache rows (kb, n rows of d values)
  const uint8_t* w;
  int KT, tb, g0, nr, c0, nc;
  int tm;    // GEMV tiles that go through the TMEM stage
  const uint16_t* kb;
  const uint16_t* vb;
  int n, d;
};

// Walks a CTA's task list and yields its chunks in consumption order (the
// enumeration the consumers use).  Routed-expert tasks first wait for the
// router's counter: their tiles are the only ones that depend on activations.
template <bool MLA, int MOE>
struct ChunkStream {
  int ti, end, state;  // state 0: next task, 1: GEMV-like pieces, 2: attention, 3: latent attention
  Task t;
  Mat m, m2;
  Pieces pc;
  ChunkIt ci;
  PieceSrc src;
  int tb, xcap;
  const uint16_t* kb;
  const uint16_t* vb;
  int t0, b, d;
  __device__ void init(int beg, int end_) {
    ti = beg;
    end = end_;
    state = 0;
  }
  // returns 1 with a chunk, 0 at the end of the list, -1 on abort
  __device__ int next(const Ctx& C, Chunk& c) {
    const Launch& P = *C.P;
    const Model& md = *C.md;
    while (true) {
      if (state == 1) {
        c.kind = 1;
        c.w = src.w;
        c.KT = m.KT;
        c.tb = tb;
        c.g0 = ci.g0;
        c.nr = ci.nr;
        c.c0 = ci.c0;
        c.nc = ci.nc;
        c.tm = ci.tm ? 1 : 0;
        if (!ci.next()) {
          if (!pc.next()) {
            state = 0;
          } else {
            src = piece_src<MOE>(md, t, m, m2, C.ms->rt_ex[RR_PROD], pc);
            ci.init(src.lg0, src.lg0 + pc.nr, m.KT, tb, 0, xcap);
          }
        }
        return 1;
      }
      if (!MLA && state == 2) {
        if (t0 < b) {
          c.kind = 2;
          c.tm = 0;
          c.kb = kb + (size_t)t0 * d;
          c.vb = vb + (size_t)t0 * d;
          c.n = min(ATT_CT, b - t0);
          c.d = d;
          t0 += ATT_CT;
          return 1;
        }
        state = 0;
      }
      if (MLA && state == 3) {
        if (t0 < b) {
          c.kind = 3;
          c.tm = 0;
          c.kb = kb + (size_t)t0 * d;
          c.n = min(mla_ct(md.R, md.dr), b - t0);
          c.d = d;
          t0 += mla_ct(md.R, md.dr);
          return 1;
        }
        state = 0;
      }
      if (ti >= end) return 0;
      t = P.tasks[ti++];
      if (gemv_like<MOE>(t)) {
        m = t.m;
        m2 = (MOE && t.type == T_MOE_DOWN && t.mat2 >= 0) ? md.mats[t.mat2] : m;
        tb = m.fp8 ? TILE_FP8 : TILE_BF16;
        xcap = x_cap(t, P.M);
        int U = 0;
        if (task_needs_route<MOE>(t)) {
          if (!warp_wait_counter(C, t.layer * P.ctr_layer_stride + C_ROUTER, (uint32_t)gridDim.x, 0x70000)) return -1;
          U = moe_route(P, md, t.layer, C.ms, RR_PROD, false, false);
        }
        int rt0, rt1, gsz, nseg;
        task_rows<MOE>(md, t, m, U, rt0, rt1, gsz, nseg);
        if (pc.init(rt0, rt1, gsz, nseg)) {
          src = piece_src<MOE>(md, t, m, m2, C.ms->rt_ex[RR_PROD], pc);
          ci.init(src.lg0, src.lg0 + pc.nr, m.KT, tb, 0, xcap);
          state = 1;
        }
      } else if (!MLA && t.type == T_ATTN) {
        const Item itm = decode_item(t.rt0, P.n_pairs, P.n_items);
        const int s = itm.pair / md.Hkv, g = itm.pair % md.Hkv;
        const int T0 = seq_pos0(P, s);
        t0 = (int)(((int64_t)itm.j * T0) / itm.ns);
        b = (int)(((int64_t)(itm.j + 1) * T0) / itm.ns);
        d = md.d;
        const size_t head = (((size_t)t.layer * P.kv_seqs + s) * md.Hkv + g) * (size_t)P.kv_ctx;
        kb = P.kv_k + head * d;
        vb = P.kv_v + head * d;
        state = 2;
      } else if (t.type == T_PREFETCH) {
        // the rows this CTA streams beyond the phase's even share: requested
        // into L2 one phase early, so that the CTA with an extra row tile does
        // not set the phase's end at the HBM rate
        if ((threadIdx.x & 31) == 0) {
          const size_t rowb = (size_t)t.m.KT * (t.m.fp8 ? TILE_FP8 : TILE_BF16);
          bulk_prefetch_l2(t.m.w + (size_t)t.rt0 * rowb, (uint32_t)((t.rt1 - t.rt0) * rowb));
        }
      } else if (MLA && t.type == T_MLA) {
        // cached positions [0, T0) of the query row's sequence, split like GQA
        const Item itm = decode_item(t.rt0, P.n_pairs, P.n_items);
        const int s = itm.pair / P.Q;
        const int T0 = seq_pos0(P, s);
        t0 = (int)(((int64_t)itm.j * T0) / itm.ns);
        b = (int)(((int64_t)(itm.j + 1) * T0) / itm.ns);
        d = md.R + md.dr;
        kb = P.kv_k + ((size_t)t.layer * P.kv_seqs + s) * (size_t)P.kv_ctx * d;
        state = 3;
      }
    }
  }
};

template <bool MLA, int MOE>
__device__ void producer(const Ctx& C) {
  const Launch& P = *C.P;
  const int lane = threadIdx.x & 31;
  const uint64_t pol = policy_evict_first();
  uint32_t it = 0;
  const int beg = P.task_off[blockIdx.x], end = task_end_of(P);
  long long blocked = 0;
  const uint64_t t_first = globaltimer();
  const long long c_first = clock64();
  ChunkStream<MLA, MOE> is;
  is.init(beg, end);
  Chunk c;
  while (is.next(C, c) > 0) {
    uint8_t* dst = C.ring + (size_t)(it % NSTAGE) * STAGE_BYTES;
    uint64_t* bar = &C.ms->full[it % NSTAGE];
    if (c.kind == 1) {
      const uint32_t tbytes = (uint32_t)(c.nr * c.nc * c.tb);
      if (!prod_reserve(C, it, tbytes, blocked, c.tm ? (c.nr * c.nc) >> 2 : 0)) goto drain;
      if (lane < c.nr) {
        const uint8_t* srcp = c.w + ((size_t)(c.g0 + lane) * c.KT + c.c0) * c.tb;
        bulk_g2s(dst + (size_t)lane * c.nc * c.tb, srcp, (uint32_t)(c.nc * c.tb), bar, pol);
      }
    } else if (MLA) {
      // latent rows, one copy each into padded shared-memory rows
      const int pitch = c.d * 2 + 16;
      const uint32_t rb = (uint32_t)(c.d * 2);
      if (!prod_reserve(C, it, rb * (uint32_t)c.n, blocked)) goto drain;
      for (int r = lane; r < c.n; r += 32) bulk_g2s(dst + (size_t)r * pitch, c.kb + (size_t)r * c.d, rb, bar, pol);
    } else {
      // the cache rows of this chunk are contiguous: one copy for K, one for V
      const int pitch = att_pitch(c.d);
      const uint32_t rb = (uint32_t)(c.n * c.d * 2);
      if (!prod_reserve(C, it, 2 * rb, blocked)) goto drain;
      if (lane == 0) bulk_g2s(dst, c.kb, rb, bar, pol);
      if (lane == 1) bulk_g2s(dst + (size_t)ATT_CT * pitch, c.vb, rb, bar, pol);
    }
    __syncwarp();
    ++it;
  }
  // end of the stream for the mover
  if (NTS > 0) {
    if (!prod_reserve(C, it, 0, blocked, 0, true)) goto drain;
    __syncwarp();
    ++it;
  }
drain:
  if (MK_TRACE && lane == 0 && P.trace && P.trace_cap > 0) {
    int64_t* rec = P.trace + (size_t)blockIdx.x * P.trace_cap * TRACE_FIELDS;
    rec[12] = blocked;
    rec[13] = it;
    rec[14] = (int64_t)t_first;
    rec[15] = (int64_t)globaltimer();
    if (P.trace_cap > 1) {
      // effective SM clock over the producer's lifetime: cycles and ns
      rec[TRACE_FIELDS + 12] = clock64() - c_first;
      rec[TRACE_FIELDS + 13] = (int64_t)(globaltimer() - t_first);
    }
  }
  // Wait (bounded) for every bulk copy this CTA issued, so none is in flight
  // when the CTA exits, whether it finished or aborted.
  if (lane == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      if (it <= (uint32_t)s) continue;
      const uint32_t last = it - 1 - ((it - 1 - s) % NSTAGE);
      const uint32_t par = (last / NSTAGE) & 1;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&C.ms->full[s], par)) {
        if (globaltimer() - t0 > (uint64_t)P.timeout_ns) break;
      }
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// TMEM mover warp
// ---------------------------------------------------------------------------
// Follows the ring in order.  A stage whose descriptor says "TMEM" is copied
// (tcgen05.cp, 2 KB per instruction) into the next TMEM slot once that slot
// has been read by every consumer warp; the copy's completion both fills the
// slot (tfull) and releases the stage to the producer (empty).  Any other
// stage is only acknowledged: the consumers read it in place and release it.
// Bounded waits end on the global abort flag or the time limit.
__device__ bool mover_wait(const Ctx& C, uint64_t* bar, uint32_t par, int code) {
  uint64_t t0 = 0;
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, par)) {
    if (++spins >= 64) {
      spins = 0;
      if (C.ms->abort || global_abort(*C.P)) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) t0 = now;
      else if (now - t0 > (uint64_t)C.P->timeout_ns * 2) {
        raise_error(*C.P, C.ms, DERR_TIMEOUT, code);
        return false;
      }
    }
  }
  return true;
}

__device__ void mover(const Ctx& C) {
  if (NTS == 0) return;
  if ((threadIdx.x & 31) != 0) return;
  uint32_t i = 0, tc = 0;
  while (true) {
    const int s = i % NSTAGE;
    if (!mover_wait(C, &C.ms->full[s], (i / NSTAGE) & 1, 0x90000 | s)) break;
    const int d = C.ms->cdesc[s];
    if (d < 0) break;
    if (d > 0) {
      const int t = tc % NTSD;
      if (tc >= (uint32_t)NTSD && !mover_wait(C, &C.ms->tempty[t], ((tc / NTSD) + 1) & 1, 0xA0000 | t)) break;
      tc_fence_after();
      const uint32_t src = smem_u32(C.ring + (size_t)s * STAGE_BYTES);
      const uint32_t dst = C.tmem + (uint32_t)(t * TSLOT_COLS);
      for (int g = 0; g < d; ++g) tmem_cp_rows16(dst + 4 * g, sdesc_rows16(src + 2048 * g));
      tc_commit(&C.ms->empty[s]);  // the stage is free once the copies have read it
      tc_commit(&C.ms->tfull[t]);  // the slot is full
      mbar_arrive_cnt(&C.ms->empty[s], NCW);
      ++tc;
    } else {
      mbar_arrive(&C.ms->empty[s]);
    }
    ++i;
  }
  // every copy issued has completed before the CTA frees its tensor memory
  if (tc > 0) {
    const uint32_t last = tc - 1;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(&C.ms->tfull[last % NTSD], (last / NTSD) & 1)) {
      if (globaltimer() - t0 > (uint64_t)C.P->timeout_ns) break;
    }
  }
}

// ---------------------------------------------------------------------------
// activation producer warp
// ---------------------------------------------------------------------------
// Walks the same task list.  For each GEMV task it waits for the task's
// dependency (acquire), then streams the activation slice of every chunk
// (M rows x the chunk's columns) into the x ring with bulk copies, so the
// consumers never wait on a global-memory round trip inside a task.
// Convert an activation window in place into ready mma B fragments: col tile
// jj of row m (16 fp32, 64 B) becomes, for each quad lane tq, 16 B =
// {hi(k 2tq,2tq+1), hi(k 2tq+8,2tq+9), lo(..), lo(..)} of x * rms_scale * gain
// (bf16 split; f16 for fp8 weights).  All consumer threads share the work.
// Only inputs that no producer writes in fragment layout need it (the
// absorbed-query GEMV of latent attention reads the raw QKV output).  Out of
// line: keeps the GEMV inner loops small (one CTA runs every phase of the
// step, so their instruction footprint matters).
__device__ __noinline__ void convert_window_coop(uint8_t* dst, int rb, int M, int wn, int w0, bool has_gain,
                                                 const uint16_t* gain, const float* scale, bool f16) {
  for (int e = threadIdx.x; e < M * wn; e += NCT) {
    const int mm = e / wn, jj = e - mm * wn;
    float4* p4 = reinterpret_cast<float4*>(dst + (size_t)mm * rb + (size_t)jj * 64);
    float v[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = p4[q];
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
    if (has_gain) {
      const float sc = scale[mm];
      const uint4* gp = reinterpret_cast<const uint4*>(gain + (size_t)(w0 + jj) * 16);
      const uint4 ga = __ldg(gp), gb = __ldg(gp + 1);
      const uint32_t gw[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[2 * q] = v[2 * q] * sc * bf16lo(gw[q]);
        v[2 * q + 1] = v[2 * q + 1] * sc * bf16hi(gw[q]);
      }
    }
    uint4 o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (!f16) {
        split_bf16(v[2 * q], v[2 * q + 1], o[q].x, o[q].z);
        split_bf16(v[2 * q + 8], v[2 * q + 9], o[q].y, o[q].w);
      } else {
        split_f16(v[2 * q], v[2 * q + 1], o[q].x, o[q].z);
        split_f16(v[2 * q + 8], v[2 * q + 9], o[q].y, o[q].w);
      }
    }
    uint4* o4 = reinterpret_cast<uint4*>(p4);
#pragma unroll
    for (int q = 0; q < 4; ++q) o4[q] = o[q];
  }
  // the slot is written again by bulk copies (async proxy) once released
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ bool xprod_reserve(const Ctx& C, uint32_t ix, uint32_t bytes) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) {
    const int s = ix % XSLOTS;
    if (ix >= (uint32_t)XSLOTS) {
      const uint32_t par = ((ix / XSLOTS) + 1) & 1;
      uint64_t t0 = 0;
      uint32_t spins = 0;
      while (!mbar_try_wait(&C.ms->xempty[s], par)) {
        __nanosleep(64);
        if (++spins >= 64) {
          spins = 0;
          if (C.ms->abort || global_abort(*C.P)) { ok = 0; break; }
          uint64_t now = globaltimer();
          if (t0 == 0) t0 = now;
          else if (now - t0 > (uint64_t)C.P->timeout_ns * 2) {
            raise_error(*C.P, C.ms, DERR_TIMEOUT, 0x40000 | s);
            ok = 0;
            break;
          }
        }
      }
    }
    if (ok) mbar_arrive_expect_tx(&C.ms->xfull[s], bytes);
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

template <int MOE>
__device__ void xproducer(const Ctx& C) {
  const Launch& P = *C.P;
  const Model& md = *C.md;
  const int lane = threadIdx.x & 31;
  const int M = P.M;
  const uint64_t pol = policy_evict_last();
  uint32_t ix = 0;
  const int beg = P.task_off[blockIdx.x], end = task_end_of(P);
  if (P.stall_ctr >= 0) return;
  phase_dependency_wait(P);
  for (int ti = beg; ti < end; ++ti) {
    const Task t = P.tasks[ti];
    if (!gemv_like<MOE>(t)) continue;
    const Mat m = t.m;
    const Mat m2 = (MOE && t.type == T_MOE_DOWN && t.mat2 >= 0) ? md.mats[t.mat2] : m;
    const int tb = m.fp8 ? TILE_FP8 : TILE_BF16;
    const int xcap = x_cap(t, M);
    if (t.wait_ctr >= 0 && !warp_wait_counter(C, t.wait_ctr, (uint32_t)t.wait_tgt, 0x30000)) goto drain;
    int U = 0;
    if (task_needs_route<MOE>(t)) {
      // a one-kernel-per-phase launch starts the down projection with fresh
      // shared memory, so it computes the layer's route again
      if (t.type == T_MOE_GU || P.phase_mode) {
        // the layer's route, with the routed weights, for this warp and for
        // the consumers (published through shared memory)
        U = moe_route(P, md, t.layer, C.ms, RR_XPROD, true, blockIdx.x == 0 && t.type == T_MOE_GU);
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          *reinterpret_cast<volatile int*>(&C.ms->route_layer) = t.layer + 1;
        }
      } else {
        U = C.ms->rt_u[RR_XPROD];  // the down projection of the same layer: same route
      }
    }
    int rt0, rt1, gsz, nseg;
    task_rows<MOE>(md, t, m, U, rt0, rt1, gsz, nseg);
    Pieces pc;
    if (!pc.init(rt0, rt1, gsz, nseg)) continue;
    // RMSNorm scale of every activation row (fixed-order reduction of the
    // per-CTA sums of squares), computed once the task's first activation
    // copy is in flight
    float scale[MAXM];
    const bool has_gain = t.in_kind == IN_X_NORM;
    bool have_scale = !has_gain;
#pragma unroll
    for (int mm = 0; mm < MAXM; ++mm) scale[mm] = 1.f;
    do {
      const PieceSrc src = piece_src<MOE>(md, t, m, m2, C.ms->rt_ex[RR_XPROD], pc);
      ChunkIt ci;
      ci.init(src.lg0, src.lg0 + pc.nr, m.KT, tb, 0, xcap);
      do {
        if (!ci.win_first()) continue;
        const int rb = x_rowbytes(t, ci.WC);
        const int wn = ci.wn(), w0 = ci.w0();
        const uint32_t rowdata = (uint32_t)(wn * 64);
        const int sl = ix % XSLOTS;
        if (!xprod_reserve(C, ix, (uint32_t)M * rowdata)) goto drain;
        uint8_t* dst = C.xring + (size_t)sl * XSLOT_BYTES;
        if (lane < M) {
          const uint8_t* xsrc = reinterpret_cast<const uint8_t*>(
              P.buf[src.xbuf] + (size_t)(src.xrow0 + lane) * P.ld[src.xbuf] + src.xcol0 + ci.c0 * 16);
          bulk_g2s(dst + (size_t)lane * rb, xsrc, rowdata, &C.ms->xfull[sl], pol);
        }
        if (!have_scale) {
#pragma unroll
          for (int mm = 0; mm < MAXM; ++mm) {
            if (mm < M) {
              const float* srcs = P.ss_part + (size_t)t.ss_src * gridDim.x * MAXM;
              float ss = 0.f;
              for (int c = lane; c < (int)gridDim.x; c += 32) ss += __ldcg(srcs + c * MAXM + mm);
              for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
              scale[mm] = rsqrtf(ss / (float)md.H + md.eps);
            }
          }
          have_scale = true;
        }
        // the slot's second arrival publishes the rows' scales (release)
        if (lane == 0) {
#pragma unroll
          for (int q = 0; q < MAXM; ++q) C.ms->xscale[sl][q] = scale[q];
          mbar_arrive(&C.ms->xfull[sl]);
        }
        __syncwarp();
        ++ix;  // the consumers convert the window, where it needs converting
      } while (ci.next());
    } while (pc.next());
  }
drain:
  if (lane == 0) {
    for (int s = 0; s < XSLOTS; ++s) {
      if (ix <= (uint32_t)s) continue;
      const uint32_t last = ix - 1 - ((ix - 1 - s) % XSLOTS);
      const uint32_t par = (last / XSLOTS) & 1;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&C.ms->xfull[s], par)) {
        if (globaltimer() - t0 > (uint64_t)P.timeout_ns) break;
      }
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// consumer helpers
// ---------------------------------------------------------------------------
// Wait for ring slot `it` to be filled.  On an abort the wait ends without
// the data; callers keep walking their task list (so every consumer thread
// passes the same barriers) and the outputs of the step are discarded.
__device__ __forceinline__ void wait_full(const Ctx& C, uint32_t it) {
  const int s = it % NSTAGE;
  const uint32_t par = (it / NSTAGE) & 1;
  const bool tr = MK_TRACE && C.P->trace && threadIdx.x == 0;
  const long long c0 = tr ? clock64() : 0;
  if (tr) C.ms->tr_chunks++;
  if ((threadIdx.x & 31) == 0) {
    uint32_t spins = 0;
    uint64_t t0 = 0;
    while (!mbar_try_wait(&C.ms->full[s], par)) {
      if (++spins >= 64) {
        spins = 0;
        if (C.ms->abort) break;
        uint64_t now = globaltimer();
        if (t0 == 0) t0 = now;
        else if (now - t0 > (uint64_t)C.P->timeout_ns * 2) {
          raise_error(*C.P, C.ms, DERR_TIMEOUT, 0x20000 | s);
          break;
        }
      }
    }
  }
  __syncwarp();
  // the other lanes observe the completed phase (async-proxy writes visible)
  if (!C.ms->abort) while (!mbar_try_wait(&C.ms->full[s], par)) {}
  if (tr) C.ms->tr_wf += clock64() - c0;
}

__device__ __forceinline__ void release_stage(const Ctx& C, uint32_t it) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&C.ms->empty[it % NSTAGE]);
}

// Wait for TMEM slot of TMEM chunk `tc` to be filled (the mover's copy commit).
__device__ __forceinline__ void wait_tfull(const Ctx& C, uint32_t tc) {
  const int t = tc % NTSD;
  const uint32_t par = (tc / NTSD) & 1;
  const bool tr = MK_TRACE && C.P->trace && threadIdx.x == 0;
  const long long c0 = tr ? clock64() : 0;
  if (tr) C.ms->tr_chunks++;
  if ((threadIdx.x & 31) == 0) {
    uint32_t spins = 0;
    uint64_t t0 = 0;
    while (!mbar_try_wait(&C.ms->tfull[t], par)) {
      if (++spins >= 64) {
        spins = 0;
        if (C.ms->abort) break;
        uint64_t now = globaltimer();
        if (t0 == 0) t0 = now;
        else if (now - t0 > (uint64_t)C.P->timeout_ns * 2) {
          raise_error(*C.P, C.ms, DERR_TIMEOUT, 0xB0000 | t);
          break;
        }
      }
    }
  }
  __syncwarp();
  if (!C.ms->abort) while (!mbar_try_wait(&C.ms->tfull[t], par)) {}
  tc_fence_after();
  if (tr) C.ms->tr_wf += clock64() - c0;
}

// Thread 0 decides, every consumer thread gets the same answer (a barrier
// on each side of the read keeps the flag slot free for the next use).
__device__ __forceinline__ int broadcast_from0(const Ctx& C, int v) {
  if (threadIdx.x == 0) C.ms->flag = v;
  bar_consumers();
  const int r = C.ms->flag;
  bar_consumers();
  return r;
}

// Wait until counter `idx` reaches `target` (thread 0 polls with acquire).
// Ends early, without the dependency, when the step is being aborted.
__device__ void wait_counter(const Ctx& C, int idx, uint32_t target) {
  const Launch& P = *C.P;
  if (threadIdx.x == 0) {
    const uint32_t* p = P.ctr + idx;
    uint64_t t0 = 0;
    uint32_t spins = 0;
    while ((int)(ld_acquire(p) - target) < 0) {
      if (C.ms->abort) break;
      __nanosleep(64);
      if (++spins >= 16) {
        spins = 0;
        if (global_abort(P)) { C.ms->abort = 1; break; }
        uint64_t now = globaltimer();
        if (t0 == 0) t0 = now;
        else if (now - t0 > (uint64_t)P.timeout_ns) {
          raise_error(P, C.ms, DERR_TIMEOUT, idx);
          break;
        }
      }
    }
  }
  bar_consumers();
}

// The consumers' writes of the task precede thread 0's release through the
// barrier (causality order is transitive; the release is cumulative), so the
// release alone publishes them at gpu scope: no separate full fence.
__device__ __forceinline__ void signal_counter(const Ctx& C, int idx) {
  bar_consumers();
  if (threadIdx.x == 0 && !C.ms->abort) red_release_add(C.P->ctr + idx, 1u);
}

// ---------------------------------------------------------------------------
// GEMV task: out rows [rt0, rt1) of W (16-row tiles) times M activation rows
// ---------------------------------------------------------------------------
__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

// Wait for activation slot `ix`: converted by the activation producer
// (`landed` false), or only landed, for the consumers to convert (true).
__device__ __forceinline__ void wait_x(const Ctx& C, uint32_t ix) {
  const int s = ix % XSLOTS;
  const uint32_t par = (ix / XSLOTS) & 1;
  uint64_t* bar = &C.ms->xfull[s];
  const bool tr = MK_TRACE && C.P->trace && threadIdx.x == 0;
  const long long c0 = tr ? clock64() : 0;
  if ((threadIdx.x & 31) == 0) {
    uint32_t spins = 0;
    uint64_t t0 = 0;
    while (!mbar_try_wait(bar, par)) {
      if (++spins >= 64) {
        spins = 0;
        if (C.ms->abort) break;
        uint64_t now = globaltimer();
        if (t0 == 0) t0 = now;
        else if (now - t0 > (uint64_t)C.P->timeout_ns * 2) {
          raise_error(*C.P, C.ms, DERR_TIMEOUT, 0x58000 | s);
          break;
        }
      }
    }
  }
  __syncwarp();
  if (!C.ms->abort) while (!mbar_try_wait(bar, par)) {}
  if (tr) C.ms->tr_wx += clock64() - c0;
}

// Per-lane constants of a GEMV task.
struct GemvLane {
  int warp, lane, g, tq, M, rowbytes;
  bool has_gain, trc;
  bool conv;              // the windows need converting (false: the input buffer holds fragments)
  const uint16_t* gain;   // norm gain of the task's input
  // K segments taken in one call (the MoE down projection: shared experts,
  // then the routed experts of the union, each Ie wide); the fp8 block
  // scales of segment s are those of shared expert s (s < NS) or of routed
  // expert ex[s - NS]
  int nseg, NS;
  const float* sc_sh;
  const float* sc_rt;
  int64_t ss_sh, ss_rt;
  const int16_t* ex;
};

// All chunks of one row group [g0, g0 + NR): each warp takes col tiles
// j = warp + 8 i of every chunk, builds the activation fragment (hi/lo) of
// each and runs NR independent accumulator chains; the per-warp partial sums
// are left in `red` for the cross-warp reduction.
// acc += block scale * raw for col block cb of the rows of row tiles g0.. (raw
// is cleared).  Gate / up interleaved tiles take the gate scale for rows
// 0-7 and the up scale for rows 8-15 of each tile.
template <int NR>
__device__ __forceinline__ void fp8_apply_scales(const Mat& m, const float* sct, int rb0, int nrb, int g0, int cb,
                                                 float (&raw)[NR][4], float (&acc)[NR][4], int nrr) {
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    if (r >= nrr) continue;
    const int rt = g0 + r;
    float s_top, s_bot;
    if (m.gu) {
      const int rb = (rt >> 4) - rb0;
      s_top = sct[rb * m.nbc + cb];
      s_bot = sct[(nrb + rb) * m.nbc + cb];
    } else {
      s_top = s_bot = sct[((rt >> 3) - rb0) * m.nbc + cb];
    }
    acc[r][0] += s_top * raw[r][0];
    acc[r][1] += s_top * raw[r][1];
    acc[r][2] += s_bot * raw[r][2];
    acc[r][3] += s_bot * raw[r][3];
    raw[r][0] = raw[r][1] = raw[r][2] = raw[r][3] = 0.f;
  }
}

// Packed accumulators (M <= 4): column n < M holds the hi-part products of
// activation row n, column n + M its lo-part products.  A lane holds columns
// 2tq, 2tq + 1 of rows g and g + 8 (c0 c1 / c2 c3); the partner of column n
// sits in lane tq' = (n + M) / 2 of the same quad, slot (n + M) & 1.  After
// the fold, columns >= M are zero as in the unpacked layout.
__device__ __forceinline__ void fold_lo_cols(float (&c)[4], int M, int tq, int lane) {
  const bool odd = M & 1;
  const int s0 = (lane & ~3) | ((tq + (M >> 1)) & 3);
  const int s1 = (lane & ~3) | ((tq + ((M + 1) >> 1)) & 3);
  const float u0 = __shfl_sync(0xffffffffu, odd ? c[1] : c[0], s0);
  const float u1 = __shfl_sync(0xffffffffu, odd ? c[0] : c[1], s1);
  const float u2 = __shfl_sync(0xffffffffu, odd ? c[3] : c[2], s0);
  const float u3 = __shfl_sync(0xffffffffu, odd ? c[2] : c[3], s1);
  const bool k0 = 2 * tq < M, k1 = 2 * tq + 1 < M;
  c[0] = k0 ? c[0] + u0 : 0.f;
  c[1] = k1 ? c[1] + u1 : 0.f;
  c[2] = k0 ? c[2] + u2 : 0.f;
  c[3] = k1 ? c[3] + u3 : 0.f;
}

// The GEMV row-group loop: one out-of-line instance per row count (small
// instruction footprint) or inlined into the task body (no call frame).
#ifndef MK_GEMV_INLINE
#define MK_GEMV_INLINE 1
#endif
#ifndef MK_FP8_UNROLL
#define MK_FP8_UNROLL 1
#endif
// Row-group instances compiled (8: one per row count 1..RMAX; 4: 1, 2, 4 and
// RMAX; 1: RMAX only), bf16 and fp8 weights: fewer instances, less code.
#ifndef MK_GEMV_SET
#define MK_GEMV_SET 8
#endif
#ifndef MK_FP8_SET
#define MK_FP8_SET 8
#endif
constexpr int FP8_UNROLL = MK_FP8_UNROLL;
#if MK_GEMV_INLINE
#define MK_GEMV_ATTR __forceinline__
#else
#define MK_GEMV_ATTR __noinline__
#endif
template <int NR, bool FP8>
__device__ MK_GEMV_ATTR void gemv_group(const Ctx& Cr, ChunkIt& cir, const Mat& mr, const GemvLane& Lr, uint32_t& itr,
                                        uint32_t& ixr, uint32_t& tcr, float* red, bool accum) {
  // register copies (the arguments live in the caller's frame)
  const Ctx C = Cr;
  const Mat m0 = mr;
  const GemvLane L = Lr;
  ChunkIt ci = cir;
  uint32_t it = itr, ix = ixr, tc = tcr;
  // row tiles of this group: NR, or fewer when one instance serves several
  // row counts (rows nrr..NR-1 then load and multiply nothing)
  constexpr bool exact = NR == 1 || (FP8 ? MK_FP8_SET == 8 : MK_GEMV_SET == 8);
  const int nrr = exact ? NR : ci.nr;
  float acc[NR][4];
#pragma unroll
  for (int r = 0; r < NR; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
  const int lane = L.lane, g = L.g, tq = L.tq;
  // M <= 4: the hi and lo parts of activation row n feed mma columns n and
  // n + M, so one mma per tile covers both; the column pairs are summed once
  // at the end.  Otherwise column n is row n and each tile takes two mmas.
  const bool pk = L.M <= MAXM / 2;
  const bool lo_col = pk && g >= L.M;
  const int gr = lo_col ? g - L.M : g;
  const bool xok = g < (pk ? 2 * L.M : L.M);  // other columns are zero
  long long tc0 = 0, tl0 = L.trc ? clock64() : 0;
  const ChunkIt ci0 = ci;
  // fp8: the block scales of the group's rows (every column block) staged in
  // shared memory; read through L1 they miss for every chunk (the L1 beside a
  // 227 KB carve-out holds little).  A call over several K segments (the MoE
  // down projection: one per expert) stages every segment's rows in one pass
  // when they fit (one global round trip instead of one per segment), else
  // one segment at a time in two tables alternating by segment.
  const int rb0 = FP8 ? (m0.gu ? (ci0.g0 >> 4) : (ci0.g0 >> 3)) : 0;
  const int nrb = FP8 ? (m0.gu ? ((ci0.g0 + nrr - 1) >> 4) : ((ci0.g0 + nrr - 1) >> 3)) - rb0 + 1 : 1;
  const int sc_per = nrb * m0.nbc;
  const bool sc_all = FP8 && L.nseg > 1 && !m0.gu && L.nseg * sc_per <= 2 * FP8_SCALE_TAB;
  float* const sc_base = reinterpret_cast<float*>(C.att + FP8_SCALE_OFF);
  if (sc_all) {
    for (int i = threadIdx.x; i < L.nseg * sc_per; i += NCT) {
      const int sg = i / sc_per, j = i - sg * sc_per;
      const float* scs = sg < L.NS ? L.sc_sh + (size_t)sg * L.ss_sh : L.sc_rt + (size_t)L.ex[sg - L.NS] * L.ss_rt;
      sc_base[i] = __ldg(scs + (size_t)rb0 * m0.nbc + j);
    }
    bar_consumers();
  }
  for (int seg = 0; seg < L.nseg; ++seg) {
  if (seg > 0) ci = ci0;
  Mat m = m0;
  if (FP8 && L.nseg > 1)
    m.scales = seg < L.NS ? L.sc_sh + (size_t)seg * L.ss_sh : L.sc_rt + (size_t)L.ex[seg - L.NS] * L.ss_rt;
  const float* sct = sc_all ? sc_base + seg * sc_per : sc_base + (seg & 1) * FP8_SCALE_TAB;
  if (FP8 && !sc_all) {
    const int per = sc_per, n = (m.gu ? 2 : 1) * per;
    float* dst = const_cast<float*>(sct);
    for (int i = threadIdx.x; i < n; i += NCT) {
      const int hf = i >= per ? 1 : 0;
      dst[i] = __ldg(m.scales + (size_t)hf * m.nbr * m.nbc + (size_t)rb0 * m.nbc + (i - hf * per));
    }
    bar_consumers();
  }
  while (true) {
    const uint8_t* slot = C.xring + (size_t)(ix % XSLOTS) * XSLOT_BYTES;
    if (ci.win_first()) {
      if (!L.conv) {
        wait_x(C, ix);  // the window arrives in fragment layout: nothing to do
        // normed input: the rows' RMS scales, applied to the group's sums
        if (L.has_gain && ci.c0 == 0 && L.warp == 0 && lane < MAXM)
          C.ms->gscale[lane] = C.ms->xscale[ix % XSLOTS][lane];
      } else {
        wait_x(C, ix);
        const long long tv0 = L.trc ? clock64() : 0;
        convert_window_coop(const_cast<uint8_t*>(slot), L.rowbytes, L.M, ci.wn(), ci.w0(), L.has_gain, L.gain,
                            C.ms->xscale[ix % XSLOTS], FP8);
        bar_consumers();
        if (L.trc) C.ms->tr_frag += clock64() - tv0;
      }
    }
    const bool tm = !FP8 && ci.tm;
    if (tm) wait_tfull(C, tc);
    else wait_full(C, it);
    const uint8_t* stage = C.ring + (size_t)(it % NSTAGE) * STAGE_BYTES;
    const uint8_t* xs = slot + (size_t)gr * L.rowbytes + (size_t)(ci.c0 - ci.w0()) * 64 + tq * 16;
    const int nc = ci.nc;
    if (L.trc) tc0 = clock64();
    // kept rolled: the instruction working set of the whole kernel must stay
    // small (one CTA executes every phase of every layer)
    if (tm) {
      // tile (r, j) = tile r * nc + j of the chunk sits in 4-column group
      // (r * nc + j) / 4, lane quarter j mod 4 = warp mod 4
      const uint32_t tbase = C.tmem + (uint32_t)((tc % NTSD) * TSLOT_COLS) + ((uint32_t)(L.warp & 3) << 21);
#pragma unroll 1
      for (int j = L.warp; j < nc; j += NCW) {
        const uint4 xf = xok ? lds128(xs + j * 64) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t b0 = lo_col ? xf.z : xf.x, b1 = lo_col ? xf.w : xf.y;
        uint4 a[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r)
          if (r < nrr) a[r] = tmem_ld16(tbase + 4 * (uint32_t)((r * nc + j) >> 2));
        tmem_ld_wait();
#pragma unroll
        for (int r = 0; r < NR; ++r)
          if (r < nrr) mma_bf16(acc[r], a[r], b0, b1);
        if (!pk) {
#pragma unroll
          for (int r = 0; r < NR; ++r)
            if (r < nrr) mma_bf16(acc[r], a[r], xf.z, xf.w);
        }
      }
    } else if (!FP8) {
#pragma unroll 1
      for (int j = L.warp; j < nc; j += NCW) {
        const uint4 xf = xok ? lds128(xs + j * 64) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t b0 = lo_col ? xf.z : xf.x, b1 = lo_col ? xf.w : xf.y;
        uint4 a[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r)
          if (r < nrr) a[r] = lds128(stage + ((size_t)r * nc + j) * TILE_BF16 + lane * 16);
#pragma unroll
        for (int r = 0; r < NR; ++r)
          if (r < nrr) mma_bf16(acc[r], a[r], b0, b1);
        if (!pk) {
#pragma unroll
          for (int r = 0; r < NR; ++r)
            if (r < nrr) mma_bf16(acc[r], a[r], xf.z, xf.w);
        }
      }
    } else {
      // fp8: each warp takes a contiguous run of the chunk's col tiles and
      // sums raw products per 128-column scale block, applying the block's
      // scale once per block rather than once per tile
      const int per = (nc + NCW - 1) / NCW;
      const int j0 = min(nc, L.warp * per), j1 = min(nc, j0 + per);
      float raw[NR][4];
#pragma unroll
      for (int r = 0; r < NR; ++r) raw[r][0] = raw[r][1] = raw[r][2] = raw[r][3] = 0.f;
      int cb = (ci.c0 + j0) >> 3;
#pragma unroll FP8_UNROLL
      for (int j = j0; j < j1; ++j) {
        const int cbj = (ci.c0 + j) >> 3;
        if (cbj != cb) {
          fp8_apply_scales<NR>(m, sct, rb0, nrb, ci.g0, cb, raw, acc, nrr);
          cb = cbj;
        }
        const uint4 xf = xok ? lds128(xs + j * 64) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t b0 = lo_col ? xf.z : xf.x, b1 = lo_col ? xf.w : xf.y;
        uint2 a8[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r)
          if (r < nrr) a8[r] = lds64(stage + ((size_t)r * nc + j) * TILE_FP8 + lane * 8);
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          if (r < nrr) {
            const uint4 af = fp8_frag_to_f16(a8[r]);
            mma_f16(raw[r], af, b0, b1);
            if (!pk) mma_f16(raw[r], af, xf.z, xf.w);
          }
        }
      }
      if (j0 < j1) fp8_apply_scales<NR>(m, sct, rb0, nrb, ci.g0, cb, raw, acc, nrr);
    }
    if (L.trc) {
      float sink = 0.f;
#pragma unroll
      for (int r = 0; r < NR; ++r) sink += acc[r][0];
      if (sink == 12345.678f) C.ms->flag = 0;
      const long long t1 = clock64();
      C.ms->tr_mma += t1 - tc0;
      tc0 = t1;
    }
    if (tm) tc_fence_before();
    __syncwarp();
    const bool xlast = ci.win_last();
    if (lane == 0) {
      if (tm) mbar_arrive(&C.ms->tempty[tc % NTSD]);
      else mbar_arrive(&C.ms->empty[it % NSTAGE]);
      if (xlast) mbar_arrive(&C.ms->xempty[ix % XSLOTS]);
    }
    ++it;
    if (tm) ++tc;
    if (xlast) ++ix;
    if (L.trc) C.ms->tr_rel += clock64() - tc0;
    if (ci.group_done()) break;
    ci.next();
  }
  }
  if (L.trc) C.ms->tr_loop += clock64() - tl0;
  if (pk) {
#pragma unroll
    for (int r = 0; r < NR; ++r) fold_lo_cols(acc[r], L.M, tq, lane);
  }
  // per-warp partial sums (added to the previous K segments' when accum)
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    float4* pr = reinterpret_cast<float4*>(red + ((L.warp * RMAX + r) * 32 + lane) * 4);
    if (accum) {
      const float4 q = *pr;
      *pr = make_float4(q.x + acc[r][0], q.y + acc[r][1], q.z + acc[r][2], q.w + acc[r][3]);
    } else {
      *pr = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    }
  }
  cir = ci;
  itr = it;
  ixr = ix;
  tcr = tc;
}

// fp8 row groups: the same loop, in its own function (MK_FP8_GEMV_NOINLINE)
// or inlined like the bf16 ones.
#ifndef MK_FP8_GEMV_NOINLINE
#define MK_FP8_GEMV_NOINLINE 0
#endif
#if MK_FP8_GEMV_NOINLINE
#define MK_FP8_GEMV_ATTR __noinline__
#else
#define MK_FP8_GEMV_ATTR __forceinline__
#endif
template <int NR>
__device__ MK_FP8_GEMV_ATTR void gemv_group_fp8(const Ctx& C, ChunkIt& ci, const Mat& m, const GemvLane& L, uint32_t& it,
                                                uint32_t& ix, uint32_t& tc, float* red, bool accum) {
  gemv_group<NR, true>(C, ci, m, L, it, ix, tc, red, accum);
}

template <bool MLA, int MOE>
__device__ void gemv_task(const Ctx& C, const Task& t, uint32_t& it, uint32_t& ix, uint32_t& tc) {
  const Launch& P = *C.P;
  const long long tpre = (MK_TRACE && P.trace && threadIdx.x == 0) ? clock64() : 0;
  const Model& md = *C.md;
  // Copies in registers: the barrier asm below clobbers "memory", which would
  // otherwise force a reload of every struct field on every chunk.
  const Mat m = t.m;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int M = P.M;
  const int tb = m.fp8 ? TILE_FP8 : TILE_BF16;
  const bool has_gain = t.in_kind != IN_BUF;

  float ss_acc[2] = {0.f, 0.f};
  float am_v[2] = {-INFINITY, -INFINITY};
  int am_i[2] = {0x7fffffff, 0x7fffffff};

  // MoE: this task's rows / K segments follow the router's union of experts
  int U = 0;
  if (task_needs_route<MOE>(t)) {
    // the activation producer publishes the layer's route (it waits on the
    // router's counter anyway); the consumers only check that it is there
    const long long tr0 = (MK_TRACE && P.trace && tid == 0) ? clock64() : 0;
    if (tid == 0) {
      const uint64_t t0 = globaltimer();
      while (*reinterpret_cast<volatile int*>(&C.ms->route_layer) != t.layer + 1) {
        if (C.ms->abort) break;
        if (globaltimer() - t0 > (uint64_t)P.timeout_ns * 2) {
          raise_error(P, C.ms, DERR_TIMEOUT, 0x80000 | t.layer);
          break;
        }
      }
      __threadfence_block();
    }
    if (MK_TRACE && P.trace && tid == 0) C.ms->tr_route += clock64() - tr0;
    bar_consumers();
    U = C.ms->rt_u[RR_XPROD];
  }
  const Mat m2 = (MOE && t.type == T_MOE_DOWN && t.mat2 >= 0) ? md.mats[t.mat2] : m;
  int rt0, rt1, gsz, nseg;
  task_rows<MOE>(md, t, m, U, rt0, rt1, gsz, nseg);
  Pieces pc;
  bool have = pc.init(rt0, rt1, gsz, nseg);
  const int xcap = x_cap(t, M);
  float* red = reinterpret_cast<float*>(C.att);
  GemvLane L;
  L.warp = warp;
  L.lane = lane;
  L.g = g;
  L.tq = tq;
  L.M = M;
  L.has_gain = has_gain;
  L.rowbytes = 0;
  L.trc = MK_TRACE && P.trace && tid == 0;
  L.conv = t.in_kind != IN_X_NORM && !frag_buf(t.in_buf);
  L.gain = t.gvec;
  L.nseg = 1;
  L.NS = md.NS;
  L.sc_sh = L.sc_rt = nullptr;
  L.ss_sh = L.ss_rt = 0;
  L.ex = C.ms->rt_ex[RR_XPROD];
  if (L.trc) C.ms->tr_pre += clock64() - tpre;
  while (have) {
    const PieceSrc src = piece_src<MOE>(md, t, m, m2, C.ms->rt_ex[RR_XPROD], pc);
    ChunkIt ci;
    ci.init(src.lg0, src.lg0 + pc.nr, m.KT, tb, 0, xcap);
    L.rowbytes = x_rowbytes(t, ci.WC);
    Mat mg = (MOE && t.type == T_MOE_DOWN && pc.seg < md.NS) ? m2 : m;
    mg.w = src.w;
    mg.scales = src.scales;
    const bool accum = false;
    if (MOE && t.type == T_MOE_DOWN) {
      // every K segment of the row group in one call, the sums kept in registers
      L.nseg = pc.nseg;
      L.sc_sh = m2.scales;
      L.ss_sh = m2.sstride;
      L.sc_rt = m.scales;
      L.ss_rt = m.sstride;
    }
    // one instance per row-tile count: every loop over rows is static (fp8
    // weights exist only for experts, so only the fp8-expert MoE kernels
    // (MOE == 2) hold the fp8 ones)
    if (MOE != 2 || !m.fp8) {
      switch (ci.nr) {
#if MK_GEMV_SET == 8
        case 1: gemv_group<1, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 2: gemv_group<2, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 3: gemv_group<3, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
#if MK_RMAX > 4
        case 4: gemv_group<4, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 5: gemv_group<5, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 6: gemv_group<6, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 7: gemv_group<7, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
#endif
        default: gemv_group<RMAX, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
#elif MK_GEMV_SET == 4
        case 1: gemv_group<1, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 2: gemv_group<2, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 3:
        case 4: gemv_group<4, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
        default: gemv_group<RMAX, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
#else
        default: gemv_group<RMAX, false>(C, ci, mg, L, it, ix, tc, red, accum); break;
#endif
      }
    } else if constexpr (MOE == 2) {
      switch (ci.nr) {
#if MK_FP8_SET == 8
        case 1: gemv_group_fp8<1>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 2: gemv_group_fp8<2>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 3: gemv_group_fp8<3>(C, ci, mg, L, it, ix, tc, red, accum); break;
#if MK_RMAX > 4
        case 4: gemv_group_fp8<4>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 5: gemv_group_fp8<5>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 6: gemv_group_fp8<6>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 7: gemv_group_fp8<7>(C, ci, mg, L, it, ix, tc, red, accum); break;
#endif
        default: gemv_group_fp8<RMAX>(C, ci, mg, L, it, ix, tc, red, accum); break;
#elif MK_FP8_SET == 4
        case 1: gemv_group_fp8<1>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 2: gemv_group_fp8<2>(C, ci, mg, L, it, ix, tc, red, accum); break;
        case 3:
        case 4: gemv_group_fp8<4>(C, ci, mg, L, it, ix, tc, red, accum); break;
        default: gemv_group_fp8<RMAX>(C, ci, mg, L, it, ix, tc, red, accum); break;
#else
        default: gemv_group_fp8<RMAX>(C, ci, mg, L, it, ix, tc, red, accum); break;
#endif
      }
    }
    if (MOE && t.type == T_MOE_DOWN) pc.seg = pc.nseg - 1;  // the call took every segment
    const bool trc = L.trc;
    long long tc0 = trc ? clock64() : 0;
    {
      // ---- cross-warp reduction and epilogue for row tiles [g0, g0 + nr) ----
      bar_consumers();
      {
        const int r = tid >> 5, l = lane;
        if (r < pc.nr) {
          float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int w = 0; w < NCW; ++w) {
            float4 q = *reinterpret_cast<const float4*>(red + ((w * RMAX + r) * 32 + l) * 4);
            v[0] += q.x;
            v[1] += q.y;
            v[2] += q.z;
            v[3] += q.w;
          }
          const int rt = pc.g0 + r;
          const int row0 = rt * 16 + (l >> 2), row1 = row0 + 8;
          const int m0 = 2 * (l & 3), m1 = m0 + 1;
          if (has_gain) {  // RMSNorm, a per-row scale, applied to the GEMV's sums
            const float s0 = C.ms->gscale[m0], s1 = C.ms->gscale[m1];
            v[0] *= s0;
            v[1] *= s1;
            v[2] *= s0;
            v[3] *= s1;
          }
          if (t.epi == EPI_STORE) {
            float* out = P.buf[t.out_buf];
            const int ld = P.ld[t.out_buf];
            if (MLA && t.out_buf == B_QL) {
              // absorbed queries: written as the latent attention's bf16 hi / lo
              // A fragments (row = head, col = latent dim), scaled to log2 units
              const int R = md.R, KWl = R >> 4, hiblk = ((md.Hq + 15) >> 4) * KWl * 512;
              const float qs = rsqrtf((float)(md.d + md.dr)) * 1.4426950408889634f;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int row = (q < 2) ? row0 : row1;
                const int mm = (q & 1) ? m1 : m0;
                if (row < m.rows && mm < M) {
                  uint8_t* blk = reinterpret_cast<uint8_t*>(out + (size_t)mm * ld);
                  const int off = frag_off(row / R, row - (row / R) * R, KWl);
                  const float x = v[q] * qs;
                  const __nv_bfloat16 hb = __float2bfloat16_rn(x);
                  *reinterpret_cast<__nv_bfloat16*>(blk + off) = hb;
                  *reinterpret_cast<__nv_bfloat16*>(blk + hiblk + off) = __float2bfloat16_rn(x - __bfloat162float(hb));
                }
              }
            } else if (frag_buf(t.out_buf)) {  // feeds the next GEMV only (bf16 weights)
              if (row0 < m.rows) {
                if (m0 < M) st_frag(out + (size_t)m0 * ld, row0, v[0], false);
                if (m1 < M) st_frag(out + (size_t)m1 * ld, row0, v[1], false);
              }
              if (row1 < m.rows) {
                if (m0 < M) st_frag(out + (size_t)m0 * ld, row1, v[2], false);
                if (m1 < M) st_frag(out + (size_t)m1 * ld, row1, v[3], false);
              }
            } else {
              if (row0 < m.rows) {
                if (m0 < M) out[(size_t)m0 * ld + row0] = v[0];
                if (m1 < M) out[(size_t)m1 * ld + row0] = v[1];
              }
              if (row1 < m.rows) {
                if (m0 < M) out[(size_t)m0 * ld + row1] = v[2];
                if (m1 < M) out[(size_t)m1 * ld + row1] = v[3];
              }
            }
          } else if (t.epi == EPI_RESID) {
            float* x = P.buf[B_X];
            const int ld = P.ld[B_X];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int row = (q < 2) ? row0 : row1;
              const int mm = (q & 1) ? m1 : m0;
              if (row < m.rows && mm < M) {
                const float base = __ldcg(x + (size_t)mm * ld + row);
                const float nv = base + v[q];
                x[(size_t)mm * ld + row] = nv;
                ss_acc[q & 1] += nv * nv;
                const float gx = nv * __uint_as_float((uint32_t)__ldg(t.gnext + row) << 16);
                st_frag(P.buf[B_XF] + (size_t)mm * P.ld[B_XF], row, gx, false);
                if (t.xf16) st_frag(P.buf[B_XF16] + (size_t)mm * P.ld[B_XF16], row, gx, true);
              }
            }
          } else if (MOE && t.epi == EPI_SWIGLU_MOE) {
            // virtual row tile rt of expert slot rt / RTe (shared slots first)
            const int slot = rt / m.RT;
            const int hs = (t.moe == 1 ? 0 : md.NS) + slot;
            const int i = (rt - slot * m.RT) * 8 + (l >> 2);
            float* h = P.buf[B_H];
            const int ld = P.ld[B_H];
            if (i * 2 < m.rows) {
              const float w0 = t.moe == 1 ? 1.f : C.ms->rt_w[slot][m0 < MAXM ? m0 : 0];
              const float w1 = t.moe == 1 ? 1.f : C.ms->rt_w[slot][m1 < MAXM ? m1 : 0];
              if (m0 < M) st_frag(h + ((size_t)hs * MAXM + m0) * ld, i, w0 * silu_f(v[0]) * v[2], md.fp8 != 0);
              if (m1 < M) st_frag(h + ((size_t)hs * MAXM + m1) * ld, i, w1 * silu_f(v[1]) * v[3], md.fp8 != 0);
            }
          } else if (t.epi == EPI_SWIGLU) {
            float* h = P.buf[t.out_buf];
            const int ld = P.ld[t.out_buf];
            const int i = rt * 8 + (l >> 2);
            if (i * 2 < m.rows) {
              if (m0 < M) st_frag(h + (size_t)m0 * ld, i, silu_f(v[0]) * v[2], false);
              if (m1 < M) st_frag(h + (size_t)m1 * ld, i, silu_f(v[1]) * v[3], false);
            }
          } else if (t.epi == EPI_LOGITS) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int row = (q < 2) ? row0 : row1;
              const int mm = (q & 1) ? m1 : m0;
              if (row < m.rows && mm < M) {
                if (P.logits) P.logits[(size_t)mm * md.V + row] = v[q];
                const int k = q & 1;
                if (v[q] > am_v[k] || (v[q] == am_v[k] && row < am_i[k])) {
                  am_v[k] = v[q];
                  am_i[k] = row;
                }
              }
            }
          }
        }
      }
      bar_consumers();
      if (trc) C.ms->tr_epi += clock64() - tc0;
    }
    have = pc.next();
  }

  const long long tpost = L.trc ? clock64() : 0;
  // ---- task-level partials: sum of squares (RESID) or argmax (LOGITS) ----
  if (t.epi == EPI_RESID || t.epi == EPI_LOGITS) {
    float* f2 = reinterpret_cast<float*>(C.att);
    int* i2 = reinterpret_cast<int*>(C.att + NCT * 2 * sizeof(float));
    if (t.epi == EPI_RESID) {
      f2[tid * 2 + 0] = ss_acc[0];
      f2[tid * 2 + 1] = ss_acc[1];
    } else {
      f2[tid * 2 + 0] = am_v[0];
      f2[tid * 2 + 1] = am_v[1];
      i2[tid * 2 + 0] = am_i[0];
      i2[tid * 2 + 1] = am_i[1];
    }
    bar_consumers();
    if (tid < MAXM) {
      const int mm = tid, tsel = mm >> 1, k = mm & 1;
      if (t.epi == EPI_RESID) {
        float s = 0.f;
        for (int th = tsel; th < NCT; th += 4) s += f2[th * 2 + k];
        P.ss_part[((size_t)t.ss_dst * C.ncta + blockIdx.x) * MAXM + mm] = s;
      } else {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int th = tsel; th < NCT; th += 4) {
          const float v = f2[th * 2 + k];
          const int ix = i2[th * 2 + k];
          if (v > bv || (v == bv && ix < bi)) {
            bv = v;
            bi = ix;
          }
        }
        P.am_val[(size_t)blockIdx.x * MAXM + mm] = bv;
        P.am_idx[(size_t)blockIdx.x * MAXM + mm] = bi;
      }
    }
  }
  if (L.trc) C.ms->tr_post += clock64() - tpost;
}

// Embedding gather: this CTA's column slice [c0, c1) of x[m] = E[token_m],
// widened exactly to fp32, and its per-row sums of squares for the first
// RMSNorm (fixed-order reduction).
__device__ void embed_task(const Ctx& C, const Task& t) {
  const Launch& P = *C.P;
  const Model& md = *C.md;
  const int tid = threadIdx.x, M = P.M;
  float* x = P.buf[B_X];
  const int ld = P.ld[B_X];
  float part[MAXM];
#pragma unroll
  for (int mm = 0; mm < MAXM; ++mm) part[mm] = 0.f;
  for (int k = t.rt0 + tid; k < t.rt1; k += NCT) {
#pragma unroll
    for (int mm = 0; mm < MAXM; ++mm) {
      if (mm < M) {
        const uint16_t* e = md.embed + (size_t)__ldg(P.tokens + mm) * md.H;
        const float v = __uint_as_float((uint32_t)__ldg(e + k) << 16);
        x[(size_t)mm * ld + k] = v;
        part[mm] += v * v;
        st_frag(P.buf[B_XF] + (size_t)mm * P.ld[B_XF], k, v * __uint_as_float((uint32_t)__ldg(t.gnext + k) << 16),
                false);
      }
    }
  }
  float* red = reinterpret_cast<float*>(C.att);
#pragma unroll
  for (int mm = 0; mm < MAXM; ++mm) red[tid * MAXM + mm] = part[mm];
  bar_consumers();
  if (tid < M) {
    float s2 = 0.f;
    for (int th = 0; th < NCT; ++th) s2 += red[th * MAXM + tid];
    P.ss_part[((size_t)t.ss_dst * C.ncta + blockIdx.x) * MAXM + tid] = s2;
  }
}

// Last CTA to finish the LM head reduces the per-CTA argmax partials and,
// for a verify step, the greedy acceptance.
__device__ void lm_finish(const Ctx& C) {
  const Launch& P = *C.P;
  bar_consumers();
  int last = 0;
  if (threadIdx.x == 0 && !C.ms->abort) {
    const uint32_t old = atom_add_acqrel(P.ctr + P.ctr_lm, 1u);
    last = (old == (uint32_t)C.ncta - 1) ? 1 : 0;
  }
  if (!broadcast_from0(C, last)) return;
  {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < P.M) {
      const int mm = warp;
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      for (int c = lane; c < C.ncta; c += 32) {
        const float v = __ldcg(P.am_val + (size_t)c * MAXM + mm);
        const int ix = __ldcg(P.am_idx + (size_t)c * MAXM + mm);
        if (v > bv || (v == bv && ix < bi)) {
          bv = v;
          bi = ix;
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (lane == 0) {
        P.argmax[mm] = bi;
        C.ms->scale[mm] = __int_as_float(bi);
      }
    }
  }
  bar_consumers();
  if (threadIdx.x == 0 && P.accepted) {
    // tokens[0] = anchor, tokens[1..Q-1] = proposals; argmax[j] = greedy after position j
    int a = 0;
    while (a + 1 < P.Q && __ldg(P.tokens + a + 1) == __float_as_int(C.ms->scale[a])) ++a;
    P.accepted[0] = a;
  }
}

// ---------------------------------------------------------------------------
// GQA attention item: split-KV flash decoding with mma.sync
// ---------------------------------------------------------------------------
// Shared layout inside the attention scratch:
//   Q fragments (hi, lo): [mt][d/16][32 lanes][16 B]
//   P fragments (hi, lo): [mt][64/16][32 lanes][16 B]
//   smax: [2][NCW][48] fp32

// Each consumer warp owns 16 positions of every 64-position chunk (position
// group w & 3) and half of the head dims (w >> 2), and runs its own online
// softmax: scores go from the QK accumulators straight into the PV A
// fragments, with no barrier inside a chunk.  The four position groups of
// each dim half are merged once per item.
template <int MT, int NTD>  // MT: 16-row tiles of query rows; NTD: 8-dim tiles of this warp's half
struct WarpAtt {
  float o[MT][NTD][4];
  float M[MT][2];  // running max (log2 units) of rows g, g + 8 of each row tile
  float L[MT][2];  // lane-partial running sums
};

template <int MT, int NTD>
__device__ __forceinline__ void warp_att_chunk(WarpAtt<MT, NTD>& st, const uint8_t* qhi, const uint8_t* qlo,
                                               const uint8_t* Ks, const uint8_t* Vs, int pitch, int KTq, int n_valid,
                                               bool causal, int gh, int p0, int dim0, int base) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  if (p0 >= n_valid) return;
  // ---- scores of positions p0 .. p0 + 15 (two 8-position n-tiles) ----
  float sc[MT][2][4];
#pragma unroll
  for (int mi = 0; mi < MT; ++mi)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sc[mi][nt][0] = sc[mi][nt][1] = sc[mi][nt][2] = sc[mi][nt][3] = 0.f;
  // rows p0 + g and p0 + 8 + g share the permutation key (base + p0 + g) & 7
  const int key = (base + p0 + g) & 7;
  const uint8_t* k0 = Ks + (size_t)(p0 + g) * pitch + tq * 4;
  const uint8_t* k1 = k0 + (size_t)8 * pitch;
#pragma unroll 2
  for (int ks = 0; ks < KTq; ++ks) {
    const int c0 = ((2 * ks) ^ key) * 16, c1 = ((2 * ks + 1) ^ key) * 16;
    const uint32_t b00 = lds32(k0 + c0), b01 = lds32(k0 + c1);
    const uint32_t b10 = lds32(k1 + c0), b11 = lds32(k1 + c1);
#pragma unroll
    for (int mi = 0; mi < MT; ++mi) {
      const uint4 ah = lds128(qhi + ((mi * KTq + ks) * 32 + lane) * 16);
      const uint4 al = lds128(qlo + ((mi * KTq + ks) * 32 + lane) * 16);
      mma_bf16(sc[mi][0], ah, b00, b01);
      mma_bf16(sc[mi][0], al, b00, b01);
      mma_bf16(sc[mi][1], ah, b10, b11);
      mma_bf16(sc[mi][1], al, b10, b11);
    }
  }
  // ---- masking, online softmax, P as A fragments (bf16 hi / lo) ----
  uint4 ph[MT], pl[MT];
#pragma unroll
  for (int mi = 0; mi < MT; ++mi) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int row = mi * 16 + g + 8 * h2;
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int pos = p0 + nt * 8 + 2 * tq + e;
          float& v = sc[mi][nt][2 * h2 + e];
          if (pos >= n_valid || (causal && pos > row / gh)) v = -INFINITY;
          mx = fmaxf(mx, v);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(st.M[mi][h2], mx);
      const float corr = (mnew == -INFINITY) ? 1.f : exp2f(st.M[mi][h2] - mnew);
      const float msafe = (mnew == -INFINITY) ? 0.f : mnew;
      st.M[mi][h2] = mnew;
      float ls = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float& v = sc[mi][nt][2 * h2 + e];
          v = exp2f(v - msafe);
          ls += v;
        }
      st.L[mi][h2] = st.L[mi][h2] * corr + ls;
#pragma unroll
      for (int nt = 0; nt < NTD; ++nt) {
        st.o[mi][nt][2 * h2 + 0] *= corr;
        st.o[mi][nt][2 * h2 + 1] *= corr;
      }
    }
    // A fragment of P (16 rows x 16 positions): a0 rows g / k 2tq.., a1 rows g+8,
    // a2 rows g / k 8+2tq.., a3 rows g+8 / k 8+2tq..
    split_bf16(sc[mi][0][0], sc[mi][0][1], ph[mi].x, pl[mi].x);
    split_bf16(sc[mi][0][2], sc[mi][0][3], ph[mi].y, pl[mi].y);
    split_bf16(sc[mi][1][0], sc[mi][1][1], ph[mi].z, pl[mi].z);
    split_bf16(sc[mi][1][2], sc[mi][1][3], ph[mi].w, pl[mi].w);
  }
  // ---- O += P V over this warp's dims; rows past n_valid of V are zeroed ----
  const int pk = p0 + 2 * tq;
  const int vr = p0 + (lane & 15), vkey = (base + vr) & 7;
  const uint8_t* vrow = Vs + (size_t)vr * pitch;
#pragma unroll
  for (int nt = 0; nt < NTD; ++nt) {
    uint32_t b0, b1;
    ldsm_x2_trans(vrow + (((dim0 >> 3) + nt) ^ vkey) * 16, b0, b1);
    if (pk >= n_valid) b0 = 0u;
    else if (pk + 1 >= n_valid) b0 &= 0xFFFFu;
    if (pk + 8 >= n_valid) b1 = 0u;
    else if (pk + 9 >= n_valid) b1 &= 0xFFFFu;
#pragma unroll
    for (int mi = 0; mi < MT; ++mi) {
      mma_bf16(st.o[mi][nt], ph[mi], b0, b1);
      mma_bf16(st.o[mi][nt], pl[mi], b0, b1);
    }
  }
}

template <int MT, int NTD>
__device__ void attn_item(const Ctx& C, const Task& t, uint32_t& it) {
  const Launch& P = *C.P;
  const Model& md = *C.md;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const bool trc = MK_TRACE && P.trace && threadIdx.x == 0;
  long long tA = trc ? clock64() : 0;
  const Item itm = decode_item(t.rt0, P.n_pairs, P.n_items);
  const int s = itm.pair / md.Hkv, kvh = itm.pair % md.Hkv;
  const int d = md.d, pitch = att_pitch(d), KTq = d / 16;
  const int gh = md.Hq / md.Hkv, Q = P.Q, nr = Q * gh, mt = MT;
  const int T0 = seq_pos0(P, s);
  const int a = (int)(((int64_t)itm.j * T0) / itm.ns), b = (int)(((int64_t)(itm.j + 1) * T0) / itm.ns);
  const bool last = itm.j == itm.ns - 1;
  const float qscale = rsqrtf((float)d) * 1.4426950408889634f;
  const float* qkv = P.buf[B_QKV];
  const int ldq = P.ld[B_QKV];
  const float2* rope = md.rope;
  const int half = d / 2;

  // ---- stage Q (RoPE, scaled to log2 units) as bf16 hi/lo A fragments; the
  //      last split also appends the step's own new positions (RoPE(k), bf16)
  //      to the cache.  One pass over both, so all their loads overlap. ----
  uint8_t* qhi = C.att;
  uint8_t* qlo = qhi + mt * KTq * 512;
  uint8_t* nk = C.newkv;
  uint8_t* nv = C.newkv + 16 * pitch;
  const size_t head = (((size_t)t.layer * P.kv_seqs + s) * md.Hkv + kvh) * (size_t)P.kv_ctx;
  const int nq = mt * 16 * half, nkv = last ? 16 * half : 0;
  for (int e = tid; e < max(nq, nkv); e += NCT) {
    const int r = e / half, i = e % half;  // r: query row (Q part), or step position (K/V part)
    const bool dq = e < nq && r < nr, dk = e < nkv && r < Q;
    float qa0 = 0.f, qa1 = 0.f, ka0 = 0.f, ka1 = 0.f, va0 = 0.f, va1 = 0.f;
    float2 qcs = make_float2(1.f, 0.f), kcs = make_float2(1.f, 0.f);
    if (dq) {
      const int qi = r / gh, hh = r % gh;
      const float* q = qkv + (size_t)(s * Q + qi) * ldq + (size_t)(kvh * gh + hh) * d;
      qa0 = __ldcg(q + i);
      qa1 = __ldcg(q + i + half);
      qcs = __ldg(rope + (size_t)(T0 + qi) * half + i);
    }
    if (dk) {
      const float* kr = qkv + (size_t)(s * Q + r) * ldq + (size_t)(md.Hq + kvh) * d;
      const float* vr = qkv + (size_t)(s * Q + r) * ldq + (size_t)(md.Hq + md.Hkv + kvh) * d;
      ka0 = __ldcg(kr + i);
      ka1 = __ldcg(kr + i + half);
      va0 = __ldcg(vr + i);
      va1 = __ldcg(vr + i + half);
      kcs = __ldg(rope + (size_t)(T0 + r) * half + i);
    }
    if (e < nq) {
      const float x0 = dq ? (qa0 * qcs.x - qa1 * qcs.y) * qscale : 0.f;
      const float x1 = dq ? (qa0 * qcs.y + qa1 * qcs.x) * qscale : 0.f;
      const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
      *reinterpret_cast<__nv_bfloat16*>(qhi + frag_off(r, i, KTq)) = h0;
      *reinterpret_cast<__nv_bfloat16*>(qhi + frag_off(r, i + half, KTq)) = h1;
      *reinterpret_cast<__nv_bfloat16*>(qlo + frag_off(r, i, KTq)) = __float2bfloat16_rn(x0 - __bfloat162float(h0));
      *reinterpret_cast<__nv_bfloat16*>(qlo + frag_off(r, i + half, KTq)) =
          __float2bfloat16_rn(x1 - __bfloat162float(h1));
    }
    if (e < nkv) {
      __nv_bfloat16 k0 = __float2bfloat16_rn(0.f), k1 = k0, v0 = k0, v1 = k0;
      if (dk) {
        const int pos = T0 + r;
        k0 = __float2bfloat16_rn(ka0 * kcs.x - ka1 * kcs.y);
        k1 = __float2bfloat16_rn(ka0 * kcs.y + ka1 * kcs.x);
        v0 = __float2bfloat16_rn(va0);
        v1 = __float2bfloat16_rn(va1);
        __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(P.kv_k) + (head + pos) * d;
        __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(P.kv_v) + (head + pos) * d;
        kc[kv_swz(pos, i)] = k0;
        kc[kv_swz(pos, i + half)] = k1;
        vc[kv_swz(pos, i)] = v0;
        vc[kv_swz(pos, i + half)] = v1;
      }
      // shared-memory row r: permuted by r (the reader's key for these rows)
      *reinterpret_cast<__nv_bfloat16*>(nk + r * pitch + kv_swz(r, i) * 2) = k0;
      *reinterpret_cast<__nv_bfloat16*>(nk + r * pitch + kv_swz(r, i + half) * 2) = k1;
      *reinterpret_cast<__nv_bfloat16*>(nv + r * pitch + kv_swz(r, i) * 2) = v0;
      *reinterpret_cast<__nv_bfloat16*>(nv + r * pitch + kv_swz(r, i + half) * 2) = v1;
    }
  }
  bar_consumers();
  if (trc) {
    const long long t1 = clock64();
    C.ms->tr_pre += t1 - tA;
    tA = t1;
  }

  WarpAtt<MT, NTD> st;
#pragma unroll
  for (int mi = 0; mi < MT; ++mi) {
    st.M[mi][0] = st.M[mi][1] = -INFINITY;
    st.L[mi][0] = st.L[mi][1] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NTD; ++nt) st.o[mi][nt][0] = st.o[mi][nt][1] = st.o[mi][nt][2] = st.o[mi][nt][3] = 0.f;
  }
  const int pg = warp & 3, dh = warp >> 2;
  const int p0 = pg * 16, dim0 = dh * half;
  for (int t0 = a; t0 < b; t0 += ATT_CT) {
    const int n = min(ATT_CT, b - t0);
    wait_full(C, it);
    const uint8_t* stage = C.ring + (size_t)(it % NSTAGE) * STAGE_BYTES;
    // a warp takes its 16 positions of each 64-position part of the chunk
#pragma unroll
    for (int h64 = 0; h64 < ATT_CT / 64; ++h64)
      warp_att_chunk<MT, NTD>(st, qhi, qlo, stage, stage + (size_t)ATT_CT * pitch, pitch, KTq, n, false, gh,
                              p0 + 64 * h64, dim0, t0);
    release_stage(C, it);  // per warp: the ring's empty barrier counts the consumer warps
    ++it;
  }
  if (last) warp_att_chunk<MT, NTD>(st, qhi, qlo, nk, nv, pitch, KTq, Q, true, gh, p0, dim0, 0);
  bar_consumers();  // every warp is done with the query fragments: the scratch is reused below
  if (trc) {
    const long long t1 = clock64();
    C.ms->tr_loop += t1 - tA;
    tA = t1;
  }

  // ---- merge the four position groups of each dim half, one row tile at a
  //      time, into the item's partial (O | M | L per query row) ----
  const int rows_max = P.att_rows_max;
  const int dP = d + 4;
  float* part = P.att_part + (size_t)t.rt0 * rows_max * dP;
  float* Ow = reinterpret_cast<float*>(C.att);              // [warp][16 rows][half]
  float* Mw = Ow + NCW * 16 * half;                           // [warp][16]
  float* Lw = Mw + NCW * 16;                                  // [warp][16]
#pragma unroll
  for (int mi = 0; mi < MT; ++mi) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      float l = st.L[mi][h2];
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      if (tq == 0) {
        Mw[warp * 16 + g + 8 * h2] = st.M[mi][h2];
        Lw[warp * 16 + g + 8 * h2] = l;
      }
    }
#pragma unroll
    for (int nt = 0; nt < NTD; ++nt) {
      float* o0 = Ow + ((size_t)warp * 16 + g) * half + nt * 8 + 2 * tq;
      o0[0] = st.o[mi][nt][0];
      o0[1] = st.o[mi][nt][1];
      o0[8 * half] = st.o[mi][nt][2];
      o0[8 * half + 1] = st.o[mi][nt][3];
    }
    bar_consumers();
    // thread -> (row, 8 consecutive dims)
    for (int e = tid; e < 16 * (d / 8); e += NCT) {
      const int r = e / (d / 8), k0 = (e - r * (d / 8)) * 8;
      const int row = mi * 16 + r;
      const int dhk = k0 / half, kl = k0 - dhk * half;
      float mx = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q) mx = fmaxf(mx, Mw[(dhk * 4 + q) * 16 + r]);
      float wq[4], lsum = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float mq = Mw[(dhk * 4 + q) * 16 + r];
        wq[q] = (mq == -INFINITY) ? 0.f : exp2f(mq - mx);
        lsum += wq[q] * Lw[(dhk * 4 + q) * 16 + r];
      }
      float acc8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc8[i] = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float* src = Ow + ((size_t)(dhk * 4 + q) * 16 + r) * half + kl;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc8[i] += wq[q] * src[i];
      }
      if (row < nr) {
        float* dst = part + (size_t)row * dP;
        *reinterpret_cast<float4*>(dst + k0) = make_float4(acc8[0], acc8[1], acc8[2], acc8[3]);
        *reinterpret_cast<float4*>(dst + k0 + 4) = make_float4(acc8[4], acc8[5], acc8[6], acc8[7]);
        if (k0 == 0) {
          dst[d] = mx;
          dst[d + 1] = lsum;
        }
      }
    }
    bar_consumers();
  }
  if (trc) {
    const long long t1 = clock64();
    C.ms->tr_post += t1 - tA;
    tA = t1;
  }

  // ---- the split combine, spread over the pair's items: each item counts
  //      itself in (publishing its partial), waits until every item of its
  //      (sequence, kv head) has, then merges a slice of the pair's outputs.
  //      Eight threads per output (4 dims of one row), each over every 8th
  //      split, with an online max; one round of loads, then quad-octet
  //      shuffles.  Each item has at most one CTA's worth of work per layer
  //      whenever a pair has more than one item (n_items = max(pairs, CTAs)),
  //      so no item waits for an item queued behind it. ----
  if (tid == 0 && !C.ms->abort) {
    uint32_t* pc = P.ctr + P.ctr_pair_base + t.layer * P.n_pairs + itm.pair;
    red_release_add(pc, 1u);
    const uint64_t w0 = globaltimer();
    uint32_t spins = 0;
    while (ld_acquire(pc) < (uint32_t)itm.ns) {
      if (C.ms->abort) break;
      if (++spins >= 16) {
        spins = 0;
        if (global_abort(P)) { C.ms->abort = 1; break; }
        if (globaltimer() - w0 > (uint64_t)P.timeout_ns) {
          raise_error(P, C.ms, DERR_TIMEOUT, 0xE0000 | itm.pair);
          break;
        }
      }
    }
  }
  bar_consumers();
  if (trc) {
    const long long t1 = clock64();
    C.ms->tr_post += t1 - tA;
    tA = t1;
  }
  {
    float* out = P.buf[B_ATTN];
    const int ldo = P.ld[B_ATTN];
    const int ns = itm.ns, d4 = d / 4, U = nr * d4;
    const int u0 = (int)(((int64_t)itm.j * U) / ns), u1 = (int)(((int64_t)(itm.j + 1) * U) / ns);
    const int sub = tid & 7;
    const size_t js = (size_t)rows_max * dP;
    for (int base = u0; base < u1; base += NCT / 8) {
      const int u = base + (tid >> 3);
      const bool act = u < u1;
      const int r = act ? u / d4 : 0, k = act ? (u - r * d4) * 4 : 0;
      const float* src = P.att_part + ((size_t)itm.first * rows_max + r) * dP;
      float mr = -INFINITY, den = 0.f;
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
      if (act) {
#pragma unroll 4
        for (int jj = sub; jj < ns; jj += 8) {
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(src + jj * js + d));
          const float4 o = __ldcg(reinterpret_cast<const float4*>(src + jj * js + k));
          if (ml.x == -INFINITY) continue;
          const float mn = fmaxf(mr, ml.x);
          const float a = mr == -INFINITY ? 0.f : exp2f(mr - mn), b = exp2f(ml.x - mn);
          den = den * a + b * ml.y;
          num.x = num.x * a + b * o.x;
          num.y = num.y * a + b * o.y;
          num.z = num.z * a + b * o.z;
          num.w = num.w * a + b * o.w;
          mr = mn;
        }
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, mr, off);
        const float dno = __shfl_xor_sync(0xffffffffu, den, off);
        const float nx = __shfl_xor_sync(0xffffffffu, num.x, off), ny = __shfl_xor_sync(0xffffffffu, num.y, off);
        const float nz = __shfl_xor_sync(0xffffffffu, num.z, off), nw = __shfl_xor_sync(0xffffffffu, num.w, off);
        const float mn = fmaxf(mr, mo);
        const float a = mr == -INFINITY ? 0.f : exp2f(mr - mn), b = mo == -INFINITY ? 0.f : exp2f(mo - mn);
        den = den * a + dno * b;
        num.x = num.x * a + nx * b;
        num.y = num.y * a + ny * b;
        num.z = num.z * a + nz * b;
        num.w = num.w * a + nw * b;
        mr = mn;
      }
      if (act && sub == 0) {
        const float inv = 1.f / den;
        const int qi = r / gh, hh = r % gh;
        float* orow = out + (size_t)(s * Q + qi) * ldo;
        const int kc = (kvh * gh + hh) * d + k;
        st_frag(orow, kc, num.x * inv, false);
        st_frag(orow, kc + 1, num.y * inv, false);
        st_frag(orow, kc + 2, num.z * inv, false);
        st_frag(orow, kc + 3, num.w * inv, false);
      }
    }
  }
  bar_consumers();
  if (tid == 0 && !C.ms->abort) red_release_add(P.ctr + t.layer * P.ctr_layer_stride + C_ATTN, 1u);
  if (trc) C.ms->tr_epi += clock64() - tA;
}


// Attention task bodies: inlined into the consumer loop (no call frame) or
// out of line (own register allocation).  Measured: inlining the grouped
// query attention body shortens the dense and MoE steps (about 6% and 13% at
// B = 1); inlining the latent-attention body lengthens that step by 3%.
#ifndef MK_ATTN_INLINE
#define MK_ATTN_INLINE 1
#endif
#ifndef MK_MLA_INLINE
#define MK_MLA_INLINE 0
#endif
#if MK_ATTN_INLINE
#define MK_ATTN_ATTR __forceinline__
#else
#define MK_ATTN_ATTR __noinline__
#endif
#if MK_MLA_INLINE
#define MK_MLA_ATTR __forceinline__
#else
#define MK_MLA_ATTR __noinline__
#endif
__device__ MK_ATTN_ATTR void attn_task(const Ctx& C, const Task& t, uint32_t& it) {
  const Model& md = *C.md;
  const int nr = C.P->Q * (md.Hq / md.Hkv);
  const int mt = (nr + 15) >> 4;
  if (md.d == 128) {
    if (mt == 1) attn_item<1, 8>(C, t, it);
    else if (mt == 2) attn_item<2, 8>(C, t, it);
    else attn_item<3, 8>(C, t, it);
  } else {
    if (mt == 1) attn_item<1, 4>(C, t, it);
    else if (mt == 2) attn_item<2, 4>(C, t, it);
    else attn_item<3, 4>(C, t, it);
  }
}

// ---------------------------------------------------------------------------
// multi-head latent attention items (absorbed form)
// ---------------------------------------------------------------------------
// The cache holds per position the latent row [c (R) | k_rope (dr)], shared by
// all heads.  With the key up-projection absorbed into the query
// (q_abs,h = W_uk,h^T q_nope,h, computed by the preceding grouped GEMV), the
// score of head h at position t is (q_abs,h . c_t + q_rope,h . k_rope,t) /
// sqrt(dn + dr), and the head's value is W_uv,h applied to sum_t p_t c_t
// (the following grouped GEMV).  So one item attends one query row over a
// range of latent rows with all heads as the mma M dimension: multi-query
// attention with 576-wide keys and 512-wide values.
struct MlaState {
  float o[2][8][4];  // [m-tile][latent-dim tile of this warp][frag]
  float M[2][2];     // running max (log2 units) of rows g, g + 8 of each m-tile
  float L[2][2];     // lane-partial running sums
};

__device__ __forceinline__ void mla_chunk(const Ctx& C, MlaState& st, const uint8_t* rows, int n_valid, int mt,
                                          int KW, int NTW, int pitch, int par, const MlaLayout& lay) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  uint8_t* base = C.xring;
  const uint8_t* qhi = base + lay.qhi;
  const uint8_t* qlo = base + lay.qlo;
  uint8_t* phi = base + lay.phi;
  uint8_t* plo = base + lay.plo;
  float* smx = reinterpret_cast<float*>(base + lay.smax) + par * NCW * 32;

  // ---- scores of positions [8 warp, 8 warp + 8) over all KW k-steps ----
  float sacc[2][4];
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) sacc[mi][0] = sacc[mi][1] = sacc[mi][2] = sacc[mi][3] = 0.f;
  const int n0 = warp * 8;
  if (n0 < n_valid) {
    const uint8_t* krow = rows + (size_t)(n0 + g) * pitch + tq * 4;
#pragma unroll 2
    for (int ks = 0; ks < KW; ++ks) {
      const uint32_t b0 = lds32(krow + ks * 32);
      const uint32_t b1 = lds32(krow + ks * 32 + 16);
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        if (mi < mt) {
          const uint4 ah = lds128(qhi + ((mi * KW + ks) * 32 + lane) * 16);
          const uint4 al = lds128(qlo + ((mi * KW + ks) * 32 + lane) * 16);
          mma_bf16(sacc[mi], ah, b0, b1);
          mma_bf16(sacc[mi], al, b0, b1);
        }
      }
    }
  }
  const int p0 = n0 + 2 * tq, p1 = p0 + 1;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
    if (mi < mt) {
      if (p0 >= n_valid) sacc[mi][0] = sacc[mi][2] = -INFINITY;
      if (p1 >= n_valid) sacc[mi][1] = sacc[mi][3] = -INFINITY;
      float mA = fmaxf(sacc[mi][0], sacc[mi][1]), mB = fmaxf(sacc[mi][2], sacc[mi][3]);
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
      if (tq == 0) {
        smx[warp * 32 + mi * 16 + g] = mA;
        smx[warp * 32 + mi * 16 + g + 8] = mB;
      }
    }
  }
  bar_consumers();
  // ---- online softmax; P written as A fragments (k-step warp / 2) ----
  const int kt = warp >> 1;
  const int regA = (warp & 1) ? 2 : 0;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
    if (mi < mt) {
      float cm[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        cm[0] = fmaxf(cm[0], smx[w * 32 + mi * 16 + g]);
        cm[1] = fmaxf(cm[1], smx[w * 32 + mi * 16 + g + 8]);
      }
      float pv[4];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const float mnew = fmaxf(st.M[mi][h2], cm[h2]);
        const float corr = (mnew == -INFINITY) ? 1.f : exp2f(st.M[mi][h2] - mnew);
        const float msafe = (mnew == -INFINITY) ? 0.f : mnew;
        st.M[mi][h2] = mnew;
        pv[2 * h2 + 0] = exp2f(sacc[mi][2 * h2 + 0] - msafe);
        pv[2 * h2 + 1] = exp2f(sacc[mi][2 * h2 + 1] - msafe);
        st.L[mi][h2] = st.L[mi][h2] * corr + pv[2 * h2 + 0] + pv[2 * h2 + 1];
#pragma unroll
        for (int jn = 0; jn < 8; ++jn) {
          st.o[mi][jn][2 * h2 + 0] *= corr;
          st.o[mi][jn][2 * h2 + 1] *= corr;
        }
      }
      uint32_t hA, lA, hB, lB;
      split_bf16(pv[0], pv[1], hA, lA);
      split_bf16(pv[2], pv[3], hB, lB);
      uint32_t* ph = reinterpret_cast<uint32_t*>(phi + ((mi * 4 + kt) * 32 + lane) * 16);
      uint32_t* pl = reinterpret_cast<uint32_t*>(plo + ((mi * 4 + kt) * 32 + lane) * 16);
      ph[regA] = hA;
      ph[regA + 1] = hB;
      pl[regA] = lA;
      pl[regA + 1] = lB;
    }
  }
  bar_consumers();
  // ---- O += P C over this warp's latent dims [8 NTW warp, 8 NTW (warp + 1)) ----
  for (int ks = 0; ks < 4; ++ks) {
    if (ks * 16 >= n_valid) break;
    const int pk = ks * 16 + 2 * tq;
    uint4 ah[2], al[2];
#pragma unroll
    for (int mi = 0; mi < 2; ++mi) {
      if (mi < mt) {
        ah[mi] = lds128(phi + ((mi * 4 + ks) * 32 + lane) * 16);
        al[mi] = lds128(plo + ((mi * 4 + ks) * 32 + lane) * 16);
      }
    }
    // B fragments of C by transposed 8x8 matrix loads; lanes 0-15 address
    // the 16 positions of the k-step (clamped to the valid rows: the rows
    // past n_valid are masked below), 16-byte aligned since the pitch is
    const uint8_t* vrow = rows + (size_t)min(ks * 16 + (lane & 15), n_valid - 1) * pitch;
#pragma unroll
    for (int jn = 0; jn < 8; ++jn) {
      if (jn < NTW) {
        uint32_t b0, b1;
        ldsm_x2_trans(vrow + (size_t)((warp * NTW + jn) * 8) * 2, b0, b1);
        if (pk >= n_valid) b0 = 0u;
        else if (pk + 1 >= n_valid) b0 &= 0xFFFFu;
        if (pk + 8 >= n_valid) b1 = 0u;
        else if (pk + 9 >= n_valid) b1 &= 0xFFFFu;
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          if (mi < mt) {
            mma_bf16(st.o[mi][jn], ah[mi], b0, b1);
            mma_bf16(st.o[mi][jn], al[mi], b0, b1);
          }
        }
      }
    }
  }
}

__device__ MK_MLA_ATTR void mla_task(const Ctx& C, const Task& t, uint32_t& it) {
  const Launch& P = *C.P;
  const Model& md = *C.md;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const bool trc = MK_TRACE && P.trace && threadIdx.x == 0;
  long long tA = trc ? clock64() : 0;
  const Item itm = decode_item(t.rt0, P.n_pairs, P.n_items);
  const int mrow = itm.pair, Q = P.Q, s = mrow / Q, qi = mrow % Q;
  const int Hq = md.Hq, R = md.R, dr = md.dr, dn = md.d, W = R + dr, KW = W / 16, mt = (Hq + 15) >> 4;
  const int pitch = mla_pitch(R, dr), MCT = mla_ct(R, dr), NTW = R / 64;
  const MlaLayout lay = mla_layout(Hq, R, dr);
  const int T0 = seq_pos0(P, s);
  const int a = (int)(((int64_t)itm.j * T0) / itm.ns), b = (int)(((int64_t)(itm.j + 1) * T0) / itm.ns);
  const bool last = itm.j == itm.ns - 1;
  const float qscale = rsqrtf((float)(dn + dr)) * 1.4426950408889634f;
  const float* qkv = P.buf[B_QKV];
  const int ldq = P.ld[B_QKV];
  const float* qa = P.buf[B_QL];
  const int lda = P.ld[B_QL];
  const int QW = Hq * (dn + dr), half = dr / 2;
  const float2* rope = md.rope;
  uint8_t* base = C.xring;
  uint8_t* qhi = base + lay.qhi;
  uint8_t* qlo = base + lay.qlo;

  // ---- queries as bf16 hi / lo A fragments scaled to log2 units: first the
  //      rotary part (RoPE at this row's position) and the step's own latent
  //      rows, which need only the QKV projection (done: this CTA's absorbing
  //      projection task waited for it), then, once every CTA's absorbing
  //      projection is done, the absorbed latent part ----
  const int pos = T0 + qi;
  for (int e = tid; e < mt * 16 * half; e += NCT) {
    const int r = e / half, i = e - r * half;
    float x0 = 0.f, x1 = 0.f;
    if (r < Hq) {
      const float* q = qkv + (size_t)mrow * ldq + (size_t)r * (dn + dr) + dn;
      const float a0 = __ldcg(q + i), a1 = __ldcg(q + i + half);
      const float2 cs = __ldg(rope + (size_t)pos * half + i);
      x0 = (a0 * cs.x - a1 * cs.y) * qscale;
      x1 = (a0 * cs.y + a1 * cs.x) * qscale;
    }
    const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
    *reinterpret_cast<__nv_bfloat16*>(qhi + frag_off(r, R + i, KW)) = h0;
    *reinterpret_cast<__nv_bfloat16*>(qhi + frag_off(r, R + i + half, KW)) = h1;
    *reinterpret_cast<__nv_bfloat16*>(qlo + frag_off(r, R + i, KW)) = __float2bfloat16_rn(x0 - __bfloat162float(h0));
    *reinterpret_cast<__nv_bfloat16*>(qlo + frag_off(r, R + i + half, KW)) =
        __float2bfloat16_rn(x1 - __bfloat162float(h1));
  }
  // ---- the step's own latent rows 0..qi of this sequence (RoPE on k_rope, bf16);
  //      row qi is this query's position and is appended to the cache here ----
  uint8_t* newr = base + lay.newr;
  if (last) {
    __nv_bfloat16* cache = reinterpret_cast<__nv_bfloat16*>(P.kv_k) +
                           (((size_t)t.layer * P.kv_seqs + s) * (size_t)P.kv_ctx + pos) * W;
    const int per = R + half;
    for (int e = tid; e < (qi + 1) * per; e += NCT) {
      const int j = e / per, k = e - j * per;
      const float* src = qkv + (size_t)(s * Q + j) * ldq + QW;
      __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(newr + (size_t)j * pitch);
      if (k < R) {
        const __nv_bfloat16 v = __float2bfloat16_rn(__ldcg(src + k));
        row[k] = v;
        if (j == qi) cache[k] = v;
      } else {
        const int i = k - R;
        const float a0 = __ldcg(src + R + i), a1 = __ldcg(src + R + i + half);
        const float2 cs = __ldg(rope + (size_t)(T0 + j) * half + i);
        const __nv_bfloat16 k0 = __float2bfloat16_rn(a0 * cs.x - a1 * cs.y);
        const __nv_bfloat16 k1 = __float2bfloat16_rn(a0 * cs.y + a1 * cs.x);
        row[R + i] = k0;
        row[R + i + half] = k1;
        if (j == qi) {
          cache[R + i] = k0;
          cache[R + i + half] = k1;
        }
      }
    }
  }
  if (t.wait_ctr >= 0) wait_counter(C, t.wait_ctr, (uint32_t)t.wait_tgt);
  {
    // the latent part arrives in fragment layout (written by the absorbing
    // projection's epilogue): per row tile, R / 16 contiguous tiles, hi then
    // lo; four bulk copies (every item of the step reads these same bytes at
    // once, which the copy engine serves far better than per-thread loads)
    const int KWl = R >> 4, tiles = mt * KWl;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(qa + (size_t)mrow * lda);
    uint64_t* qb = &C.ms->qbar;
    const uint32_t par = C.ms->qpar & 1u;
    if (tid == 0 && !C.ms->abort) {
      // earlier generic-proxy accesses of this scratch precede the copies
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(qb, (uint32_t)(2 * tiles * 512));
      const uint64_t pol = policy_evict_last();
      for (int hl = 0; hl < 2; ++hl)
        for (int mi = 0; mi < mt; ++mi)
          bulk_g2s((hl ? qlo : qhi) + (size_t)mi * KW * 512, src + ((size_t)hl * tiles + (size_t)mi * KWl) * 512,
                   (uint32_t)(KWl * 512), qb, pol);
    }
    if (lane == 0 && !C.ms->abort) {
      uint32_t spins = 0;
      uint64_t w0 = 0;
      while (!mbar_try_wait(qb, par)) {
        if (++spins >= 64) {
          spins = 0;
          if (C.ms->abort) break;
          const uint64_t now = globaltimer();
          if (w0 == 0) w0 = now;
          else if (now - w0 > (uint64_t)P.timeout_ns * 2) {
            raise_error(P, C.ms, DERR_TIMEOUT, 0x5A000);
            break;
          }
        }
      }
    }
    __syncwarp();
    if (!C.ms->abort) while (!mbar_try_wait(qb, par)) {}
    if (Hq < mt * 16) {  // rows past the last head: zero (nothing writes them)
      const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
      for (int e = tid; e < (mt * 16 - Hq) * R; e += NCT) {
        const int r = Hq + e / R, k = e % R;
        *reinterpret_cast<__nv_bfloat16*>(qhi + frag_off(r, k, KW)) = z;
        *reinterpret_cast<__nv_bfloat16*>(qlo + frag_off(r, k, KW)) = z;
      }
    }
  }
  bar_consumers();
  if (tid == 0) C.ms->qpar += 1;  // every thread has read it; read again after the next item's dependency barrier
  if (trc) {
    const long long t1 = clock64();
    C.ms->tr_pre += t1 - tA;
    tA = t1;
  }

  MlaState st;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
    st.M[mi][0] = st.M[mi][1] = -INFINITY;
    st.L[mi][0] = st.L[mi][1] = 0.f;
#pragma unroll
    for (int jn = 0; jn < 8; ++jn) st.o[mi][jn][0] = st.o[mi][jn][1] = st.o[mi][jn][2] = st.o[mi][jn][3] = 0.f;
  }
  int par = 0;
  for (int t0 = a; t0 < b; t0 += MCT) {
    const int n = min(MCT, b - t0);
    wait_full(C, it);
    const uint8_t* stage = C.ring + (size_t)(it % NSTAGE) * STAGE_BYTES;
    mla_chunk(C, st, stage, n, mt, KW, NTW, pitch, par, lay);
    par ^= 1;
    bar_consumers();  // every warp is done with the stage
    release_stage(C, it);
    ++it;
  }
  if (last) {
    mla_chunk(C, st, newr, qi + 1, mt, KW, NTW, pitch, par, lay);
    par ^= 1;
  }
  bar_consumers();
  if (trc) {
    const long long t1 = clock64();
    C.ms->tr_loop += t1 - tA;
    tA = t1;
  }

  // ---- the item's partial (M, L, O) per head ----
  float* smx = reinterpret_cast<float*>(base + lay.smax);
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
    if (mi < mt) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float l = st.L[mi][h2];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (tq == 0) smx[warp * 32 + mi * 16 + g + 8 * h2] = l;
      }
    }
  }
  bar_consumers();
  const int rows_max = P.att_rows_max, dP = R + 4;  // O (R) | M | L | 2 pad
  float* part = P.att_part + (size_t)t.rt0 * rows_max * dP;
  if (tid < Hq) {
    float l = 0.f;
    for (int w = 0; w < NCW; ++w) l += smx[w * 32 + tid];
    part[(size_t)tid * dP + R + 1] = l;
  }
  if (warp == 0 && tq == 0) {
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
      if (mi < mt) {
        if (mi * 16 + g < Hq) part[(size_t)(mi * 16 + g) * dP + R] = st.M[mi][0];
        if (mi * 16 + g + 8 < Hq) part[(size_t)(mi * 16 + g + 8) * dP + R] = st.M[mi][1];
      }
  }
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
    if (mi < mt) {
#pragma unroll
      for (int jn = 0; jn < 8; ++jn) {
        if (jn < NTW) {
          const int dim = (warp * NTW + jn) * 8 + 2 * tq;
          const int rA = mi * 16 + g, rB = rA + 8;
          if (rA < Hq) {
            part[(size_t)rA * dP + dim] = st.o[mi][jn][0];
            part[(size_t)rA * dP + 1 + dim] = st.o[mi][jn][1];
          }
          if (rB < Hq) {
            part[(size_t)rB * dP + dim] = st.o[mi][jn][2];
            part[(size_t)rB * dP + 1 + dim] = st.o[mi][jn][3];
          }
        }
      }
    }
  }
  // this region is the activation ring, which bulk copies write again later
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  bar_consumers();
  if (trc) {
    const long long t1 = clock64();
    C.ms->tr_post += t1 - tA;
    tA = t1;
  }

  (void)trc;
}

// The split combine of every query row's latent attention, spread over all
// CTAs: CTA c owns a contiguous slice of the outputs [pair][head][R] and
// forms each as sum_j exp2(M_j - M*) O_j / sum_j exp2(M_j - M*) L_j over the
// pair's splits j (fixed order).
__device__ __noinline__ void mla_comb_task(const Ctx& C, const Task& t) {
  const Launch& P = *C.P;
  const Model& md = *C.md;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = md.Hq, R = md.R, dP = R + 4, rows_max = P.att_rows_max;
  // slices of whole float4 groups (R is a multiple of 64, so a group never
  // straddles two rows)
  const int64_t total4 = (int64_t)P.n_pairs * Hq * (R / 4);
  const int64_t q0 = total4 * blockIdx.x / gridDim.x, q1 = total4 * (blockIdx.x + 1) / gridDim.x;
  if (q0 >= q1) return;
  float* out = P.buf[B_OL];
  const int ldo = P.ld[B_OL];
  float* wsh = reinterpret_cast<float*>(C.att);                  // [row][160] split weights
  float4* red = reinterpret_cast<float4*>(C.att + 32 * 160 * 4);  // [split group][unit]
  const int R4 = R / 4;
  const int row0 = (int)(q0 / R4), row1 = (int)((q1 - 1) / R4) + 1;
  for (int rb = row0; rb < row1; rb += 32) {
    const int re = min(row1, rb + 32);
    const int64_t a = max(q0, (int64_t)rb * R4), b = min(q1, (int64_t)re * R4);
    for (int rr = rb + warp; rr < re; rr += NCW) {
      const int pair = rr / Hq, h = rr - pair * Hq;
      const Item itm = decode_item(pair_first_item(pair, P.n_pairs, P.n_items), P.n_pairs, P.n_items);
      const int ns = itm.ns;
      float mj[5], lj[5];
      float mx = -INFINITY;
#pragma unroll
      for (int q = 0; q < 5; ++q) {
        const int jj = lane + 32 * q;
        mj[q] = -INFINITY;
        lj[q] = 0.f;
        if (jj < ns) {
          const float* pp = P.att_part + ((size_t)(itm.first + jj) * rows_max + h) * dP + R;
          mj[q] = __ldcg(pp);
          lj[q] = __ldcg(pp + 1);
        }
        mx = fmaxf(mx, mj[q]);
      }
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float den = 0.f, w[5];
#pragma unroll
      for (int q = 0; q < 5; ++q) {
        w[q] = (mj[q] == -INFINITY) ? 0.f : exp2f(mj[q] - mx);
        den += w[q] * lj[q];
      }
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
#pragma unroll
      for (int q = 0; q < 5; ++q) {
        const int jj = lane + 32 * q;
        if (jj < ns) wsh[(rr - rb) * 160 + jj] = w[q] / den;
      }
    }
    bar_consumers();
    // units of 4 outputs; when there are fewer units than threads, the
    // splits of each unit are shared by `sg_n` thread groups and the groups'
    // sums added in group order
    const int units = (int)(b - a);
    const int sg_n = max(1, min(NCT / max(units, 1), 16));
    for (int base = 0; base < units; base += NCT / sg_n) {
      const int per = NCT / sg_n;
      const int u = base + tid % per, sg = tid / per;
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
      if (u < units && sg < sg_n) {
        const int64_t q = a + u;
        const int rr = (int)(q / R4), k = (int)(q - (int64_t)rr * R4) * 4;
        const int pair = rr / Hq, h = rr - pair * Hq;
        const Item itm = decode_item(pair_first_item(pair, P.n_pairs, P.n_items), P.n_pairs, P.n_items);
        const float* wr = wsh + (rr - rb) * 160;
        const float* src = P.att_part + ((size_t)itm.first * rows_max + h) * dP + k;
        const size_t js = (size_t)rows_max * dP;
#pragma unroll 16
        for (int jj = sg; jj < itm.ns; jj += sg_n) {
          const float wv = wr[jj];
          const float4 v = __ldcg(reinterpret_cast<const float4*>(src + jj * js));
          num.x += wv * v.x;
          num.y += wv * v.y;
          num.z += wv * v.z;
          num.w += wv * v.w;
        }
      }
      if (sg < sg_n) red[sg * per + tid % per] = num;
      bar_consumers();
      if (tid < per && base + tid < units) {
        float4 tot = red[tid];
        for (int g2 = 1; g2 < sg_n; ++g2) {
          const float4 v = red[g2 * per + tid];
          tot.x += v.x;
          tot.y += v.y;
          tot.z += v.z;
          tot.w += v.w;
        }
        const int64_t q = a + base + tid;
        const int rr = (int)(q / R4), k = (int)(q - (int64_t)rr * R4) * 4;
        const int pair = rr / Hq, h = rr - pair * Hq;
        float* orow = out + (size_t)pair * ldo;
        st_frag(orow, h * R + k, tot.x, false);
        st_frag(orow, h * R + k + 1, tot.y, false);
        st_frag(orow, h * R + k + 2, tot.z, false);
        st_frag(orow, h * R + k + 3, tot.w, false);
      }
      bar_consumers();
    }
  }
}

// ---------------------------------------------------------------------------
// consumer warps
// ---------------------------------------------------------------------------
template <bool MLA, int MOE>
__device__ void consumer(const Ctx& C) {
  const Launch& P = *C.P;
  uint32_t it = 0, ix = 0, tc = 0;
  if (P.stall_ctr >= 0) {
    // test hook: a dependency that nothing signals
    wait_counter(C, P.stall_ctr, 1u);
    return;
  }
  const int beg = P.task_off[blockIdx.x], end = task_end_of(P);
  phase_dependency_wait(P);
  for (int ti = beg; ti < end; ++ti) {
    // the task record into shared memory, once every consumer thread is done
    // with the previous one (not every task ends with a barrier: a task
    // without a signal, or thread 0's trace record after it)
    bar_consumers();
    for (int i = threadIdx.x; i < (int)(sizeof(Task) / 4); i += NCT)
      reinterpret_cast<uint32_t*>(&C.ms->ctask)[i] = __ldg(reinterpret_cast<const uint32_t*>(P.tasks + ti) + i);
    bar_consumers();
    const Task& t = C.ms->ctask;
    // while this task waits and runs: the next task's record into L1, and
    // the gain that this task's x updates are multiplied by for the next norm
    if (ti + 1 < end && threadIdx.x < 3) {
      const uintptr_t a = reinterpret_cast<uintptr_t>(P.tasks + ti + 1);
      const uintptr_t line = (a & ~(uintptr_t)127) + threadIdx.x * 128;
      if (line < a + sizeof(Task)) prefetch_l1(reinterpret_cast<const void*>(line));
    }
    if (t.gnext) {
      const int lines = (C.md->H * 2 + 127) / 128;
      for (int i = threadIdx.x; i < lines; i += NCT) prefetch_l1(reinterpret_cast<const char*>(t.gnext) + i * 128);
    }
    const bool tr = MK_TRACE && P.trace && (ti - beg) < P.trace_cap && threadIdx.x == 0;
    uint64_t tb = 0, td = 0;
    if (tr) {
      tb = globaltimer();
      C.ms->tr_wf = C.ms->tr_wx = C.ms->tr_bytes = 0;
      C.ms->tr_frag = C.ms->tr_mma = C.ms->tr_epi = C.ms->tr_rel = 0;
      C.ms->tr_loop = C.ms->tr_pre = C.ms->tr_post = C.ms->tr_sig = 0;
      C.ms->tr_route = 0;
      C.ms->tr_chunks = 0;
    }
    // a latent-attention item stages what it can before its dependency and
    // waits inside
    if (t.wait_ctr >= 0 && !(MLA && t.type == T_MLA)) wait_counter(C, t.wait_ctr, (uint32_t)t.wait_tgt);
    if (tr) td = globaltimer();
    if (gemv_like<MOE>(t)) {
      gemv_task<MLA, MOE>(C, t, it, ix, tc);
    } else if (!MLA && t.type == T_ATTN) {
      attn_task(C, t, it);
    } else if (MLA && t.type == T_MLA) {
      mla_task(C, t, it);
    } else if (MLA && t.type == T_MLA_COMB) {
      mla_comb_task(C, t);
    } else if (t.type == T_EMBED) {
      embed_task(C, t);
    }
    const long long tsg = tr ? clock64() : 0;
    if (t.type == T_GEMV && t.epi == EPI_LOGITS) lm_finish(C);
    else if (t.sig_ctr >= 0) signal_counter(C, t.sig_ctr);
    if (tr) C.ms->tr_sig += clock64() - tsg;
    if (tr) {
      int64_t* rec = P.trace + ((size_t)blockIdx.x * P.trace_cap + (ti - beg)) * TRACE_FIELDS;
      rec[0] = (int64_t)tb;
      rec[1] = (int64_t)td;
      rec[2] = (int64_t)globaltimer();
      rec[3] = C.ms->tr_wf;
      rec[4] = C.ms->tr_wx;
      rec[5] = C.ms->tr_chunks;
      rec[6] = (int64_t)t.layer | ((int64_t)t.phase << 16);  // layer, and the phase (multi-kernel split) above bit 16
      rec[7] = (int64_t)t.type * 16 + t.epi;
      rec[8] = C.ms->tr_frag;
      rec[9] = C.ms->tr_mma;
      rec[10] = C.ms->tr_epi;
      rec[11] = C.ms->tr_rel;
      rec[16] = C.ms->tr_loop;
      rec[17] = C.ms->tr_pre;
      rec[18] = C.ms->tr_post;
      rec[19] = C.ms->tr_sig;
      if (ti - beg >= 2) rec[12] = C.ms->tr_route;  // records 0 and 1 carry the producer's counters there
    }
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// One instance per model family (GQA or latent attention, dense or MoE FFN): each kernel holds only
// the code its models run, which keeps the instruction footprint of the
// whole-step loop small.
// 10 warps put 3 warps on two of the SM's four register-file partitions
// (16K registers each), so a thread gets at most 168 registers.
template <bool MLA, int MOE>
__global__ void __launch_bounds__(NTHREADS, 1) mk_step_kernel(const __grid_constant__ Launch P) {
  extern __shared__ __align__(128) uint8_t smem[];
  Ctx C;
  C.P = &P;
  C.md = P.model;
  C.ring = smem;
  C.xring = smem + (size_t)NSTAGE * STAGE_BYTES;
  C.att = C.xring + (size_t)XSLOTS * XSLOT_BYTES;
  C.newkv = C.att + ATT_BYTES;
  C.ms = reinterpret_cast<Misc*>(C.newkv + NEWKV_BYTES);
  C.ncta = gridDim.x;
  const int tid = threadIdx.x;

  // ---- input validation (every CTA checks, so all return together) ----
  int bad = 0;
  if (tid < P.M) {
    const int tok = __ldg(P.tokens + tid);
    if (tok < 0 || tok >= C.md->V) bad = 1;
  }
  if (tid < P.S) {
    const int p0 = seq_pos0(P, tid);
    if (p0 < 0 || p0 + P.Q > P.kv_ctx || p0 + P.Q > C.md->rope_ctx) bad = 1;
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0 && blockIdx.x == 0) {
      atomicCAS(P.status, 0, DERR_BOUNDS);
      atomicExch(P.status + 1, 1);
    }
    return;
  }
  for (int i = tid; i < (int)(sizeof(Model) / 4); i += NTHREADS)
    reinterpret_cast<uint32_t*>(&C.ms->cmodel)[i] = __ldg(reinterpret_cast<const uint32_t*>(P.model) + i);
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&C.ms->full[s], 1);
      mbar_init(&C.ms->empty[s], NCW + (NTS > 0 ? 1 : 0));
    }
    for (int t = 0; t < NTS; ++t) {
      mbar_init(&C.ms->tfull[t], 1);
      mbar_init(&C.ms->tempty[t], NCW);
    }
    for (int s = 0; s < XSLOTS; ++s) {
      mbar_init(&C.ms->xfull[s], 2);  // the copies' expect-tx arrival + the scales
      mbar_init(&C.ms->xempty[s], NCW);
    }
    mbar_init(&C.ms->qbar, 1);
    C.ms->qpar = 0;
    C.ms->abort = 0;
    C.ms->route_layer = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the next phase kernel may be scheduled as soon as SMs free up
  if (P.phase_mode == 1) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (NTS > 0 && (tid >> 5) == WARP_MV) tmem_alloc(&C.ms->tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  C.tmem = C.ms->tmem_base;
  C.md = &C.ms->cmodel;

  if ((tid >> 5) == WARP_WP) producer<MLA, MOE>(C);
  else if ((tid >> 5) == WARP_XP) xproducer<MOE>(C);
  else if ((tid >> 5) == WARP_MV) mover(C);
  else consumer<MLA, MOE>(C);
  tc_fence_before();
  __syncthreads();
  // every TMEM read and copy of the CTA has completed: free the columns
  if (NTS > 0 && (tid >> 5) == WARP_MV) {
    tc_fence_after();
    tmem_dealloc(C.tmem, TMEM_COLS);
  }

  // ---- teardown: the last CTA out zeroes every counter for the next launch ----
  // (a phase kernel other than the step's last leaves them to later phases)
  if (P.phase_mode == 1) return;
  if (tid == 0) {
    int last = 0;
    if (!global_abort(P)) {
      __threadfence();
      const uint32_t old = atom_add_acqrel(P.ctr + P.ctr_done, 1u);
      last = (old == (uint32_t)C.ncta - 1);
    }
    C.ms->flag = last;
  }
  __syncthreads();
  if (C.ms->flag) {
    for (int i = tid; i < P.n_ctr; i += NTHREADS) P.ctr[i] = 0u;
    __threadfence();
  }
}

// The host code (another translation unit) takes the kernel instances from here.
const void* step_kernel_for(bool mla, bool moe, bool fp8) {
  // MOE: 0 dense FFN, 1 MoE with bf16 experts, 2 MoE with fp8 experts
  if (mla) {
    if (!moe) return (const void*)mk_step_kernel<true, 0>;
    return fp8 ? (const void*)mk_step_kernel<true, 2> : (const void*)mk_step_kernel<true, 1>;
  }
  if (!moe) return (const void*)mk_step_kernel<false, 0>;
  return fp8 ? (const void*)mk_step_kernel<false, 2> : (const void*)mk_step_kernel<false, 1>;
}

}  // namespace MK_KNS
}  // namespace mk

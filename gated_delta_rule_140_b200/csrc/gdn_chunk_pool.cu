// gdn_chunk_pool.cu -- chunkwise gated delta rule prefill on the tensor cores
// with the chunk-local work spread over a pool of SMs and the sequential state
// pass on dedicated "chain" SMs: one persistent CTA per SM, bf16 inputs,
// d_k = d_v = 128, scalar decay (Gated DeltaNet).
//
// Chunkwise form (FG2-GDN paper, section 3.6: WY representation, UT
// transform, inter-chunk state propagation; Gated Delta Networks page,
// section 3.3, for the cumulative decay g_r inside a chunk), C = 64 tokens,
// g_r = sum_{t<=r} log alpha_t, gamma_r = e^{g_r}:
//
//   A_rs = beta_r e^{g_r-g_s} k_r.k_s (s < r),   T = (I + A)^{-1}
//   P_rs = e^{g_r-g_s} q_r.k_s (s <= r),          T_b = T diag(beta)
//   W = T_b diag(gamma) K,  U = T_b V,  Kt_r = e^{g_C-g_r} k_r
//   V' = U - W S^T,  S <- e^{g_C} S + V'^T Kt,  o = (gamma.Q) S^T + P V'.
//
// Regrouped so that the sequential chain is ONE product per chunk:
//   S <- e^{g_C} S + V^T Z + S G,    Z = T_b^T Kt (C x d_k),  G = -W^T Kt (d_k x d_k)
//   o^T = S Qh^T + V^T R^T,          Qh = gamma.Q - P W,  R = P T_b
// (V'^T Kt = U^T Kt - S W^T Kt; o = (gamma.Q - P W) S^T + P T_b V).
//
// Roles (blockIdx.x < nch: chain CTA b; otherwise a local CTA of the pool):
//  * Local CTAs take chunk tasks in a fixed global order (round by round, and
//    inside a round chunk-major over the round's chains; local CTA c takes
//    tasks c, c + nloc, c + 2 nloc, ...).  Two groups of 8 warps work on
//    alternate tasks of the CTA, with three raw K/Q tile buffers between them.
//    Per task: [K;Q] K^T on the tensor cores; A and P with the decay (exact
//    exponentials inside each row's own 16-token block, factored at the block
//    boundaries elsewhere, both factors <= 1); T by blocked forward
//    substitution (fp32 16x16 diagonal blocks, tf32 MMAs above them);
//    [P T_bg | R] = P [T_bg | T_b]; [W; P W] = [T_bg; P T_bg] K; then -W, Qh and
//    Kt.  The tiles T_b, -W, Kt, Qh, R (64 KB, bf16, in the layouts the chain
//    CTA's MMAs read) and e^{g_C} go by bulk copy into a ring slot in global
//    memory (chain CTA b, slot m % 4), L2-resident; a release store of the
//    slot's tag hands it over.
//  * Chain CTA b owns the chains b, b + nch, ... one after another, S (fp32)
//    in registers of 8 warps (thread = value row j, 64 key columns).  Per
//    chunk: a loader thread bulk-loads the slot and TMA-loads the V tile into
//    one of two stages; X = Kt^T [T_b | -W] (one M=128, N=192 MMA) gives Z^T and
//    G^T, which 4 warps write back as bf16 operands; D_S = V^T Z (issued ahead)
//    and then the chain product D_S += S G; the 8 state warps update
//    S <- e^{g_C} S + D_S and write it back as the bf16 operand of the next
//    chunk; D_O = V^T R^T + S Qh^T = o^T, which 4 warps write out.
//
// The hand-offs through global memory: ready[b][slot] holds the tag of the
// (round, chunk) written there; cons[b] the chain CTA's progress (round,
// chunks consumed), which a local CTA waits for before it rewrites a slot.
// All CTAs are co-resident (cooperative launch, one CTA per SM).  Every wait is
// bounded: on expiry a CTA records kErrTimeout, raises the grid-wide abort
// word, drains what it issued and returns.
#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = kChunk;  // 64
constexpr int DK = 128, DV = 128;
constexpr int kThreads = 512;                      // 16 warps
constexpr long long kWaitLimit = kDefaultWaitLimit;  // drains after an abort
constexpr int LDA = 68;                            // fp32 row stride of A / T
constexpr int NR = 8;                              // ring slots per chain CTA
constexpr int kFlagWords = 16;                     // per chain CTA: cons, ready[NR], pad

// ---- ring slot (global) and chain-CTA buffers (shared), bytes ----------------
// slot: [e^{g_C} x128 (1 KB) | Z^T | R] then two 64-wide atoms [Y_h | Qh_h] of
// the key dimension (Y = G^T).  Z^T and Y have 128 rows (16 KB per atom), R and
// Qh 64 rows (8 KB); every tile bf16, K-major, 128-byte swizzled, so that
// [Z^T; R] (N = 192, K = 64 tokens) and [Y; Qh] (N = 192, K = d_k) are the B
// operands of the chain CTA's two products V^T [Z | R^T] and S [Y^T | Qh^T]:
// one accumulator holds the state increment (columns 0-127) and o^T (128-191).
// The chain CTA loads a slot, and V (one TMA load of both 64-wide halves), into
// one of two stages.
constexpr uint32_t RG_DEC = 0, RG_ZT = 1024, RG_R = RG_ZT + 16384, RG_YQ = RG_R + 8192;
constexpr uint32_t YQ_HALF = 24576, YQ_QH = 16384;  // atom stride; Qh inside an atom
constexpr uint32_t RG_BYTES = RG_YQ + 2 * YQ_HALF;
constexpr uint32_t RING_STRIDE = RG_BYTES;
constexpr uint32_t CS_V = RG_BYTES, CS_BYTES = RG_BYTES + 16384;
constexpr uint32_t STAGE_TX = CS_BYTES;
// o tiles of the output warps: two buffers of two 64 x 64 halves (bf16, 128-byte
// swizzled), written back by TMA tensor stores
constexpr uint32_t OFF_OBUF = 2 * CS_BYTES, OBUF_BYTES = 16384;
static_assert((RG_ZT | RG_R | RG_YQ | YQ_HALF | YQ_QH | CS_V | CS_BYTES) % 1024 == 0, "chain buffer layout");

// ---- local-CTA layout (GDN) -------------------------------------------------
// three raw tile buffers [K0 | Q0 | K1 | Q1] shared by the two groups (task k in
// buffer k % 3; Kt replaces K in place), then per group [P | X1 | X2 | X3]
// (X1 = T_bg, X2 = P T_bg, X3 = T_b), A and then T in place (fp32 [64][LDA]),
// and two gate-row buffers.
constexpr uint32_t L_RAW_AC = 16384, RAW_BYTES = 32768;
constexpr uint32_t PZ_P = 0, PZ_X1 = 8192, PZ_X2 = 16384, PZ_X3 = 24576, PZT_BYTES = 32768;
constexpr uint32_t AT_BYTES = 64 * LDA * 4;
constexpr uint32_t GATES_STRIDE = 3584;
constexpr uint32_t L_G0 = 3 * RAW_BYTES;
constexpr uint32_t L_PZT = 0, L_AT = PZT_BYTES, L_GATES = L_AT + AT_BYTES;
constexpr uint32_t L_GSZ = L_GATES + 2 * GATES_STRIDE;
static_assert(L_GATES % 1024 == 0 && L_GSZ % 1024 == 0, "local group layout");
// gate rows (floats): g beta beta*gamma colf rowf[4] kh gamma, e^{g_C} x128, and
// (raw inputs) the inverse key and query norms of the task's rows
constexpr int GR_G = 0, GR_B = 64, GR_BG = 128, GR_COLF = 192, GR_ROWF = 256, GR_KH = 512,
              GR_GAM = 576, GR_DEC = 640, GR_INVK = 768, GR_INVQ = 832;

// ---- bookkeeping (same offset in both roles) --------------------------------
constexpr uint32_t OFF_COMMON = OFF_OBUF + 2 * OBUF_BYTES;  // 215040
static_assert(L_G0 + 2 * L_GSZ <= OFF_COMMON, "local shared memory layout");
constexpr uint32_t CM_ABORT = 0, CM_TMEM = 8, CM_ISSUED = 16, CM_LANDED = 48, CM_BARS = 64;  // issued: 8 ints
constexpr int NBARS = 24;
// local CTAs: the descriptors of their first kDescCache tasks
constexpr int kDescCache = 960;
constexpr uint32_t OFF_DESC = OFF_COMMON + 256;
static_assert(CM_BARS + NBARS * 8 <= 256, "bookkeeping");
constexpr uint32_t SMEM_USED = OFF_DESC + kDescCache * 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
// chain-CTA mbarriers
// (FULL: a stage's loads landed; DSFULL: a chunk's products done; DFREE: its
// accumulator read by the 8 state and 4 output warps; AISS: V^T [Z | R^T] issued)
constexpr int CB_FULL = 0, CB_DSFULL = 2, CB_DFREE = 4, CB_AISS = 6, CB_DRAIN = 8;
constexpr uint32_t kDfreeCount = 12;
static_assert(1 + NR <= kFlagWords, "flag words per chain CTA");
// local-CTA mbarriers (TMA: one per raw buffer)
constexpr int LB_TMA = 0, LB_L = 3, LB_OFFSET = 5, LB_DRAIN = 6, LB_X = 8;

// TMEM columns.  Chain: two accumulators D = [D_S | D_O] of 192 columns, and S
// as the bf16 A operand of S [Y^T | Qh^T] (two buffers of 64 columns, two values
// per column: S_{u+1} is written while chunk u's product may still read S_u).
// Local: per group 256 (D_kq; D_ab, and X over D_ab and the 64 columns after it:
// X of task k stays until task k + 2's inversion phase has converted it).
constexpr uint32_t TM_D = 0, TM_DSTRIDE = 192, TM_O = 128, TM_S = 384;
constexpr uint32_t TM_KQ = 0, TM_AB = 64, TM_X = 64, TM_GROUP = 256;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);    // [K;Q] K^T
constexpr uint32_t ID_N128 = idesc_bf16(128, 128, false, true);  // [P;0][T_bg|T_b], [X1;X2] K
constexpr uint32_t ID_X = idesc_bf16(128, 192, true, true);      // Kt^T [T_b | -W] (local)
constexpr uint32_t ID_VZR = idesc_bf16(128, 192, true, false);   // V^T [Z | R^T]
constexpr uint32_t ID_SYQ = idesc_bf16(128, 192, false, false);  // S [Y^T | Qh^T]

// named barriers
constexpr int BAR_UPD = 5;  // chain: the state warps (local: 1-2 groups, 3-4 inversion warps)
constexpr int BAR_OUT = 6;  // chain: the output warps

struct PoolArgs {
    uint8_t *ring;         // nch x NR slots of RING_STRIDE bytes
    uint64_t *flags;       // per chain CTA 8 words: cons, ready[NR], pad
    uint32_t *gabort;      // grid-wide abort word
    const long long *rbase;  // packed batches: task offset of each round [nrounds + 1]
    int nrounds;
    long long ntask;       // task count (fixed rows)
    int nch;               // chain CTAs
    int nck;               // chunks per chain (fixed rows)
};

// One chunk task: token range, head, its chain CTA and ring tag.
struct Task {
    long long t0;
    int L;      // tokens (0: an empty padding task)
    int h;
    int b;      // chain CTA
    int m;      // chunk index in its chain
    int rho;    // round
};

__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void st_release_cta_u32(uint32_t *p, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_cta_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t ready_tag(int rho, int m) {
    return ((uint64_t)(rho + 1) << 32) | (uint32_t)(m + 1);
}
// cons[b] after chunk m of round rho has been read out of its slot
__device__ __forceinline__ uint64_t cons_after(int rho, int m, int nck) {
    return m + 1 == nck ? ((uint64_t)(rho + 1) << 32) : (((uint64_t)rho << 32) | (uint32_t)(m + 1));
}
// cons[b] a local CTA needs before it writes chunk m of round rho into its slot
// (the slot's previous occupant, chunk m - NR or a chunk of an earlier round,
// has been read)
__device__ __forceinline__ uint64_t cons_needed(int rho, int m) {
    return ((uint64_t)rho << 32) | (uint32_t)(m >= NR ? m - NR + 1 : 0);
}

// Task t of the global order.  Chains are x = rho * nch + b (sequence x / H,
// head x % H); round rho holds the chains of its nch chain CTAs and lists their
// chunks chunk-major, every chain padded to the round's longest (padding tasks
// are empty).  Fixed rows: closed form.  Packed batches: the round offsets
// (rbase, written by the schedule kernel) are searched.
__device__ __forceinline__ Task task_of(const PrefillArgs &a, const PoolArgs &p, long long t) {
    Task k;
    const long long nchains = (long long)a.n_seqs * a.H;
    int rho;
    long long rem;
    if (p.rbase == nullptr) {
        const long long per_round = (long long)p.nch * p.nck;
        rho = (int)(t / per_round);
        rem = t - (long long)rho * per_round;
    } else {
        int lo = 0, hi = p.nrounds - 1;  // last round with rbase <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.rbase[mid] <= t) lo = mid; else hi = mid - 1;
        }
        rho = lo;
        rem = t - p.rbase[rho];
    }
    const int nround = (int)min((long long)p.nch, nchains - (long long)rho * p.nch);
    const int m = (int)(rem / nround), i = (int)(rem % nround);
    const long long x = (long long)rho * p.nch + i;
    const int n = (int)(x / a.H);
    long long tb, te;
    seq_range(a, n, &tb, &te);
    k.h = (int)(x % a.H);
    k.t0 = tb + (long long)m * C;
    const long long rest = te - k.t0;
    k.L = rest <= 0 ? 0 : (rest < C ? (int)rest : C);
    k.b = i;
    k.m = m;
    k.rho = rho;
    return k;
}

// log(1 + e^x) without overflow, and 1 / (1 + e^-x), in fp32
__device__ __forceinline__ float softplusf(float x) {
    return x > 0.f ? x + log1pf(expf(-x)) : log1pf(expf(x));
}
__device__ __forceinline__ float sigmoidf(float x) { return 1.f / (1.f + expf(-x)); }

__device__ __forceinline__ int4 pack_task(const Task &k) {
    return make_int4((int)k.t0, k.h | (k.L << 16), k.b | (k.rho << 8), k.m);
}
__device__ __forceinline__ Task unpack_task(int4 d) {
    Task k;
    k.t0 = (long long)(uint32_t)d.x;
    k.h = d.y & 0xffff;
    k.L = d.y >> 16;
    k.b = d.z & 0xff;
    k.rho = (int)((uint32_t)d.z >> 8);
    k.m = d.w;
    return k;
}

__device__ __forceinline__ uint4 pack8(const float *x) {
    uint4 u;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(x[0], x[1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(x[2], x[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(x[4], x[5]);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(x[6], x[7]);
    u.x = *reinterpret_cast<uint32_t *>(&h0);
    u.y = *reinterpret_cast<uint32_t *>(&h1);
    u.z = *reinterpret_cast<uint32_t *>(&h2);
    u.w = *reinterpret_cast<uint32_t *>(&h3);
    return u;
}
__device__ __forceinline__ void unpack8(uint4 u, float *x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&t);
}

// Decay of 32 entries (columns 32*half ..) of row r of a C x C product,
// e^{g_r - g_s} for s < r (strict) or s <= r.  rq = r / 32 is uniform per warp:
// the diagonal 32x32 block takes exact exponentials inside the row's own
// 16-block (g_r - g_s <= 0 wherever kept) and is factored across the 16-block
// boundary; a block strictly below it is factored at the 16-block boundary:
// e^{g_r - g_e} e^{g_e - g_s}, both factors <= 1.
__device__ __forceinline__ void decay_row(float *x, int r, int rq, int half, const float *gr,
                                          bool incl) {
    const float *g = gr + GR_G;
    if (rq == half) {
        const int rb = r >> 4;
        const float g_r = g[r];
        float d[16];
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
            const float4 gs = *reinterpret_cast<const float4 *>(g + 16 * rb + 4 * e4);
            d[4 * e4] = __expf(g_r - gs.x);
            d[4 * e4 + 1] = __expf(g_r - gs.y);
            d[4 * e4 + 2] = __expf(g_r - gs.z);
            d[4 * e4 + 3] = __expf(g_r - gs.w);
        }
        const bool upper = rb & 1;
        const float f0 = gr[GR_ROWF + 4 * r + 2 * half];
        const float *colf = gr + GR_COLF + 32 * half;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int s = 32 * half + j;
            const bool keep = incl ? (s <= r) : (s < r);
            const bool own = (j >> 4) == (upper ? 1 : 0);
            const float fac = own ? d[j & 15] : f0 * colf[j];
            x[j] = keep ? x[j] * fac : 0.f;
        }
    } else {
        const float *colf = gr + GR_COLF + 32 * half;
        const float f0 = gr[GR_ROWF + 4 * r + 2 * half], f1 = gr[GR_ROWF + 4 * r + 2 * half + 1];
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
            const float4 c = *reinterpret_cast<const float4 *>(colf + 4 * j4);
            const float f = j4 < 4 ? f0 : f1;
            const float2 lo = __fmul2_rn(make_float2(x[4 * j4], x[4 * j4 + 1]), make_float2(f * c.x, f * c.y));
            const float2 hi = __fmul2_rn(make_float2(x[4 * j4 + 2], x[4 * j4 + 3]), make_float2(f * c.z, f * c.w));
            x[4 * j4] = lo.x; x[4 * j4 + 1] = lo.y; x[4 * j4 + 2] = hi.x; x[4 * j4 + 3] = hi.y;
        }
    }
}

// Bounded waits.  `abort` is this CTA's flag, `gabort` the grid's: a wait on
// another CTA's progress gives up when either is raised or after `limit` cycles.
struct Waiter {
    volatile int *abort;
    volatile uint32_t *gabort;
    uint32_t *err;
    long long limit;
    __device__ __forceinline__ void raise() const {
        *abort = 1;
        atomicExch(const_cast<uint32_t *>(gabort), 1u);
        atomicOr(err, kErrTimeout);
    }
    // a phase completed inside this CTA (MMA commits, TMA, other warps)
    __device__ __forceinline__ bool wait(uint64_t *bar, uint32_t parity) const {
        if (mbar_try_wait(bar, parity)) return true;
        const long long t0 = clock64();
        while (!mbar_try_wait(bar, parity)) {
            if (*abort) return false;
            if (clock64() - t0 > limit) {
                raise();
                return false;
            }
        }
        return true;
    }
    // one lane waits, the warp gets the answer
    __device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int lane) const {
        bool ok = true;
        if (lane == 0) ok = wait(bar, parity);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    // a shared counter written by another warp of this CTA reaches `want`
    __device__ __forceinline__ bool wait_count(const uint32_t *c, uint32_t want) const {
        if (ld_acquire_cta_u32(c) >= want) return true;
        const long long t0 = clock64();
        while (ld_acquire_cta_u32(c) < want) {
            if (*abort) return false;
            if (clock64() - t0 > limit) {
                raise();
                return false;
            }
        }
        return true;
    }
    // a global word written by another CTA reaches `want` (== or >=)
    __device__ __forceinline__ bool wait_global(const uint64_t *p, uint64_t want, bool exact) const {
        uint64_t v = ld_acquire_u64(p);
        if (exact ? v == want : v >= want) return true;
        const long long t0 = clock64();
        for (;;) {
            __nanosleep(64);
            v = ld_acquire_u64(p);
            if (exact ? v == want : v >= want) return true;
            if (*abort || *gabort) {
                *abort = 1;
                return false;
            }
            if (clock64() - t0 > limit) {
                raise();
                return false;
            }
        }
    }
};

// RAW: q, k arrive unnormalised and the gates as logits (the fused input
// prologue: L2 norms folded into the row and column scales of the products,
// beta = sigmoid(b), log alpha = -softplus(a + bias)).
template <bool RAW>
__global__ void __launch_bounds__(kThreads, 1)
chunk_pool_kernel(const PrefillArgs a, const PoolArgs p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v2,
                  const __grid_constant__ CUtensorMap tm_o) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint8_t *cm = sm + OFF_COMMON;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(cm + CM_ABORT);
    uint64_t *bars = reinterpret_cast<uint64_t *>(cm + CM_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(cm + CM_TMEM);
    int *issued = reinterpret_cast<int *>(cm + CM_ISSUED);  // loads issued per buffer
    uint32_t *landed = reinterpret_cast<uint32_t *>(cm + CM_LANDED);  // chain: chunks landed

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool chain_role = (int)blockIdx.x < p.nch;
    const int H = a.H;

    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i) {
            uint32_t cnt = 1;
            if (chain_role && (i == CB_DFREE || i == CB_DFREE + 1)) cnt = kDfreeCount;
            mbar_init(bars + i, cnt);
        }
        fence_mbar_init();
        *abort_flag = 0;
        *landed = 0;
        for (int i = 0; i < 8; ++i) issued[i] = 0;
        if (chain_role) {
            tma_prefetch_desc(&tm_v2);
        } else {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter wt{abort_flag, p.gabort, a.err, data_wait_limit(a.err)};

    if (!chain_role) {
        // ============================ local CTA ============================
        const int c = (int)blockIdx.x - p.nch, nloc = (int)gridDim.x - p.nch;
        const long long ntask_all = p.rbase ? p.rbase[p.nrounds] : p.ntask;
        const int ntask = c < ntask_all ? (int)((ntask_all - c + nloc - 1) / nloc) : 0;
        auto gid = [&](int k) -> long long { return (long long)c + (long long)k * nloc; };
        // this CTA's first kDescCache task descriptors, decoded once by all threads
        // (the decode takes several 64-bit divisions, or a search of the rounds)
        int4 *sdesc = reinterpret_cast<int4 *>(sm + OFF_DESC);
        for (int k = tid; k < min(ntask, kDescCache); k += kThreads)
            sdesc[k] = pack_task(task_of(a, p, gid(k)));
        __syncthreads();
        auto task = [&](int k) -> Task {
            if (k < kDescCache) return unpack_task(sdesc[k]);
            return task_of(a, p, gid(k));
        };
        if (warp < 16) {
            const int g = warp >> 3, lw = warp & 7, lq = warp & 3, lhalf = lw >> 2;
            const int gtid = tid & 255;
            const int BAR_G = 1 + g, BAR_INV = 3 + g;
            uint8_t *grp = sm + L_G0 + g * L_GSZ;
            const uint32_t gbase = sbase + L_G0 + g * L_GSZ;
            auto raw_of = [&](int k) -> uint8_t * { return sm + (k % 3) * RAW_BYTES; };
            auto tma_phase = [&](int k) -> uint32_t { return (uint32_t)((k / 3) & 1); };
            uint8_t *pzt = grp + L_PZT;
            float *AT = reinterpret_cast<float *>(grp + L_AT);
            uint64_t *bar_l = bars + LB_L + g;
            // the X product completes on a barrier of its own: it and the next task's
            // first product are both in flight before either is waited for, and two
            // phases of one barrier completing before a wait would look like none
            uint64_t *bar_x = bars + LB_X + g;
            const uint32_t tm_kq = tmem + g * TM_GROUP + TM_KQ, tm_ab = tmem + g * TM_GROUP + TM_AB;
            const uint32_t tm_x = tmem + g * TM_GROUP + TM_X;
            // the group's task whose X product is issued but not yet converted (-1: none)
            int xk = -1;
            const uint32_t lane_off = (uint32_t)(32 * lq) << 16;
            const uint64_t d_pz = desc_sw128(gbase + L_PZT + PZ_P, 16, 1024);                // [P; X1]
            const uint64_t d_x1b = desc_sw128(gbase + L_PZT + PZ_X1, PZ_X3 - PZ_X1, 1024);  // X1 | X3
            const uint64_t d_x1x2 = desc_sw128(gbase + L_PZT + PZ_X1, 16, 1024);            // [X1; X2]
            uint32_t bl_wait = 0, bx_wait = 0;
            const bool issuer = gtid == 0;       // MMAs
            const bool storer = gtid == 7 * 32;  // tile loads, the slot wait and the hand-off
            // X of task kx -> Z^T (columns 0-63) and G^T = Y (64-191) of row n = 32 lq +
            // lane, bf16, to the task's ring slot (K-major, 128-byte swizzled), 64
            // columns (one 128-byte row segment) per pass: lw 4-7 take passes 0-1 while
            // lw 0-3 invert, lw 0-3 pass 2 after.  Each 8-lane group transposes its 8
            // rows x 8 16-byte chunks with three xor-shuffle stages, so that every store
            // instruction writes whole 128-byte rows.  The storer hands the task over
            // (publish_x) two barriers later, once the stores have drained.
            auto convert_x = [&](int kx, int p0, int p1) {
                const Task tx = task(kx);
                uint8_t *xs = p.ring + ((size_t)tx.b * NR + (tx.m % NR)) * RING_STRIDE;
                const int j8 = lane & 7;
                const int n0 = 32 * lq + (lane & ~7);
                tc_fence_after();
#pragma unroll 1
                for (int pass = p0; pass < p1; ++pass) {
                    uint32_t w[32];
#pragma unroll
                    for (int hq = 0; hq < 2; ++hq) {
                        float x[32];
                        tmem_ld16(tm_x + lane_off + 64 * pass + 32 * hq, x);
                        tmem_ld16(tm_x + lane_off + 64 * pass + 32 * hq + 16, x + 16);
                        tmem_wait_ld16(x);
                        reg_fence16(x + 16);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint4 v = pack8(x + 8 * c);
                            w[16 * hq + 4 * c] = v.x; w[16 * hq + 4 * c + 1] = v.y;
                            w[16 * hq + 4 * c + 2] = v.z; w[16 * hq + 4 * c + 3] = v.w;
                        }
                    }
                    // w[4c..] = chunk c of row n0 + j8  ->  w[4t..] = chunk j8 of row n0 + t
#pragma unroll
                    for (int bb = 1; bb < 8; bb <<= 1) {
                        const bool hi = (lane & bb) != 0;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            if (c & bb) continue;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const uint32_t send = hi ? w[4 * c + e] : w[4 * (c | bb) + e];
                                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, bb);
                                if (hi) w[4 * c + e] = recv;
                                else w[4 * (c | bb) + e] = recv;
                            }
                        }
                    }
                    uint8_t *dst = xs + (pass == 0 ? RG_ZT : RG_YQ + (pass - 1) * YQ_HALF);
#pragma unroll
                    for (int t = 0; t < 8; ++t)
                        *reinterpret_cast<uint4 *>(dst + (n0 + t) * 128 + ((j8 ^ t) << 4)) =
                            make_uint4(w[4 * t], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
                }
                tc_fence_before();
            };
            // (storer) task kx's tiles are all in its slot: the group barriers since its
            // stores order them before this release
            auto publish_x = [&](int kx) {
                const Task tx = task(kx);
                st_release_u64(p.flags + (size_t)tx.b * kFlagWords + 1 + (tx.m % NR), ready_tag(tx.rho, tx.m));
            };
            auto convert_part = [&](int kx) { convert_x(kx, lw >= 4 ? 0 : 2, lw >= 4 ? 2 : 3); };
            // raw tiles of task k into buffer k % 3 (an empty task completes the
            // buffer's phase with a plain arrive)
            auto issue_tma = [&](int k) {
                const Task tk = task(k);
                uint8_t *dst = raw_of(k);
                uint64_t *bt = bars + LB_TMA + (k % 3);
                if (tk.L == 0) {
                    mbar_arrive(bt);
                } else {
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(bt, 4 * 8192);
                    tma_load_3d(dst + 0, &tm_k, 0, tk.h, (int)tk.t0, bt);
                    tma_load_3d(dst + 8192, &tm_q, 0, tk.h, (int)tk.t0, bt);
                    tma_load_3d(dst + L_RAW_AC, &tm_k, 64, tk.h, (int)tk.t0, bt);
                    tma_load_3d(dst + L_RAW_AC + 8192, &tm_q, 64, tk.h, (int)tk.t0, bt);
                }
                atomicAdd(issued + (k % 3), 1);
            };
            auto gate_rows = [&](int k) {
                return reinterpret_cast<float *>(grp + L_GATES + ((k >> 1) & 1) * GATES_STRIDE);
            };
            // gates of the group's task after next, prefetched in warp lw 4's registers
            float nla0 = 0.f, nla1 = 0.f, nbe0 = 0.f, nbe1 = 0.f;
            auto load_gates = [&](int k) {
                const Task tk = task(k);
                const int r0 = 2 * lane, r1 = 2 * lane + 1;
                nla0 = r0 < tk.L ? a.log_alpha[(tk.t0 + r0) * H + tk.h] : 0.f;
                nla1 = r1 < tk.L ? a.log_alpha[(tk.t0 + r1) * H + tk.h] : 0.f;
                nbe0 = r0 < tk.L ? a.beta[(tk.t0 + r0) * H + tk.h] : 0.f;
                nbe1 = r1 < tk.L ? a.beta[(tk.t0 + r1) * H + tk.h] : 0.f;
                if constexpr (RAW) {
                    // logits -> gates; rows past the sequence end stay (0, 0)
                    const float bias = a.alpha_bias ? a.alpha_bias[tk.h] : 0.f;
                    nla0 = r0 < tk.L ? -softplusf(nla0 + bias) : 0.f;
                    nla1 = r1 < tk.L ? -softplusf(nla1 + bias) : 0.f;
                    nbe0 = r0 < tk.L ? sigmoidf(nbe0) : 0.f;
                    nbe1 = r1 < tk.L ? sigmoidf(nbe1) : 0.f;
                }
            };
            // gate rows of task kk (one warp): cumulative log decay, beta, the
            // factored block decays, kh and gamma, e^{g_C} for every channel
            auto compute_gates = [&](int kk) {
                float *gr = gate_rows(kk);
                const int r0 = 2 * lane, r1 = 2 * lane + 1;
                const float la0 = nla0, la1 = nla1, be0 = nbe0, be1 = nbe1;
                if (kk + 2 < ntask) load_gates(kk + 2);
                float incl = la0 + la1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                const float g1 = incl, g0 = incl - la1;
                float gend[4];
#pragma unroll
                for (int b = 0; b < 4; ++b) gend[b] = __shfl_sync(0xffffffffu, incl, 8 * b + 7);
                const float gC = gend[3];
                const int blk = r0 >> 4;
                const float e0 = __expf(g0), e1 = __expf(g1);
                const float c0 = __expf(gend[blk] - g0), c1 = __expf(gend[blk] - g1);
                const float k0 = __expf(gC - g0), k1 = __expf(gC - g1);
                float f0[3], f1[3];
#pragma unroll
                for (int b = 0; b < 3; ++b) {
                    f0[b] = __expf(fminf(g0 - gend[b], 0.f));
                    f1[b] = __expf(fminf(g1 - gend[b], 0.f));
                }
                gr[GR_G + r0] = g0; gr[GR_G + r1] = g1;
                gr[GR_B + r0] = be0; gr[GR_B + r1] = be1;
                gr[GR_BG + r0] = be0 * e0; gr[GR_BG + r1] = be1 * e1;
                gr[GR_COLF + r0] = c0; gr[GR_COLF + r1] = c1;
                gr[GR_KH + r0] = k0; gr[GR_KH + r1] = k1;
                gr[GR_GAM + r0] = e0; gr[GR_GAM + r1] = e1;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    gr[GR_ROWF + 4 * r0 + b] = b < blk ? f0[b < 3 ? b : 0] : 0.f;
                    gr[GR_ROWF + 4 * r1 + b] = b < blk ? f1[b < 3 ? b : 0] : 0.f;
                }
                const float dC = __expf(gC);
                *reinterpret_cast<float4 *>(gr + GR_DEC + 4 * lane) = make_float4(dC, dC, dC, dC);
            };

            // the first tasks' tiles (one per raw buffer) and the group's first gates
            if (storer && g < ntask) issue_tma(g);
            if (storer && g == 0 && 2 < ntask) issue_tma(2);
            if (lw == 4 && g < ntask) {
                load_gates(g);
                compute_gates(g);
            }
            // group 1 starts half a task after group 0, so that the two groups'
            // CUDA-core phases tend to overlap the other's MMA and load waits
            bool ok0 = true;
            if (g == 1 && issuer && ntask >= 2) ok0 = wt.wait(bars + LB_OFFSET, 0);
            named_bar_or(BAR_G, 256, !ok0);

            for (int k = g; k < ntask; k += 2) {
                const Task tk = task(k);
                // this task's ring slot (chain CTA tk.b, slot tk.m % NR): every thread
                // writes its part of the tiles there with plain 16-byte stores
                uint8_t *slot = p.ring + ((size_t)tk.b * NR + (tk.m % NR)) * RING_STRIDE;
                uint64_t *fl = p.flags + (size_t)tk.b * kFlagWords;
                float *gr = gate_rows(k);
                uint8_t *rawp = raw_of(k);
                const uint32_t raw_s = smem_u32(rawp);
                const uint64_t d_raw = desc_sw128(raw_s, 16, 1024);        // [K;Q], K (K-major)
                const uint64_t d_kmn = desc_sw128(raw_s, L_RAW_AC, 1024);  // K (MN-major)
                const int L = tk.L;
                bool ok = true;
                // the next-but-two task's tiles into L2 while this one runs
                if (issuer && k + 3 < ntask) {
                    const Task t3 = task(k + 3);
                    if (t3.L > 0) {
                        tma_prefetch_l2_3d(&tm_k, 0, t3.h, (int)t3.t0);
                        tma_prefetch_l2_3d(&tm_k, 64, t3.h, (int)t3.t0);
                        tma_prefetch_l2_3d(&tm_q, 0, t3.h, (int)t3.t0);
                        tma_prefetch_l2_3d(&tm_q, 64, t3.h, (int)t3.t0);
                    }
                }
                if (issuer) ok = wt.wait(bars + LB_TMA + (k % 3), tma_phase(k));
                if (L == 0) {
                    // empty padding task: only the duties other tasks rely on
                    if (issuer && ok && xk >= 0) ok = wt.wait(bar_x, bx_wait & 1);
                    if (xk >= 0) ++bx_wait;
                    if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                    if (xk >= 0) convert_part(xk);
                    if (storer && k >= 2 && k + 1 < ntask) issue_tma(k + 1);
                    if (lw == 4 && k + 2 < ntask) compute_gates(k + 2);
                    if (g == 0 && k == 0 && issuer) mbar_arrive(bars + LB_OFFSET);
                    named_bar_sync(BAR_G, 256);
                    if (storer && xk >= 0) publish_x(xk);
                    xk = -1;
                    continue;
                }
                if (L < C) {
                    if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                    for (int idx = gtid; idx < (C - L) * 8; idx += 256) {
                        const uint32_t o = (L + (idx >> 3)) * 128 + (idx & 7) * 16;
                        const uint4 z = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(rawp + o) = z;
                        *reinterpret_cast<uint4 *>(rawp + 8192 + o) = z;
                        *reinterpret_cast<uint4 *>(rawp + L_RAW_AC + o) = z;
                        *reinterpret_cast<uint4 *>(rawp + L_RAW_AC + 8192 + o) = z;
                    }
                    fence_proxy_async_smem();
                    if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                }
                // raw inputs: every thread reads the tiles for the norms below
                if (RAW && L == C) {
                    if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                }
                // ---- D_kq = [K; Q] K^T (a full task's MMA goes out as soon as its
                //      tiles are in; an abort is seen at the barrier after it) -------
                if (issuer && ok) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * L_RAW_AC + (kk & 3) * 32) >> 4;
                        mma_bf16(tm_kq, d_raw + off, d_raw + off, ID_KK, kk > 0);
                    }
                    mma_commit(bar_l);
                }
                // (this group's previous task's X product completes first, then D_kq)
                if (!RAW && issuer && ok && xk >= 0) ok = wt.wait(bar_x, bx_wait & 1);
                if (!RAW && xk >= 0) ++bx_wait;
                if (!RAW && issuer && ok) ok = wt.wait(bar_l, bl_wait & 1);
                if constexpr (RAW) {
                    // 1 / ||k_r||, 1 / ||q_r|| of the raw bf16 rows (norm clamped at
                    // 1e-12) while the product runs: thread pair per (tile, row)
                    const int tsel = gtid >> 7, r = (gtid & 127) >> 1, at = gtid & 1;
                    const uint8_t *rowp = rawp + at * L_RAW_AC + tsel * 8192;
                    float ss = 0.f;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        float v8[8];
                        unpack8(*reinterpret_cast<const uint4 *>(rowp + sw128(r, cc)), v8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) ss = fmaf(v8[e], v8[e], ss);
                    }
                    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                    if (at == 0) gr[(tsel ? GR_INVQ : GR_INVK) + r] = rsqrtf(fmaxf(ss, 1e-24f));
                    if (issuer && ok && xk >= 0) ok = wt.wait(bar_x, bx_wait & 1);
                    if (xk >= 0) ++bx_wait;
                    if (issuer && ok) ok = wt.wait(bar_l, bl_wait & 1);
                }
                ++bl_wait;
                if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                // the raw buffer of this group's previous task (k - 2, an operand of its
                // X product, complete now) takes task k + 1, the other group's next
                if (storer && k >= 2 && k + 1 < ntask) issue_tma(k + 1);
                tc_fence_after();
                // ---- A rows (lanes 0-63) -> fp32 with beta; P rows (lanes 64-127) -> bf16
                const float *gb = gr + GR_B;
                if ((lq & 1) >= lhalf) {
                    float x[32];
                    tmem_load<32>(tm_kq + lane_off + 32 * lhalf, x);
                    if constexpr (RAW) {
                        // normalised rows and columns: x_rs / (||row_r|| ||k_s||)
                        const int r = 32 * (lq & 1) + lane;
                        const float rsc = gr[(lq < 2 ? GR_INVK : GR_INVQ) + r];
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 cs = *reinterpret_cast<const float4 *>(gr + GR_INVK + 32 * lhalf + j);
                            x[j] *= rsc * cs.x; x[j + 1] *= rsc * cs.y;
                            x[j + 2] *= rsc * cs.z; x[j + 3] *= rsc * cs.w;
                        }
                    }
                    if (lq < 2) {
                        const int r = 32 * lq + lane;
                        decay_row(x, r, lq, lhalf, gr, false);
                        const float br = gb[r];
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            *reinterpret_cast<float4 *>(AT + r * LDA + 32 * lhalf + j) =
                                make_float4(br * x[j], br * x[j + 1], br * x[j + 2], br * x[j + 3]);
                        }
                    } else {
                        const int r = 32 * (lq - 2) + lane;
                        decay_row(x, r, lq - 2, lhalf, gr, true);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(pzt + PZ_P + sw128(r, 4 * lhalf + j)) = pack8(x + 8 * j);
                    }
                } else if (lq >= 2) {
                    // P rows 0-31, columns 32-63 (above the diagonal): zero
#pragma unroll
                    for (int j = 4; j < 8; ++j)
                        *reinterpret_cast<uint4 *>(pzt + PZ_P + sw128(lane, j)) = make_uint4(0, 0, 0, 0);
                }
                named_bar_sync(BAR_G, 256);
                if (g == 0 && k == 0 && issuer) mbar_arrive(bars + LB_OFFSET);
                // ---- T = (I + A)^{-1} in place of A: lw 0-3; meanwhile lw 4 prepares
                //      the group's next gates and the storer hands over its last task
                // (the X product converted here is handed over below, before this task's
                // slot wait)
                const int xpub = xk;
                if (lw >= 4) {
                    // the group's previous task's X product -> its ring slot
                    if (xk >= 0) convert_part(xk);
                    if (lw == 4 && k + 2 < ntask) compute_gates(k + 2);
                } else {
                    // (1) 16x16 diagonal blocks, right-looking forward substitution;
                    //     lane j < 16 owns column j
                    if (lane < 16) {
                        const int o = 16 * lw, j = lane;
                        float t[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) t[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
                        for (int mm = 0; mm < 15; ++mm) {
#pragma unroll
                            for (int i = mm + 1; i < 16; ++i) t[i] -= AT[(o + i) * LDA + o + mm] * t[mm];
                        }
                        __syncwarp(0x0000ffffu);
#pragma unroll
                        for (int i = 0; i < 16; ++i) AT[(o + i) * LDA + o + j] = t[i];
                    }
                    named_bar_sync(BAR_INV, 128);
                    // (2) 32x32 halves: T_10 = -T_11 (A_10 T_00), T_32 = -T_33 (A_32 T_22)
                    const int fg = lane >> 2, ft = lane & 3;
                    const int o = 32 * (lw >> 1), n0 = 8 * (lw & 1);
                    float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        uint32_t af[4], bf[2];
                        const int ar = o + 16 + fg, ac = o + 8 * ks + ft;
                        af[0] = to_tf32(AT[ar * LDA + ac]);
                        af[1] = to_tf32(AT[(ar + 8) * LDA + ac]);
                        af[2] = to_tf32(AT[ar * LDA + ac + 4]);
                        af[3] = to_tf32(AT[(ar + 8) * LDA + ac + 4]);
                        bf[0] = to_tf32(AT[(o + 8 * ks + ft) * LDA + o + n0 + fg]);
                        bf[1] = to_tf32(AT[(o + 8 * ks + ft + 4) * LDA + o + n0 + fg]);
                        mma_tf32_16x8x8(x, af, bf);
                    }
                    AT[(o + fg) * LDA + o + 16 + n0 + 2 * ft] = x[0];
                    AT[(o + fg) * LDA + o + 16 + n0 + 2 * ft + 1] = x[1];
                    AT[(o + fg + 8) * LDA + o + 16 + n0 + 2 * ft] = x[2];
                    AT[(o + fg + 8) * LDA + o + 16 + n0 + 2 * ft + 1] = x[3];
                    named_bar_sync(BAR_INV, 128);
                    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        uint32_t af[4], bf[2];
                        const int ar = o + 16 + fg, ac = o + 16 + 8 * ks + ft;
                        af[0] = to_tf32(AT[ar * LDA + ac]);
                        af[1] = to_tf32(AT[(ar + 8) * LDA + ac]);
                        af[2] = to_tf32(AT[ar * LDA + ac + 4]);
                        af[3] = to_tf32(AT[(ar + 8) * LDA + ac + 4]);
                        bf[0] = to_tf32(AT[(o + 8 * ks + ft) * LDA + o + 16 + n0 + fg]);
                        bf[1] = to_tf32(AT[(o + 8 * ks + ft + 4) * LDA + o + 16 + n0 + fg]);
                        mma_tf32_16x8x8(y, af, bf);
                    }
                    AT[(o + 16 + fg) * LDA + o + n0 + 2 * ft] = -y[0];
                    AT[(o + 16 + fg) * LDA + o + n0 + 2 * ft + 1] = -y[1];
                    AT[(o + 24 + fg) * LDA + o + n0 + 2 * ft] = -y[2];
                    AT[(o + 24 + fg) * LDA + o + n0 + 2 * ft + 1] = -y[3];
                    if (xk >= 0) convert_part(xk);
                }
                xk = -1;
                if (named_bar_or(BAR_G, 256, *abort_flag)) break;
                // (3) T_{H1,H0} = -T_{H1} (A_{H1,H0} T_{H0}), 32x32 blocks; warp lw owns
                //     output rows 16(lw/4).., columns 8(lw%4)..
                {
                    const int fg = lane >> 2, ft = lane & 3;
                    const int m0 = 16 * (lw >> 2), n0 = 8 * (lw & 3);
                    float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        uint32_t af[4], bf[2];
                        const int ar = 32 + m0 + fg, ac = 8 * ks + ft;
                        af[0] = to_tf32(AT[ar * LDA + ac]);
                        af[1] = to_tf32(AT[(ar + 8) * LDA + ac]);
                        af[2] = to_tf32(AT[ar * LDA + ac + 4]);
                        af[3] = to_tf32(AT[(ar + 8) * LDA + ac + 4]);
                        const int br = 8 * ks + ft, bc = n0 + fg;
                        bf[0] = to_tf32(br >= bc ? AT[br * LDA + bc] : 0.f);
                        bf[1] = to_tf32(br + 4 >= bc ? AT[(br + 4) * LDA + bc] : 0.f);
                        mma_tf32_16x8x8(x, af, bf);
                    }
                    AT[(m0 + fg) * LDA + 32 + n0 + 2 * ft] = x[0];
                    AT[(m0 + fg) * LDA + 32 + n0 + 2 * ft + 1] = x[1];
                    AT[(m0 + fg + 8) * LDA + 32 + n0 + 2 * ft] = x[2];
                    AT[(m0 + fg + 8) * LDA + 32 + n0 + 2 * ft + 1] = x[3];
                    named_bar_sync(BAR_G, 256);
                    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        uint32_t af[4], bf[2];
                        const int r = m0 + fg, kc = 8 * ks + ft;
                        af[0] = to_tf32(kc <= r ? AT[(32 + r) * LDA + 32 + kc] : 0.f);
                        af[1] = to_tf32(kc <= r + 8 ? AT[(40 + r) * LDA + 32 + kc] : 0.f);
                        af[2] = to_tf32(kc + 4 <= r ? AT[(32 + r) * LDA + 36 + kc] : 0.f);
                        af[3] = to_tf32(kc + 4 <= r + 8 ? AT[(40 + r) * LDA + 36 + kc] : 0.f);
                        bf[0] = to_tf32(AT[(8 * ks + ft) * LDA + 32 + n0 + fg]);
                        bf[1] = to_tf32(AT[(8 * ks + ft + 4) * LDA + 32 + n0 + fg]);
                        mma_tf32_16x8x8(y, af, bf);
                    }
                    AT[(32 + m0 + fg) * LDA + n0 + 2 * ft] = -y[0];
                    AT[(32 + m0 + fg) * LDA + n0 + 2 * ft + 1] = -y[1];
                    AT[(40 + m0 + fg) * LDA + n0 + 2 * ft] = -y[2];
                    AT[(40 + m0 + fg) * LDA + n0 + 2 * ft + 1] = -y[3];
                }
                named_bar_sync(BAR_G, 256);
                // ---- T_b and T_bg in bf16, rows r, columns s (consecutive threads on
                //      consecutive rows: no bank conflict on T's rows, beta broadcast)
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    const int idx = gtid + 256 * q2, r = idx & 63, j = idx >> 6;
                    float tv[8], bv[8], tb[8], gv[8], tg[8];
                    *reinterpret_cast<float4 *>(tv) = *reinterpret_cast<const float4 *>(AT + r * LDA + 8 * j);
                    *reinterpret_cast<float4 *>(tv + 4) = *reinterpret_cast<const float4 *>(AT + r * LDA + 8 * j + 4);
                    *reinterpret_cast<float4 *>(bv) = *reinterpret_cast<const float4 *>(gb + 8 * j);
                    *reinterpret_cast<float4 *>(bv + 4) = *reinterpret_cast<const float4 *>(gb + 8 * j + 4);
                    *reinterpret_cast<float4 *>(gv) = *reinterpret_cast<const float4 *>(gr + GR_BG + 8 * j);
                    *reinterpret_cast<float4 *>(gv + 4) = *reinterpret_cast<const float4 *>(gr + GR_BG + 8 * j + 4);
                    if constexpr (RAW) {  // W = T_b diag(gamma) K_n = T_b diag(gamma / ||k||) K
                        const float4 i0 = *reinterpret_cast<const float4 *>(gr + GR_INVK + 8 * j);
                        const float4 i1 = *reinterpret_cast<const float4 *>(gr + GR_INVK + 8 * j + 4);
                        gv[0] *= i0.x; gv[1] *= i0.y; gv[2] *= i0.z; gv[3] *= i0.w;
                        gv[4] *= i1.x; gv[5] *= i1.y; gv[6] *= i1.z; gv[7] *= i1.w;
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s2 = 8 * j + e;
                        tv[e] = s2 < r ? tv[e] : (s2 == r ? 1.f : 0.f);
                        tb[e] = tv[e] * bv[e];
                        tg[e] = tv[e] * gv[e];
                    }
                    *reinterpret_cast<uint4 *>(pzt + PZ_X3 + sw128(r, j)) = pack8(tb);
                    *reinterpret_cast<uint4 *>(pzt + PZ_X1 + sw128(r, j)) = pack8(tg);
                }
                fence_proxy_async_smem();
                named_bar_sync(BAR_G, 256);
                // the previous task handed over; then this task's slot: its previous chunk
                // must have been read by chain CTA b before R goes out (below)
                if (storer) {
                    if (xpub >= 0) publish_x(xpub);
                    const uint64_t need = cons_needed(tk.rho, tk.m);
                    if (need != 0) ok = wt.wait_global(fl, need, false);
                }
                // ---- D_ab = [P; 0] [T_bg | T_b]: rows 0-63 = [P T_bg | R] ----------
                if (issuer) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_bf16(tm_ab, d_pz + 2 * kk, d_x1b + 128 * kk, ID_N128, kk > 0);
                    mma_commit(bar_l);
                    ok = wt.wait(bar_l, bl_wait & 1);
                }
                ++bl_wait;
                if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                tc_fence_after();
                // lw 0,1: P T_bg -> X2;  lw 4,5: R -> the ring slot
                if (lq < 2) {
                    const int r = 32 * lq + lane;
                    uint8_t *dst = lhalf == 0 ? pzt + PZ_X2 : slot + RG_R;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float x[32];
                        tmem_load<32>(tm_ab + lane_off + 64 * lhalf + 32 * hh, x);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(dst + sw128(r, 4 * hh + j)) = pack8(x + 8 * j);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(BAR_G, 256);
                // ---- D_ab = [T_bg; P T_bg] K: rows 0-63 = W, rows 64-127 = P W -------
                if (issuer) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_bf16(tm_ab, d_x1x2 + 2 * kk, d_kmn + 128 * kk, ID_N128, kk > 0);
                    mma_commit(bar_l);
                    ok = wt.wait(bar_l, bl_wait & 1);
                }
                ++bl_wait;
                if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                tc_fence_after();
                // ---- -W (lanes 0-63) into A/T's space and Kt = kh . K in place of K: the
                //      operands of X below; Qh = gamma Q - P W (lanes 64-127) and e^{g_C}
                //      straight to the ring slot
                {
                    const int r = 32 * (lq & 1) + lane;
                    const float gam = gr[GR_GAM + r] * (RAW ? gr[GR_INVQ + r] : 1.f);
                    uint8_t *wst = grp + L_AT + lhalf * 8192;
                    uint8_t *qst = slot + RG_YQ + lhalf * YQ_HALF + YQ_QH;
                    const uint8_t *qt = rawp + lhalf * L_RAW_AC + 8192;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float x[32];
                        tmem_load<32>(tm_ab + lane_off + 64 * lhalf + 32 * hh, x);
                        if (lq < 2) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                float w[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) w[e] = -x[8 * j + e];
                                *reinterpret_cast<uint4 *>(wst + sw128(r, 4 * hh + j)) = pack8(w);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint32_t o = sw128(r, 4 * hh + j);
                                float qv[8];
                                unpack8(*reinterpret_cast<const uint4 *>(qt + o), qv);
#pragma unroll
                                for (int e = 0; e < 8; ++e) qv[e] = gam * qv[e] - x[8 * j + e];
                                *reinterpret_cast<uint4 *>(qst + o) = pack8(qv);
                            }
                        }
                    }
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const int idx = gtid + 256 * q2;
                        const int ac = idx >> 9, rr = (idx >> 3) & 63, j = idx & 7;
                        float kv[8];
                        unpack8(*reinterpret_cast<const uint4 *>(rawp + ac * L_RAW_AC + sw128(rr, j)), kv);
                        const float sc = gr[GR_KH + rr] * (RAW ? gr[GR_INVK + rr] : 1.f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) kv[e] *= sc;
                        *reinterpret_cast<uint4 *>(rawp + ac * L_RAW_AC + sw128(rr, j)) = pack8(kv);
                    }
                    if (lw == 5)
                        *reinterpret_cast<uint4 *>(slot + RG_DEC + 16 * lane) =
                            *reinterpret_cast<const uint4 *>(gr + GR_DEC + 4 * lane);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                if (named_bar_or(BAR_G, 256, *abort_flag)) break;
                // ---- X = Kt^T [T_b | -W] (M = d_k, N = 64 + 128) over D_ab and the 64
                //      columns after it: row n holds Z^T (columns 0-63, Z = T_b^T Kt) and
                //      G^T (64-191, G = -W^T Kt), the chain CTA's operands of V^T Z and
                //      S G.  Issued here, converted during the group's next task --------
                if (issuer) {
                    tc_fence_after();
                    const uint64_t d_tw = desc_sw128(gbase + L_PZT + PZ_X3, 8192, 1024);
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_bf16(tm_x, d_kmn + 128 * kk, d_tw + 128 * kk, ID_X, kk > 0);
                    mma_commit(bar_x);
                }
                xk = k;
            }
            // the last task's X product
            if (xk >= 0 && !*abort_flag) {
                bool ok = true;
                if (issuer) ok = wt.wait(bar_x, bx_wait & 1);
                ++bx_wait;
                if (!named_bar_or(BAR_G, 256, !ok || *abort_flag)) {
                    convert_part(xk);
                    if (!named_bar_or(BAR_G, 256, *abort_flag) && storer) publish_x(xk);
                }
            }
            // drain: every MMA this group issued
            if (*abort_flag && issuer) {
                mma_commit(bars + LB_DRAIN + g);
                mbar_wait(bars + LB_DRAIN + g, 0, kWaitLimit);
            }
        }
    } else {
        // ============================ chain CTA ============================
        const int b = (int)blockIdx.x;
        const long long nchains = (long long)a.n_seqs * H;
        // chain (round) rho of this CTA: sequence, head, token range, chunks
        struct Chain {
            int n, h, nck;
            long long t_begin, t_end;
        };
        auto chain_of = [&](int rho, Chain *ch) -> bool {
            const long long x = (long long)rho * p.nch + b;
            if (x >= nchains) return false;
            ch->n = (int)(x / H);
            ch->h = (int)(x % H);
            seq_range(a, ch->n, &ch->t_begin, &ch->t_end);
            ch->nck = (int)((ch->t_end - ch->t_begin + C - 1) / C);
            return true;
        };
        const uint32_t lane_q = (uint32_t)(32 * (warp & 3)) << 16;
        auto stage_of = [&](uint32_t u) -> uint8_t * { return sm + (u & 1) * CS_BYTES; };
        if (warp < 8) {
            // ---- state warps: row j = 32 (warp % 4) + lane, key columns 64 ch .. ------
            //      S lives in fp32 registers and, as the bf16 A operand of
            //      S [Y^T | Qh^T], in tensor memory (this thread: packed columns 32 ch ..)
            const int ch = warp >> 2, j = 32 * (warp & 3) + lane;
            const bool leader = tid == 0;  // issues S [Y^T | Qh^T]
            float s_reg[64];
            auto load_s0 = [&](const Chain &cc) {
                const size_t base = (((size_t)cc.n * H + cc.h) * DV + j) * DK + 64 * ch;
#pragma unroll
                for (int e = 0; e < 64; e += 4) {
                    const float4 v = a.s0 ? *reinterpret_cast<const float4 *>(a.s0 + base + e)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                    s_reg[e] = v.x; s_reg[e + 1] = v.y; s_reg[e + 2] = v.z; s_reg[e + 3] = v.w;
                }
            };
            auto store_sf = [&](const Chain &cc) {
                if (!a.s_final) return;
                const size_t base = (((size_t)cc.n * H + cc.h) * DV + j) * DK + 64 * ch;
#pragma unroll
                for (int e = 0; e < 64; e += 4)
                    *reinterpret_cast<float4 *>(a.s_final + base + e) =
                        make_float4(s_reg[e], s_reg[e + 1], s_reg[e + 2], s_reg[e + 3]);
            };
            auto write_s_tmem = [&](uint32_t buf) {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack2(s_reg[2 * e], s_reg[2 * e + 1]);
                tmem_st32(tmem + TM_S + 64 * buf + 32 * ch + lane_q, pk);
                tmem_wait_st();
            };
            // e^{g_C} of chunk u (scalar decay: every entry of the slot's row is the
            // same), read once the stage has landed
            auto read_dec = [&](uint32_t u, float *dC) -> bool {
                if (!wt.warp_wait(bars + CB_FULL + (u & 1), (u >> 1) & 1, lane)) return false;
                *dC = *reinterpret_cast<const volatile float *>(stage_of(u) + RG_DEC);
                return true;
            };
            // the next chain with tokens, from round rho on: empty chains get their
            // final state (the initial one) here; returns false past the last chain
            auto open_chain = [&](int *rho, Chain *cc) -> bool {
                for (;; ++*rho) {
                    if (!chain_of(*rho, cc)) return false;
                    load_s0(*cc);
                    if (cc->nck > 0) return true;
                    store_sf(*cc);
                }
            };
            int rho = 0;
            Chain cur;
            bool have = open_chain(&rho, &cur);
            uint32_t u = 0;  // chunk counter over this CTA's chains
            float dC = 0.f;
            bool okr = true;
            if (have) {
                write_s_tmem(0);
                okr = read_dec(0, &dC);
            }
            tc_fence_before();
            const bool bad0 = named_bar_or(BAR_UPD, 256, !okr);
            int m = 0;
            while (have && !bad0) {
                const int s = u & 1;
                bool ok = true;
                if (leader) {
                    // D[s] += S_u [Y^T | Qh^T] (after D[s] = V^T [Z | R^T] went out)
                    ok = wt.wait(bars + CB_AISS + s, (u >> 1) & 1);
                    if (ok) {
                        tc_fence_after();
                        const uint64_t d_yq = desc_sw128(smem_u32(stage_of(u) + RG_YQ), 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk) {
                            const uint32_t off = ((kk >> 2) * YQ_HALF + (kk & 3) * 32) >> 4;
                            mma_bf16_ts(tmem + TM_D + TM_DSTRIDE * s, tmem + TM_S + 64 * s + 8 * kk,
                                        d_yq + off, ID_SYQ, 1);
                        }
                        mma_commit(bars + CB_DSFULL + s);
                    }
                }
                // S <- e^{g_C} S + D_S (columns of this thread's half)
                bool okd = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 &&
                           wt.warp_wait(bars + CB_DSFULL + s, (u >> 1) & 1, lane);
                if (okd) {
                    tc_fence_after();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float ds[16];
                        tmem_ld16(tmem + TM_D + TM_DSTRIDE * s + 64 * ch + 16 * q4 + lane_q, ds);
                        tmem_wait_ld16(ds);
#pragma unroll
                        for (int e = 0; e < 16; ++e) s_reg[16 * q4 + e] = fmaf(dC, s_reg[16 * q4 + e], ds[e]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars + CB_DFREE + s);
                    // S_{u+1} into S buffer (u + 1) & 1: its last reader, chunk u - 1's
                    // product, is done (this warp waited for it before chunk u - 1's update)
                    if (m + 1 == cur.nck) {
                        store_sf(cur);
                        ++rho;
                        have = open_chain(&rho, &cur);
                        m = 0;
                    } else {
                        ++m;
                    }
                    if (have) {
                        write_s_tmem((u + 1) & 1);
                        // the next chunk's decay, read before the barrier below: the
                        // stage is reloaded only after the next chunk's product, which
                        // the leader issues after it
                        okd = read_dec(u + 1, &dC);
                    }
                }
                tc_fence_before();
                if (named_bar_or(BAR_UPD, 256, !okd || *abort_flag)) break;
                ++u;
            }
            if (*abort_flag && leader) {
                mma_commit(bars + CB_DRAIN);
                mbar_wait(bars + CB_DRAIN, 0, kWaitLimit);
            }
        } else if (warp < 12) {
            // ---- lane 0 of warp 8: D[s] = V^T [Z | R^T] for each chunk once its
            //      stage has landed and chunk u - 2's accumulator has been read, and
            //      the loader: chunk u + 1 goes into stage (u + 1) & 1 once chunk
            //      u - 1's products are done.  Lane 0 of warp 9 gives each ring slot
            //      back (cons) once its chunk has landed: a gpu-scope release takes
            //      about a thousand cycles, which the loader's loop cannot carry.
            if (warp == 9 && lane == 0) {
                uint64_t *fl = p.flags + (size_t)b * kFlagWords;
                uint32_t u = 0;
                bool ok = true;
                for (int rho = 0; ok; ++rho) {
                    Chain cc;
                    if (!chain_of(rho, &cc)) break;
                    // (an empty chain is passed at once: nothing of it is read)
                    if (cc.nck == 0) st_release_u64(fl, (uint64_t)(rho + 1) << 32);
                    for (int m = 0; m < cc.nck && ok; ++m, ++u) {
                        ok = wt.wait_count(landed, u + 1);
                        if (ok) st_release_u64(fl, cons_after(rho, m, cc.nck));
                    }
                }
            }
            if (warp == 8 && lane == 0) {
                uint64_t *fl = p.flags + (size_t)b * kFlagWords;
                int lrho = 0, lm = 0;  // loader cursor: the chain and chunk of the next load
                Chain lcc;
                bool lhave = false;
                bool ok = true;
                int *iss = issued;
                // the next chain with chunks from round lrho on
                auto lopen = [&]() {
                    for (;; ++lrho) {
                        lhave = chain_of(lrho, &lcc);
                        if (!lhave || lcc.nck > 0) return;
                    }
                };
                // the loads of the cursor's chunk (global index lu) into its stage (free)
                auto load_one = [&](uint32_t lu) {
                    if (ok) ok = wt.wait_global(fl + 1 + (lm % NR), ready_tag(lrho, lm), true);
                    if (!ok) return;
                    fence_proxy_async_global();
                    const uint8_t *src = p.ring + ((size_t)b * NR + (lm % NR)) * RING_STRIDE;
                    const long long t0 = lcc.t_begin + (long long)lm * C;
                    uint8_t *st = stage_of(lu);
                    uint64_t *bf = bars + CB_FULL + (lu & 1);
                    mbar_arrive_expect_tx(bf, STAGE_TX);
                    bulk_load(st, src, RG_YQ, bf);
                    bulk_load(st + RG_YQ, src + RG_YQ, YQ_HALF, bf);
                    bulk_load(st + RG_YQ + YQ_HALF, src + RG_YQ + YQ_HALF, YQ_HALF, bf);
                    tma_load_4d(st + CS_V, &tm_v2, 0, (int)t0, 0, lcc.h, bf);
                    ++iss[lu & 1];
                    // the V tile two chunks on, into L2
                    if (lm + 2 < lcc.nck) tma_prefetch_l2_4d(&tm_v2, 0, (int)(t0 + 2 * C), 0, lcc.h);
                };
                // after the chunk has landed: count it (warp 9 gives the slot back),
                // move the cursor on
                auto loaded = [&](uint32_t uu) {
                    st_release_cta_u32(landed, uu + 1);
                    if (++lm == lcc.nck) {
                        lm = 0;
                        ++lrho;
                        lopen();
                    }
                };
                lopen();
                if (lhave) load_one(0);
                uint32_t u = 0;
                for (int rho = 0; ok; ++rho) {
                    Chain cc;
                    if (!chain_of(rho, &cc)) break;
                    for (int m = 0; m < cc.nck && ok; ++m, ++u) {
                        const int s = u & 1;
                        ok = wt.wait(bars + CB_FULL + s, (u >> 1) & 1);
                        if (!ok) break;
                        loaded(u);
                        if (u >= 2) ok = wt.wait(bars + CB_DFREE + s, ((u >> 1) - 1) & 1);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t sb = smem_u32(stage_of(u));
                        const uint64_t d_v = desc_sw128(sb + CS_V, 8192, 1024);
                        const uint64_t d_zr = desc_sw128(sb + RG_ZT, 16, 1024);
#pragma unroll
                        for (int kk = 0; kk < C / 16; ++kk)
                            mma_bf16(tmem + TM_D + TM_DSTRIDE * s, d_v + 128 * kk, d_zr + 2 * kk, ID_VZR, kk > 0);
                        mbar_arrive(bars + CB_AISS + s);
                        // chunk u + 1's stage held chunk u - 1: free once its products are
                        // done (its decay was read before chunk u's product went out)
                        if (lhave) {
                            if (u >= 1)
                                ok = wt.wait(bars + CB_DSFULL + ((u - 1) & 1), ((u - 1) >> 1) & 1);
                            if (ok) load_one(u + 1);
                        }
                    }
                }
                if (*abort_flag) {
                    mma_commit(bars + CB_DRAIN + 1);
                    mbar_wait(bars + CB_DRAIN + 1, 0, kWaitLimit);
                    for (int i = 0; i < 2; ++i)
                        if (iss[i] > 0)
                            mbar_wait(bars + CB_FULL + i, (uint32_t)((iss[i] - 1) & 1), kWaitLimit);
                }
            }
        } else {
            // ---- output warps: D_O = o^T (lane j = value channel, columns = tokens).
            //      A full chunk goes through an o tile in shared memory (two buffers)
            //      and two TMA tensor stores issued by lane 0 of warp 12; a partial
            //      one (a sequence's last) is stored row by row, so that nothing past
            //      the sequence end is written.
            const int j = 32 * (warp & 3) + lane;
            const bool ostorer = warp == 12 && lane == 0;
            uint32_t u = 0;
            bool stop = false, prev_full = false;
            for (int rho = 0; !stop; ++rho) {
                Chain cc;
                if (!chain_of(rho, &cc)) break;
                for (int m = 0; m < cc.nck; ++m, ++u) {
                    const int s = u & 1;
                    const long long t0 = cc.t_begin + (long long)m * C;
                    const int L = (int)min((long long)C, cc.t_end - t0);
                    const bool full = L == C;
                    // buffer s last held chunk u - 2: its stores have read it (all stores,
                    // when chunk u - 1 was partial and committed none)
                    if (ostorer && full) {
                        if (prev_full) bulk_wait_read_but_last();
                        else bulk_wait_read();
                    }
                    const bool ok = wt.warp_wait(bars + CB_DSFULL + s, (u >> 1) & 1, lane);
                    if (named_bar_or(BAR_OUT, 128, !ok)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    float x[64];
                    tmem_load<64>(tmem + TM_D + TM_DSTRIDE * s + TM_O + lane_q, x);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars + CB_DFREE + s);
                    // lane pairs (j even, j + 1) hold bf16 pairs: the even lane row r,
                    // the odd lane row r + 1
                    const bool odd = lane & 1;
                    if (full) {
                        uint8_t *ob = sm + OFF_OBUF + s * OBUF_BYTES + (j >> 6) * 8192;
                        const int col = (j & 63) & ~1;
#pragma unroll
                        for (int r = 0; r < C; r += 2) {
                            const float mine = odd ? x[r] : x[r + 1];
                            const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
                            const int row = odd ? r + 1 : r;
                            const uint32_t v = odd ? pack2(other, x[r + 1]) : pack2(x[r], other);
                            *reinterpret_cast<uint32_t *>(ob + row * 128 + (((col >> 3) ^ (row & 7)) << 4) +
                                                          (col & 7) * 2) = v;
                        }
                        fence_proxy_async_smem();
                        named_bar_sync(BAR_OUT, 128);
                        if (ostorer) {
                            const uint8_t *ot = sm + OFF_OBUF + s * OBUF_BYTES;
                            tma_store_3d(&tm_o, ot, 0, cc.h, (int)t0);
                            tma_store_3d(&tm_o, ot + 8192, 64, cc.h, (int)t0);
                            bulk_commit();
                        }
                    } else {
                        __nv_bfloat16 *ob = reinterpret_cast<__nv_bfloat16 *>(a.o);
#pragma unroll
                        for (int r = 0; r < C; r += 2) {
                            const float mine = odd ? x[r] : x[r + 1];
                            const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
                            const int row = odd ? r + 1 : r;
                            if (row < L) {
                                const uint32_t v = odd ? pack2(other, x[r + 1]) : pack2(x[r], other);
                                *reinterpret_cast<uint32_t *>(ob + ((t0 + row) * H + cc.h) * (long long)DV +
                                                              (j & ~1)) = v;
                            }
                        }
                    }
                    prev_full = full;
                }
            }
            // every tile store complete before the CTA's shared memory goes away
            if (ostorer) bulk_wait_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        atomicOr(a.err, kErrTimeout);
        // local CTA: every raw buffer's last tile load lands before the CTA exits
        if (!chain_role)
            for (int q = 0; q < 3; ++q)
                if (issued[q] > 0) mbar_wait(bars + LB_TMA + q, (uint32_t)((issued[q] - 1) & 1), kWaitLimit);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

// Before each launch: zero the hand-off words (cons, ready, the grid's abort
// word) and, for a packed batch, write the task offset of every round: round
// rho has (its chains) x (the chunks of its longest sequence) tasks.
__global__ void __launch_bounds__(1024)
pool_schedule_kernel(const PrefillArgs a, int nch, int nrounds, long long *rbase, uint64_t *flags,
                     int nwords) {
    for (int i = threadIdx.x; i < nwords; i += blockDim.x) flags[i] = 0;
    if (rbase == nullptr) return;
    const long long nchains = (long long)a.n_seqs * a.H;
    auto round_tasks = [&](int rho) -> long long {
        const long long x0 = (long long)rho * nch, x1 = min(x0 + nch, nchains);
        long long maxck = 0;
        for (long long n = x0 / a.H; n <= (x1 - 1) / a.H; ++n) {
            long long tb, te;
            seq_range(a, (int)n, &tb, &te);
            maxck = max(maxck, (te - tb + C - 1) / C);
        }
        return (x1 - x0) * maxck;
    };
    const int per = (nrounds + (int)blockDim.x - 1) / (int)blockDim.x;
    const int r0 = (int)threadIdx.x * per, r1 = min(nrounds, r0 + per);
    long long sum = 0;
    for (int rho = r0; rho < r1; ++rho) sum += round_tasks(rho);
    __shared__ long long part[1024];
    part[threadIdx.x] = sum;
    __syncthreads();
    for (int off = 1; off < (int)blockDim.x; off <<= 1) {  // inclusive scan
        const long long v = threadIdx.x >= (unsigned)off ? part[threadIdx.x - off] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    long long base = part[threadIdx.x] - sum;
    for (int rho = r0; rho < r1; ++rho) {
        rbase[rho] = base;
        base += round_tasks(rho);
    }
    if (threadIdx.x == blockDim.x - 1) rbase[nrounds] = part[threadIdx.x];
}

// ------------------------------------------------------------------- host --
struct PoolPlan {
    int nch, nloc;
};

int device_sms() {
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return nsm;
}

// The split of the SMs between chain CTAs and the local pool: the chain CTAs
// take the chains in rounds of nch, so the state pass takes rounds x (chunks
// steps of ~kChainCost cycles + a fill and drain of ~kRoundCost); the pool works
// through every chunk at ~kLocalCost SM-cycles each.  Pick nch to balance the
// two.  (Measured on B200: ~4.0k cycles per chunk on a chain CTA running alone,
// ~10.7k SM-cycles per task when the pool is the bound.)
constexpr double kChainCost = 4000.0, kLocalCost = 10700.0, kRoundCost = 30000.0;

PoolPlan plan_for(const gdn_dims &d, int nsm) {
    PoolPlan pl{0, 0};
    const long long nchains = (long long)(d.n_seqs > 0 ? d.n_seqs : d.B) * d.H;
    const long long seqs = d.n_seqs > 0 ? d.n_seqs : (d.B > 0 ? d.B : 1);
    const double nck = std::max(1.0, (double)d.B * d.T / (double)seqs / C);
    if (nchains <= 0 || nsm < 2) return pl;
    int best = 1;
    double best_t = 1e300;
    const int hi = (int)std::min<long long>(nchains, nsm - 1);
    for (int nch = 1; nch <= hi; ++nch) {
        const double rounds = (double)((nchains + nch - 1) / nch);
        const double t_chain = rounds * (nck * kChainCost + kRoundCost);
        const double t_local = (double)nchains * nck * kLocalCost / (nsm - nch);
        const double t = std::max(t_chain, t_local);
        if (t < best_t * 0.999) {
            best_t = t;
            best = nch;
        }
    }
    if (const char *e = getenv("GDN_POOL_CHAIN_CTAS")) {
        const int v = atoi(e);
        if (v >= 1 && v <= hi) best = v;
    }
    pl.nch = best;
    pl.nloc = nsm - best;
    return pl;
}

constexpr size_t kFlagWordsPerChain = kFlagWords;

// The library's default for GDN: the pool kernel when the sequences are long
// (2048 tokens or more on average) and so few that an SM pair per (sequence,
// head) would leave most of the GPU idle (chains <= SMs / 4).  Measured on B200:
// 32 chains of 65536 tokens 1.81 ms against the two-CTA kernel's 3.48 ms; 64 chains
// of 4096 tokens 277 against 271 us; 512 packed chains of 2176 tokens on average
// 1.33 against 1.17 ms.
constexpr long long kPoolMinMeanTokens = 2048;

size_t flags_bytes(int nch) { return (((size_t)nch * kFlagWordsPerChain + 8) * 8 + 255) & ~size_t(255); }

}  // namespace

bool chunk_pool_preferred(const gdn_dims &d) {
    if (!chunk_pool_supported(d)) return false;
    int nsm = device_sms();
    if (nsm <= 0) nsm = 148;  // (no device: B200's count, so the choice is reproducible)
    const long long seqs = d.n_seqs > 0 ? d.n_seqs : (d.B > 0 ? d.B : 1);
    return (long long)d.B * d.T >= kPoolMinMeanTokens * seqs && 4 * seqs * d.H <= nsm;
}

bool chunk_pool_supported(const gdn_dims &d) {
    return d.dtype == GDN_BF16 && d.d_k == DK && d.d_v == DV && d.decay == GDN_DECAY_SCALAR &&
           (long long)d.B * d.T < (1LL << 31) && d.H < 65536;
}

size_t chunk_pool_scratch_bytes(const gdn_dims &d) {
    const PoolPlan pl = plan_for(d, device_sms());
    if (pl.nch <= 0) return 0;
    const long long nchains = (long long)(d.n_seqs > 0 ? d.n_seqs : d.B) * d.H;
    const long long nrounds = (nchains + pl.nch - 1) / pl.nch;
    return flags_bytes(pl.nch) + (size_t)pl.nch * NR * RING_STRIDE +
           (((size_t)(nrounds + 1) * 8 + 255) & ~size_t(255));
}

cudaError_t launch_chunk_pool(const PrefillArgs &a, cudaStream_t s, int *launches) {
    const long long nchains = (long long)a.n_seqs * a.H;
    const long long ntok = (long long)a.B * a.T;
    if (nchains == 0) return cudaSuccess;
    if (ntok == 0) {
        if (a.s_final && a.s_final != a.s0) {
            const size_t bytes = (size_t)nchains * a.dv * a.dk * sizeof(float);
            return a.s0 ? cudaMemcpyAsync(a.s_final, a.s0, bytes, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(a.s_final, 0, bytes, s);
        }
        return cudaSuccess;
    }
    gdn_dims d{};
    d.B = a.B; d.T = a.T; d.H = a.H; d.d_k = a.dk; d.d_v = a.dv; d.n_seqs = a.n_seqs;
    d.dtype = GDN_BF16; d.decay = GDN_DECAY_SCALAR;
    const int nsm = device_sms();
    const PoolPlan pl = plan_for(d, nsm);
    if (pl.nch <= 0) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    if (!make_tile_map(&mq, a.q, a.dk, a.H, ntok) || !make_tile_map(&mk, a.k, a.dk, a.H, ntok) ||
        !make_halves_map(&mv, a.v, a.H, ntok) || !make_tile_map(&mo, a.o, a.dv, a.H, ntok))
        return cudaErrorInvalidValue;
    PoolArgs p{};
    uint8_t *ws = reinterpret_cast<uint8_t *>(a.scratch);
    p.flags = reinterpret_cast<uint64_t *>(ws);
    p.gabort = reinterpret_cast<uint32_t *>(p.flags + (size_t)pl.nch * kFlagWordsPerChain);
    p.ring = ws + flags_bytes(pl.nch);
    p.nch = pl.nch;
    p.nrounds = (int)((nchains + pl.nch - 1) / pl.nch);
    p.rbase = a.cu_seqlens ? reinterpret_cast<const long long *>(
                                 p.ring + (size_t)pl.nch * NR * RING_STRIDE)
                           : nullptr;
    p.nck = (int)((a.T + C - 1) / C);
    p.ntask = nchains * (long long)p.nck;
    const int nwords = (int)(pl.nch * kFlagWordsPerChain + 8);
    pool_schedule_kernel<<<1, 1024, 0, s>>>(a, p.nch, p.nrounds, const_cast<long long *>(p.rbase),
                                             p.flags, nwords);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (launches) ++*launches;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(chunk_pool_kernel<false>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(chunk_pool_kernel<true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return attr_err;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(pl.nch + pl.nloc));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = a.raw ? cudaLaunchKernelEx(&cfg, chunk_pool_kernel<true>, a, p, mq, mk, mv, mo)
              : cudaLaunchKernelEx(&cfg, chunk_pool_kernel<false>, a, p, mq, mk, mv, mo);
    if (e != cudaSuccess) return e;
    if (launches) ++*launches;
    return cudaSuccess;
}

}  // namespace gdn

// gdn_chunk_pair.cu -- chunkwise gated delta rule prefill on the tensor cores
// with the chunk-local work and the sequential state pass on two different
// SMs: one 2-CTA cluster per (sequence, head), bf16 inputs, d_k = d_v = 128,
// scalar (GDN) or channel-wise (KDA) decay.
//
// Chunkwise form (FG2-GDN paper, section 3.6: WY representation, UT transform,
// inter-chunk state propagation; Gated Delta Networks page, section 3.3, for
// the cumulative decay g_r within a chunk), C = 64 tokens.  With the decay
// written per key channel (KDA; GDN has one value for all channels),
// G_rc = sum_{t<=r} log alpha_tc and Kg = K . e^{G}, Qg = Q . e^{G}:
//
//   A_rs = beta_r sum_c k_rc k_sc e^{G_rc-G_sc} (s < r),  T = (I + A)^{-1}
//   P_rs = sum_c q_rc k_sc e^{G_rc-G_sc} (s <= r)
//   T_b = T diag(beta),  W = T_b Kg,  U = T_b V
//   V'  = U - W S^T,     o = Qg S^T + P V',
//   S  <- S Diag(e^{G_C}) + V'^T Kt,  Kt_sc = k_sc e^{G_Cc - G_sc}.
//
// The output is regrouped so that it needs nothing after the state product:
//   o = (Qg - P W) S^T + (P T_b) V = Qh S^T + R V
// and one accumulator per chunk (M = 128) holds both halves of the pass:
//   D = [Qh; -W] S^T + [R; T_b] V  ->  rows 0-63: o,  rows 64-127: V'.
//
// Rank 0 ("local" CTA) computes, per chunk, everything that depends only on
// the chunk's tokens and writes Kt, Qh, -W, R, T_b (bf16 tiles in the
// swizzled layout the state CTA's MMAs read) and e^{G_C} into a 4-slot ring in
// global memory (chunk m in slot m % 4), L2-resident since it is rewritten every
// fourth chunk.  GDN: two groups of 8 warps work on two chunks at once (even / odd
// chunks); KDA: group 1 runs the next chunk's gate pass while group 0 runs the
// products of this one.  Per chunk:
//   GDN: D = [K; Q] K^T, then A and P take the decay e^{g_r-g_s} (exact inside
//        each row's own 16-token block, factored at the 16-token block
//        boundaries elsewhere, both factors <= 1); T_bg = T_b diag(e^{g}) so
//        that W = T_bg K; [P T_bg | R] = P [T_bg | T_b]; [W; P W] = [T_bg; P T_bg] K.
//   KDA (group 1, one chunk ahead): each 16-token row block i takes its start
//        as the reference (off_i = G at the end of block i - 1, off_0 = 0): K and
//        Q become KD, QD = . e^{G - off_{i(r)}} in place (<= 1), and B_i =
//        K[0, 16(i+1)) . e^{off_i - G}, stacked into one 160-row operand, so that
//        one MMA (N = 160) gives D_i = [KD; QD] B_i^T, the decayed A and P of
//        block i (masks only).  Off the diagonal block both factors are <= 1 (they
//        can only underflow, where the exact term is as small); inside it B_i's
//        factor is e^{off_i - G} <= e^{block decay}.  A channel whose decay over
//        the block passes e^{-kMaxNegLogDecay} is zeroed in B_i's diagonal rows,
//        and its exact diagonal-block terms k_r k_s e^{G_r - G_s}, q_r k_s e^{G_r
//        - G_s} (exponent <= 0, taken directly) are summed into a correction
//        table that the A/P phase adds.  Exact for any decay.  Then (group 0)
//        R = P T_b, Kg = KD . e^{off}, [W; P W] = [T_b; R] Kg, and
//        Qh = QD . e^{off} - P W.
// T comes from blocked forward substitution in fp32 (tf32 MMAs for the
// off-diagonal blocks), computed in place of A.  The ring tiles leave shared
// memory by bulk copy in two groups (what the group's next chunk rewrites early
// first), and the state CTA learns of a slot through a cluster mbarrier.
// Rank 1 ("state" CTA) holds S (fp32, registers) for all 128 value channels as
// two independent halves of 64, each with its own chain of warps, loads each
// chunk's ring slot and V tile (bulk copy + TMA), and per chunk and half
// issues D = [R;T_b] V_h + [Qh;-W] S_h^T, writes o, converts V' to bf16 and
// issues dS = Kt^T V'.
//
// The CTAs signal each other with mbarriers (ring slot written / ring slot
// read).  Every wait is bounded: on expiry the CTA records kErrTimeout, raises
// the abort flag of both CTAs, drains what it issued and leaves through the
// final cluster barrier.
#include <mutex>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = kChunk;  // 64
constexpr int DK = 128, DV = 128;
constexpr int kThreads = 512;
constexpr long long kWaitLimit = kDefaultWaitLimit;  // drains after an abort
constexpr int LDA = 68;                      // fp32 row stride of A / T
constexpr float kMaxNegLogDecay = 80.f;      // e^{80} < bf16 and fp32 max; e^{-80} normal

// ---- ring slot / state-CTA stage layout (bytes, 1024-aligned tiles) --------
// per atom column a (d_k 64a .. 64a+63):  [Kt rows 0-63 | Qh rows | -W rows]
constexpr uint32_t SG_KT = 0, SG_QH = 8192, SG_MW = 16384, SG_AC = 24576;
constexpr uint32_t SG_R = 49152, SG_TB = 57344;  // [R; T_b]  (A of the V product)
constexpr uint32_t SG_TILES = 65536;             // ring slot: the tiles, then
constexpr uint32_t SG_DECB = 512;                //   e^{G_C} per key channel
constexpr uint32_t RING_STRIDE = SG_TILES + 1024;
constexpr int NRING = 4;                         // ring slots per cluster (chunk m: slot m % 4)
constexpr uint32_t SG_V = 65536;                 // stage: V tiles, d_v halves at +8K
constexpr uint32_t SG_DEC = 81920;               //        e^{G_C}
constexpr uint32_t S_STAGE = 82944;
constexpr uint32_t S_STAGE_TX = SG_TILES + SG_DECB + 2 * 8192;
constexpr uint32_t S_OFF_SB = 2 * S_STAGE;       // S_h^T bf16, MN-major [c][i], 16 KB per half
constexpr uint32_t S_OFF_VP = S_OFF_SB + 2 * 16384;  // V'_h bf16, MN-major [r][i], 8 KB per half

// ---- local-CTA layout ------------------------------------------------------------
// A raw tile buffer is [K0 | Q0 | K1 | Q1], 8 KB each (TMA), atom column stride
// L_RAW_AC, so that [K_a; Q_a] is an M=128 tile.  A group's space holds
// [P | X1 | X2 | X3] (8 KB each; [P; X1] is the A operand of the P products,
// whose rows 64-127 are never read), A and then T in place (fp32 [64][LDA]),
// and two gate-row buffers.
//   GDN: X1 = T_bg, X2 = P T_bg, X3 = T_b;  KDA: X1 = T_b, X2 = R, X3 = Qh staging
// GDN: three raw buffers shared by the two groups (chunk m in buffer m % 3, so
// that a chunk's tiles are loaded while the chunk three back is still being
// written out), then the two group spaces; Kt replaces K in its raw buffer.
// KDA: group 0's space starts with its raw buffer and its Kt buffer; group 1's
// space holds the gate group's buffers (below).
constexpr uint32_t L_RAW_AC = 16384;
constexpr uint32_t RAW_BYTES = 32768;
constexpr uint32_t PZ_P = 0, PZ_X1 = 8192, PZ_X2 = 16384, PZ_X3 = 24576, PZT_BYTES = 32768;
constexpr uint32_t AT_BYTES = 64 * LDA * 4;
constexpr uint32_t GATES_STRIDE = 3072;
template <bool CH>
struct Lay {
    static constexpr uint32_t RAWP = 0;                           // GDN: the 3 raw buffers
    static constexpr uint32_t G0 = CH ? 0 : 3 * RAW_BYTES;        // group 0's space
    static constexpr uint32_t RAW = 0, KX = RAW_BYTES;            // KDA, within group 0's space
    static constexpr uint32_t PZT = CH ? KX + 16384 : 0;
    static constexpr uint32_t AT = PZT + PZT_BYTES;
    static constexpr uint32_t GATES = AT + AT_BYTES;
    static constexpr uint32_t GSZ = GATES + 2 * GATES_STRIDE;     // a group's space
};
static_assert(Lay<false>::GATES % 1024 == 0 && Lay<false>::GSZ % 1024 == 0 &&
              Lay<true>::GATES % 1024 == 0 && Lay<true>::GSZ % 1024 == 0, "local group layout");
// gate rows (floats).  GDN: g beta beta*gamma colf rowf[4] kh gamma, and dec;
// KDA: beta and dec (the first 512 floats are the prefix-sum scratch)
constexpr int GR_G = 0, GR_B = 64, GR_BG = 128, GR_COLF = 192, GR_ROWF = 256, GR_KH = 512,
              GR_GAM = 576, GR_DEC = 640;
constexpr int GR_KB = 512;  // KDA beta (after the scratch)
// KDA (group 0 runs the products, group 1 the gate pass of the next chunk; the
// group-1 space holds): the B operand of the decayed [K; Q] products, rows
// di_col(i) .. of it being, for 16-token row block i, B_i = K[0, 16(i+1)) .
// e^{off_i - G} (off_i: G at the block's start), 160 rows per atom column; then
// two per-block tables, a second Kt buffer, a second raw tile buffer (raw tiles
// and tables alternate by chunk parity) and the two correction tables.  W's
// operand Kg = K . e^{G} replaces KD in its raw tile once the products are done.
constexpr uint32_t L_BREG = Lay<true>::GSZ;  // (group 1's space)
constexpr uint32_t BREG_AC = 160 * 128;      // atom column stride of the stacked B
__host__ __device__ constexpr uint32_t di_col(int i) { return 8u * i * (i + 1); }  // 0, 16, 48, 96
constexpr uint32_t KTAB_BYTES = 4096;              // fp32 [4][128] x 2: block totals, e^{off_i}
constexpr uint32_t L_KTAB = L_BREG + 2 * BREG_AC;  // two tables
constexpr uint32_t L_KX2 = L_KTAB + 2 * KTAB_BYTES;  // KDA's second Kt buffer
constexpr uint32_t L_RAW2 = L_KX2 + 16384;         // KDA's second raw tiles [K0 | Q0 | K1 | Q1]
// the exact diagonal-block terms of the channels whose decay over a 16-token
// block passes e^{-kMaxNegLogDecay}: fp32 [block][A, P][lower triangle incl. the
// diagonal], and a word "the table holds this chunk's terms", two tables by chunk
// parity; then the gate group's count of such channels per block.  The channels'
// k, q, cumulative log decays G and per-token decays alpha_s = e^{G_s - G_{s-1}}
// (fp32 [16] each) are staged, up to KSTG_CAP per block at a time, in the B region
// (free between the gate pass's B_FREE wait and its rewrite of B).
constexpr int KCOR_TRI = 136, KCOR_FLAG = 8 * KCOR_TRI;
constexpr uint32_t KCOR_BYTES = (KCOR_FLAG + 4) * 4;
constexpr uint32_t L_KCOR = L_RAW2 + RAW_BYTES;
constexpr uint32_t L_KSTG = L_KCOR + 2 * KCOR_BYTES;  // 4 counts (one per block)
constexpr uint32_t KSTG_BYTES = 16;
constexpr int KSTG_CAP = 40;                          // channels per block and batch
constexpr int KSTG_REC = 64;                          // floats per staged channel
static_assert(4 * KSTG_CAP * KSTG_REC * 4 <= 2 * 160 * 128, "staging in the B region");
constexpr uint32_t TM_KD = 192;                    // D = [D_0 | D_1 | D_2 | D_3], 160 columns
constexpr uint32_t ID_KD = idesc_bf16(128, 160, false, false);
static_assert(L_RAW2 % 1024 == 0, "KDA layout");

// ---- shared bookkeeping (same offset in both CTAs, so peers can address it) --
constexpr uint32_t OFF_COMMON = 215040;
static_assert(S_OFF_VP + 2 * 8192 <= OFF_COMMON && L_KSTG + KSTG_BYTES <= OFF_COMMON &&
              Lay<false>::G0 + 2 * Lay<false>::GSZ <= OFF_COMMON, "shared memory layout");
constexpr uint32_t CM_ABORT = 0, CM_SLOT = 4, CM_TMEM = 8, CM_ISSUED = 32, CM_BARS = 64;
constexpr int NBARS = 18;
constexpr uint32_t SMEM_USED = OFF_COMMON + CM_BARS + NBARS * 8;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
// state-CTA mbarriers (READY: one per ring slot; OFREE: per stage and value half)
constexpr int SB_FULL = 0, SB_READY = 2, SB_VO = 6, SB_DS = 8, SB_OFREE = 10, SB_CONS = 14,
              SB_DRAIN = 16;
// local-CTA mbarriers (TMA: one per raw buffer; SLOTFREE: one per ring slot)
constexpr int LB_TMA = 0, LB_L = 3, LB_SLOTFREE = 5, LB_DRAIN = 9, LB_OFFSET = 11, LB_GATE = 12,
              LB_BFREE = 13;

// TMEM columns
constexpr uint32_t TM_KQ = 0, TM_AB = 64, TM_GROUP = 192;  // local: per group
constexpr uint32_t TM_DS = 256;                            // state: D_vo[st][h] at 64 (2st+h)
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);   // [K;Q] K^T, [Kg;Qg] Ki^T
constexpr uint32_t ID_N128 = idesc_bf16(128, 128, false, true); // [P;0][T_bg|T_b], [X1;X2] K
constexpr uint32_t ID_N64 = idesc_bf16(128, 64, false, true);   // [P;0] T_b, [R;T_b] V_h, [Qh;-W] S_h^T
constexpr uint32_t ID_MM = idesc_bf16(128, 64, true, true);     // Kt^T V'_h

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

// Decay of 32 entries (columns 32*half ..) of row r of a C x C product,
// e^{g_r - g_s} for s < r (strict) or s <= r.  rq = r / 32 is uniform per warp,
// so each warp takes one of three branches: the diagonal 32x32 block (exact
// exponentials inside the row's own 16-block, g_r - g_s <= 0 wherever kept,
// masked elsewhere; factored across the 16-block boundary), a block strictly
// below it (factored at the 16-block boundary: e^{g_r - g_e} e^{g_e - g_s}, both
// factors <= 1), or a block above it (not called: nothing to keep).
// KDA's correction table for one batch of staged fast-decaying channels: the
// 256 gate threads each take one row i of one block's A or P terms and one half
// of its columns s (8 of them), and sum, over the block's staged channels,
// left_i k_s e^{G_i - G_s} (left = k for A, s < i; q for P, s <= i).  Along the
// row the factor is a running product, e^{G_i - G_{s-1}} = e^{G_i - G_s} alpha_s,
// every factor <= 1 (it can only underflow, where the exact term is as small), so
// a channel costs one exponential per thread.  Inlined, with the channel loop
// rolled: as a call its code was fetched cold at every chunk, which measured
// slower.
__device__ __forceinline__ void kda_correction_entries(float *cor, const float *stg, int n0, int n1,
                                                    int n2, int n3, int p0, int cap, int gtid) {
    const int blk = gtid >> 6, ap = (gtid >> 5) & 1, i = (gtid >> 1) & 15, hf = gtid & 1;
    const int s0 = 8 * hf, top = s0 + 7;
    if (s0 > i) return;  // the row's terms all lie left of this half
    const int nb = blk == 0 ? n0 : blk == 1 ? n1 : blk == 2 ? n2 : n3;
    const int np = min(cap, nb - p0);
    float *ct = cor + (2 * blk + ap) * 136 + i * (i + 1) / 2;  // row i: entries s = 0 .. i
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = (p0 > 0 && s0 + j <= i) ? ct[s0 + j] : 0.f;
    const float *d = stg + blk * cap * KSTG_REC;
#pragma unroll 1
    for (int pp = 0; pp < np; ++pp) {
        const float *dq = d + pp * KSTG_REC;
        const float li = dq[16 * ap + i], gi = dq[32 + i];
        float k8[8], a8[8];
        *reinterpret_cast<float4 *>(k8) = *reinterpret_cast<const float4 *>(dq + s0);
        *reinterpret_cast<float4 *>(k8 + 4) = *reinterpret_cast<const float4 *>(dq + s0 + 4);
        *reinterpret_cast<float4 *>(a8) = *reinterpret_cast<const float4 *>(dq + 48 + s0);
        *reinterpret_cast<float4 *>(a8 + 4) = *reinterpret_cast<const float4 *>(dq + 48 + s0 + 4);
        // e^{G_i - G_top} when the row reaches past this half (exponent <= 0)
        float w = i > top ? __expf(gi - dq[32 + top]) : 0.f;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
            if (s0 + j == i) w = 1.f;
            const float wt = (s0 + j == i && ap == 0) ? 0.f : w;  // A: no diagonal term
            acc[j] = fmaf(li * k8[j], wt, acc[j]);
            w *= a8[j];
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (s0 + j <= i) ct[s0 + j] = acc[j];
}

// FG2-GDN: K <- sqrt(beta) . K in place for one gate thread's 16 rows (block rq)
// and two key channels (c0, c0 + 1 = column cc of atom ac); rows past the
// sequence end (>= L) are zero and stay so.  Out of line like the correction.
__device__ __noinline__ void fg2_scale_keys(uint8_t *rawp, const float *bp, size_t row_stride, int rq,
                                            int L, int ac, int cc) {
    const uint32_t cof = (uint32_t)((cc & 7) * 2);
    // all 16 rows' rate pairs in flight at once (one 8-byte load each when aligned)
    const bool al8 = ((reinterpret_cast<uintptr_t>(bp) | (row_stride * sizeof(float))) & 7) == 0;
    float2 bb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float *pi = bp + i * row_stride;
        bb[i] = 16 * rq + i >= L ? make_float2(0.f, 0.f)
                : al8            ? __ldg(reinterpret_cast<const float2 *>(pi))
                                 : make_float2(__ldg(pi), __ldg(pi + 1));
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        uint32_t *pk = reinterpret_cast<uint32_t *>(rawp + ac * L_RAW_AC + sw128(16 * rq + i, cc >> 3) + cof);
        const uint32_t kw = *pk;
        __nv_bfloat162 t = __floats2bfloat162_rn(__uint_as_float(kw << 16) * sqrtf(bb[i].x),
                                                 __uint_as_float(kw & 0xffff0000u) * sqrtf(bb[i].y));
        *pk = *reinterpret_cast<uint32_t *>(&t);
    }
}

__device__ __forceinline__ void decay_row(float *x, int r, int rq, int half, const float *gr,
                                          bool incl) {
    const float *g = gr + GR_G;
    if (rq == half) {
        // exact exponentials inside the row's own 16-block only (16 per thread);
        // the earlier 16-block of the diagonal 32-block is factored like the
        // blocks below, the later one is masked
        const int rb = r >> 4;  // 2 half or 2 half + 1: differs between the half-warps
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
        const bool upper = rb & 1;  // the row's block is the second of the 32-block
        const float f0 = gr[GR_ROWF + 4 * r + 2 * half];  // to the first block's end
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

// Column j of (I + A_d)^{-1} for the 16x16 diagonal block A_d at (o, o) of the
// fp32 [64][LDA] tile (strictly lower), by left-looking forward substitution:
// t_i = [i == j] - sum_{k < i} a_ik t_k, row i of the block read with float4
// loads (t_k = 0 for k < j makes the rows above j come out right).  Called by
// lanes 0-15 of a warp; the column replaces the block's column j once all 16
// lanes have read the block.
__device__ __forceinline__ void invert_diag16(float *AT, int o, int j) {
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float *row = AT + (o + i) * LDA + o;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < (i + 3) / 4; ++q) {
            const float4 av = *reinterpret_cast<const float4 *>(row + 4 * q);
            const float ak[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (4 * q + e < i) acc[e] = fmaf(ak[e], t[4 * q + e], acc[e]);
        }
        t[i] = (i == j ? 1.f : 0.f) - ((acc[0] + acc[1]) + (acc[2] + acc[3]));
    }
    __syncwarp(0x0000ffffu);
#pragma unroll
    for (int i = 0; i < 16; ++i) AT[(o + i) * LDA + o + j] = t[i];
}

struct Waiter {
    volatile int *abort;
    uint32_t peer_abort;  // shared::cluster address of the peer's abort flag
    long long limit;      // SM cycles before a data wait gives up
    __device__ __forceinline__ void raise() const {
        *abort = 1;
        st_peer_u32(peer_abort, 1u);
    }
    // Bounded wait for a phase completed inside this CTA (MMA commits, TMA).  No
    // sleep between polls: mbarrier.try_wait suspends the thread for a while
    // itself, and a sleep only delays the waiter (measured: 2.5% of the prefill).
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
    // Bounded wait for a phase completed by the peer CTA (acquire at cluster scope).
    __device__ __forceinline__ bool wait_peer(uint64_t *bar, uint32_t parity) const {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        const long long t0 = clock64();
        while (!mbar_try_wait_cluster(bar, parity)) {
            if (*abort) return false;
            if (clock64() - t0 > limit) {
                raise();
                return false;
            }
        }
        return true;
    }
    // One lane waits, the warp gets the answer.
    __device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int lane) const {
        bool ok = true;
        if (lane == 0) ok = wait(bar, parity);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
};

template <bool CH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
chunk_pair_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  uint8_t *ring, int ring_slots, const int32_t *order) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint8_t *cm = sm + OFF_COMMON;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(cm + CM_ABORT);
    uint64_t *bars = reinterpret_cast<uint64_t *>(cm + CM_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(cm + CM_TMEM);
    int *issued = reinterpret_cast<int *>(cm + CM_ISSUED);  // [3] loads issued per stage / raw buffer

    const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // cluster i takes (sequence, head) item i; a packed batch's sequences are taken
    // longest first (order), so that the last clusters to start are short ones
    const int item = blockIdx.x >> 1;
    const int h = item % a.H;
    const int n = order ? order[item / a.H] : item / a.H;
    const int H = a.H;
    long long t_begin, t_end;
    seq_range(a, n, &t_begin, &t_end);
    const int nchunks = (int)((t_end - t_begin + C - 1) / C);
    const size_t st_base = ((size_t)n * H + h) * DV * DK;
    auto chunk_len = [&](int m) -> int {
        const long long rem = t_end - (t_begin + (long long)m * C);
        return rem < C ? (int)rem : C;
    };

    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i)
            mbar_init(bars + i, (rank == 1 && (i == SB_CONS || i == SB_CONS + 1)) ? 2 : 1);
        fence_mbar_init();
        *abort_flag = 0;
        issued[0] = issued[1] = issued[2] = 0;
        if (rank == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
        } else {
            tma_prefetch_desc(&tm_v);
        }
    }
    if (CH && rank == 0)  // the correction tables and the staging count
        for (int i = tid; i < (int)((2 * KCOR_BYTES + 16) / 4); i += kThreads)
            reinterpret_cast<float *>(sm + L_KCOR)[i] = 0.f;
    cluster_sync();  // both CTAs' barriers and flags are initialised
    if (rank == 1 && tid == 0) {
        // the ring slot pair of this cluster: indexed by the state CTA's SM,
        // which no other running cluster shares
        const int slot = (int)sm_id();
        const int v = slot < ring_slots ? slot : -1;
        *reinterpret_cast<volatile int *>(cm + CM_SLOT) = v;
        st_peer_u32(map_peer(sbase + OFF_COMMON + CM_SLOT, peer), (uint32_t)v);
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int slot = *reinterpret_cast<volatile int *>(cm + CM_SLOT);
    const Waiter wt{abort_flag, map_peer(sbase + OFF_COMMON + CM_ABORT, peer), data_wait_limit(a.err)};
    if (slot < 0) {
        if (tid == 0) {
            atomicOr(a.err, kErrInternal);
            *abort_flag = 1;
        }
    }
    uint8_t *ring_pair = slot >= 0 ? ring + (size_t)slot * NRING * RING_STRIDE : ring;

    if (slot >= 0 && rank == 0) {
        // ============================ local CTA ============================
        const int g = warp >> 3, lw = warp & 7, lq = warp & 3, lhalf = lw >> 2;
        const int gtid = tid & 255;
        const int BAR_G = 1 + g, BAR_INV = 3 + g;
        using LY = Lay<CH>;
        uint8_t *grp = sm + LY::G0 + g * LY::GSZ;
        const uint32_t gbase = sbase + LY::G0 + g * LY::GSZ;
        // raw tiles of chunk m: GDN, buffer m % 3; KDA, by parity.  Each buffer has
        // its TMA barrier, the loads into it completing in order.
        auto rbuf = [&](int m) -> int { return CH ? (m & 1) : (m % 3); };
        auto raw_of = [&](int m) -> uint8_t * {
            return CH ? ((m & 1) ? sm + L_RAW2 : sm + LY::RAW) : sm + LY::RAWP + rbuf(m) * RAW_BYTES;
        };
        auto tma_phase = [&](int m) -> uint32_t { return (uint32_t)((CH ? (m >> 1) : (m / 3)) & 1); };
        auto ktab_of = [&](int m) { return reinterpret_cast<float *>(sm + L_KTAB + (m & 1) * KTAB_BYTES); };
        auto kcor_of = [&](int m) { return reinterpret_cast<float *>(sm + L_KCOR + (m & 1) * KCOR_BYTES); };
        uint8_t *kxt = CH ? sm + LY::KX : nullptr;  // KDA Kt of even chunks
        uint8_t *pzt = grp + LY::PZT;
        float *AT = reinterpret_cast<float *>(grp + LY::AT);
        uint64_t *bar_l = bars + LB_L + g;
        const uint32_t peer_ready0 = map_peer(smem_u32(bars + SB_READY), peer);
        const uint32_t tm_kq = tmem + g * TM_GROUP + TM_KQ, tm_ab = tmem + g * TM_GROUP + TM_AB;
        const int mstep = CH ? 1 : 2;  // chunks of this group: g, g + mstep, ...
        const bool active = !CH || g == 0;
        const uint32_t lane_off = (uint32_t)(32 * lq) << 16;
        const uint64_t d_pz = desc_sw128(gbase + LY::PZT + PZ_P, 16, 1024);    // [P; X1]
        const uint64_t d_x1b = desc_sw128(gbase + LY::PZT + PZ_X1, PZ_X3 - PZ_X1, 1024);  // X1 (| X3)
        const uint64_t d_x1x2 = desc_sw128(gbase + LY::PZT + PZ_X1, 16, 1024);  // [X1; X2]
        uint32_t bl_wait = 0;
        const bool issuer = gtid == 0;       // MMAs
        const bool storer = gtid == 7 * 32;  // tile reloads, ring stores and the hand-off
        bool pend = false;                   // storer: a chunk's ring stores are in flight
        int pend_slot = 0;
        // storer: once the pending chunk's ring stores are complete, hand it over
        auto hand_over = [&]() {
            bulk_wait_all();
            fence_proxy_async_global();
            mbar_arrive_peer(peer_ready0 + 8 * pend_slot);
            pend = false;
        };


        auto issue_tma = [&](int m) {
            const long long t0 = t_begin + (long long)m * C;
            uint8_t *dst = raw_of(m);
            uint64_t *bt = bars + LB_TMA + rbuf(m);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bt, 4 * 8192);
            tma_load_3d(dst + 0, &tm_k, 0, h, (int)t0, bt);
            tma_load_3d(dst + 8192, &tm_q, 0, h, (int)t0, bt);
            tma_load_3d(dst + L_RAW_AC, &tm_k, 64, h, (int)t0, bt);
            tma_load_3d(dst + L_RAW_AC + 8192, &tm_q, 64, h, (int)t0, bt);
            atomicAdd(issued + rbuf(m), 1);  // (GDN: both groups' storers load)
        };
        // gate rows of a chunk: two buffers, by the chunk's index within the group
        auto gate_rows = [&](int m) {
            return reinterpret_cast<float *>(grp + LY::GATES + (((CH ? m : m >> 1)) & 1) * GATES_STRIDE);
        };
        // GDN gates, prefetched one group chunk ahead in the registers of warp lw 4
        float nla0 = 0.f, nla1 = 0.f, nbe0 = 0.f, nbe1 = 0.f;
        auto load_gates = [&](int m) {
            const long long t0 = t_begin + (long long)m * C;
            const int L = chunk_len(m), r0 = 2 * lane, r1 = 2 * lane + 1;
            nla0 = r0 < L ? a.log_alpha[(t0 + r0) * H + h] : 0.f;
            nla1 = r1 < L ? a.log_alpha[(t0 + r1) * H + h] : 0.f;
            nbe0 = r0 < L ? a.beta[(t0 + r0) * H + h] : 0.f;
            nbe1 = r1 < L ? a.beta[(t0 + r1) * H + h] : 0.f;
        };
        // GDN gate rows of chunk mm (one warp): cumulative log decay, beta,
        // the factored block decays, kh and gamma, e^{g_C} for every channel
        auto compute_gates = [&](int mm) {
            float *gr = gate_rows(mm);
            const int r0 = 2 * lane, r1 = 2 * lane + 1;
            const float la0 = nla0, la1 = nla1, be0 = nbe0, be1 = nbe1;
            if (mm + 2 < nchunks) load_gates(mm + 2);
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

        // the first chunks' tiles: GDN, chunks 0-2 (one per raw buffer); KDA, 0 and 1
        if (active && storer && g < nchunks) issue_tma(g);
        if (active && storer && g == 0 && (CH ? 1 : 2) < nchunks) issue_tma(CH ? 1 : 2);
        if (!CH && lw == 4 && g < nchunks) {
            load_gates(g);
            compute_gates(g);
        }
        // group 1 starts half a chunk after group 0, so that the two groups'
        // CUDA-core phases tend to overlap the other's MMA and load waits
        bool ok0 = true;
        if (!CH && g == 1 && issuer && nchunks >= 2) ok0 = wt.wait(bars + LB_OFFSET, 0);
        named_bar_or(BAR_G, 256, !ok0);

        if (CH && g == 1) {
            // ===== KDA gate group: chunk m's per-channel gates while group 0 runs
            //       the products of chunk m - 1 =====
            for (int m = 0; m < nchunks; ++m) {
                const long long t0 = t_begin + (long long)m * C;
                const int L = chunk_len(m);
                uint8_t *rawp = raw_of(m);
                float *ktab = ktab_of(m);
                float *gr = reinterpret_cast<float *>(sm + LY::GATES + (m & 1) * GATES_STRIDE);  // group 0's
                uint8_t *kxc = (m & 1) ? sm + L_KX2 : sm + LY::KX;
                bool ok = true;
                if (m + 1 < nchunks) {  // the next chunk's per-channel gates into L2
                    const int pr = gtid >> 2, pc = gtid & 3;  // 64 rows x 4 lines of 128 B
                    if (t0 + C + pr < t_end) {
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(a.log_alpha + ((t0 + C + pr) * H + h) * DK + 32 * pc));
                        if (a.beta_channel)  // FG2-GDN: the rates per key channel likewise
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.beta + ((t0 + C + pr) * H + h) * DK + 32 * pc));
                    }
                }
                // ---- KDA gates: G_rc by a prefix sum over the rows (thread: two
                //      channels, the 16 rows of block rq) and the block totals; then
                //      KD = K e^{G - off_{i(r)}} and QD likewise in place, Kt = K
                //      e^{G_C - G} (ring tile), B_i = K[0,16(i+1)) e^{off_i - G}, and the
                //      exact diagonal-block terms of fast-decaying channels.  The sums
                //      need no tiles, so they run while the tiles load.
                const int cp = gtid & 63, rq = gtid >> 6, c0 = 2 * cp;
                float gl0[16], gl1[16], acc0 = 0.f, acc1 = 0.f;
                const float *lp0 = a.log_alpha + ((t0 + 16 * rq) * H + h) * DK + c0;
                if ((reinterpret_cast<uintptr_t>(a.log_alpha) & 7) == 0) {  // uniform
#pragma unroll
                    for (int i = 0; i < 16; ++i) {  // all loads first, then the sums
                        const float2 v = 16 * rq + i < L
                                             ? *reinterpret_cast<const float2 *>(lp0 + (size_t)i * H * DK)
                                             : make_float2(0.f, 0.f);
                        gl0[i] = v.x;
                        gl1[i] = v.y;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const bool in = 16 * rq + i < L;
                        gl0[i] = in ? lp0[(size_t)i * H * DK] : 0.f;
                        gl1[i] = in ? lp0[(size_t)i * H * DK + 1] : 0.f;
                    }
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    acc0 += gl0[i];
                    acc1 += gl1[i];
                    gl0[i] = acc0;
                    gl1[i] = acc1;
                }
                *reinterpret_cast<float2 *>(ktab + 128 * rq + c0) = make_float2(acc0, acc1);
                // a channel whose decay over this block passes e^{-kMaxNegLogDecay} leaves
                // the factored diagonal block (below): registered here, counted after the
                // next barrier (the count was reset before chunk m - 1's last barrier)
                const bool fl0 = -acc0 > kMaxNegLogDecay, fl1 = -acc1 > kMaxNegLogDecay;
                uint32_t *kst_cnt = reinterpret_cast<uint32_t *>(sm + L_KSTG);
                const int my0 = fl0 ? (int)atomicAdd(kst_cnt + rq, 1u) : -1;
                const int my1 = fl1 ? (int)atomicAdd(kst_cnt + rq, 1u) : -1;
                // chunk m's tiles: group 0 loads them once chunk m - 2 is done with
                // this parity's raw tiles, table and gate rows (rows past the sequence
                // end are zeroed here)
                if (issuer) ok = wt.wait(bars + LB_TMA + rbuf(m), tma_phase(m));
                if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                for (int idx = gtid; idx < (C - L) * 8; idx += 256) {
                    const uint32_t o = (L + (idx >> 3)) * 128 + (idx & 7) * 16;
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(rawp + o) = z;
                    *reinterpret_cast<uint4 *>(rawp + 8192 + o) = z;
                    *reinterpret_cast<uint4 *>(rawp + L_RAW_AC + o) = z;
                    *reinterpret_cast<uint4 *>(rawp + L_RAW_AC + 8192 + o) = z;
                }
                // (FG2-GDN: unit rate; the per-channel rate scales the keys below)
                if (gtid < 64)
                    gr[GR_KB + gtid] = gtid < L ? (a.beta_channel ? 1.f : a.beta[(t0 + gtid) * H + h]) : 0.f;
                // the B region (read by chunk m - 1's products), chunk m - 2's Kt and
                // e^{G_C} (read by its ring stores) are free once group 0 says so
                if (issuer && m >= 1) ok = wt.wait(bars + LB_BFREE, (uint32_t)((m - 1) & 1));
                if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
                // block starts off_b (G at the end of block b - 1; off_0 = 0) and the
                // chunk total G_C, from the block totals
                float ob0[4], ob1[4], run0 = 0.f, run1 = 0.f;
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const float2 tt = *reinterpret_cast<const float2 *>(ktab + 128 * q2 + c0);
                    ob0[q2] = run0;
                    ob1[q2] = run1;
                    run0 += tt.x;
                    run1 += tt.y;
                }
                float off0 = ob0[0], off1 = ob1[0];
#pragma unroll
                for (int q2 = 1; q2 < 4; ++q2)
                    if (q2 == rq) { off0 = ob0[q2]; off1 = ob1[q2]; }
                if (rq == 0) {
                    *reinterpret_cast<float2 *>(gr + GR_DEC + c0) = make_float2(__expf(run0), __expf(run1));
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2)
                        *reinterpret_cast<float2 *>(ktab + 512 + 128 * q2 + c0) =
                            make_float2(__expf(ob0[q2]), __expf(ob1[q2]));
                }
                const int ac = c0 >> 6, cc = c0 & 63;
                const uint32_t cof = (uint32_t)((cc & 7) * 2);
                auto bf2 = [](float x, float y) {
                    __nv_bfloat162 t = __floats2bfloat162_rn(x, y);
                    return *reinterpret_cast<uint32_t *>(&t);
                };
                // FG2-GDN: K <- sqrt(beta) . K in place, this thread's rows and channels
                if (a.beta_channel)
                    fg2_scale_keys(rawp, a.beta + ((t0 + 16 * rq) * H + h) * DK + c0, (size_t)H * DK, rq, L, ac, cc);
                // this block's end end_rq = off_rq + acc; the factors from it to the later
                // blocks' starts and to the chunk end (all <= 1)
                const float end0 = off0 + acc0, end1 = off1 + acc1;
                float tb0[4], tb1[4];
#pragma unroll
                for (int bi = 0; bi < 4; ++bi) {
                    tb0[bi] = bi > rq ? __expf(ob0[bi] - end0) : 0.f;
                    tb1[bi] = bi > rq ? __expf(ob1[bi] - end1) : 0.f;
                }
                const float tc0 = __expf(run0 - end0), tc1 = __expf(run1 - end1);
                // the exact diagonal-block terms of the flagged channels, k_r k_s e^{G_r -
                // G_s} and q_r k_s e^{G_r - G_s} (s <= r in the block, exponent <= 0), go
                // to the correction table, every thread taking a few entries over all
                // flagged (block, channel) pairs, which their owners stage
                float *cor = kcor_of(m);
                const int nc0 = (int)reinterpret_cast<volatile uint32_t *>(kst_cnt)[0];
                const int nc1 = (int)reinterpret_cast<volatile uint32_t *>(kst_cnt)[1];
                const int nc2 = (int)reinterpret_cast<volatile uint32_t *>(kst_cnt)[2];
                const int nc3 = (int)reinterpret_cast<volatile uint32_t *>(kst_cnt)[3];
                const int maxcnt = max(max(nc0, nc1), max(nc2, nc3));
                const bool anyfl = maxcnt > 0;
                if (anyfl) {
                    // [block][slot][k | q | G][16] fp32
                    float *stg = reinterpret_cast<float *>(sm + L_BREG);
                    for (int p0 = 0; p0 < maxcnt; p0 += KSTG_CAP) {
#pragma unroll 1
                        for (int hc = 0; hc < 2; ++hc) {
                            const int my = hc ? my1 : my0;
                            if (my < p0 || my >= p0 + KSTG_CAP) continue;
                            float *d = stg + (rq * KSTG_CAP + (my - p0)) * KSTG_REC;
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const uint32_t o = sw128(16 * rq + i, cc >> 3) + cof;
                                const uint32_t kw = *reinterpret_cast<const uint32_t *>(rawp + ac * L_RAW_AC + o);
                                const uint32_t qw = *reinterpret_cast<const uint32_t *>(rawp + ac * L_RAW_AC + 8192 + o);
                                const float gi = hc ? gl1[i] : gl0[i];
                                d[i] = hc ? __uint_as_float(kw & 0xffff0000u) : __uint_as_float(kw << 16);
                                d[16 + i] = hc ? __uint_as_float(qw & 0xffff0000u) : __uint_as_float(qw << 16);
                                d[32 + i] = gi;
                                // alpha_i = e^{G_i - G_{i-1}} (alpha_0 is never read)
                                d[48 + i] = i == 0 ? 1.f : __expf(gi - (hc ? gl1[i - 1] : gl0[i - 1]));
                            }
                        }
                        named_bar_sync(BAR_G, 256);
                        kda_correction_entries(cor, stg, nc0, nc1, nc2, nc3, p0, KSTG_CAP, gtid);
                        named_bar_sync(BAR_G, 256);
                    }
                }
                if (gtid == 0) *reinterpret_cast<volatile int *>(cor + KCOR_FLAG) = anyfl ? 1 : 0;
                const float eacc0 = __expf(acc0), eacc1 = __expf(acc1);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = 16 * rq + i;
                    // x = G_r - off_rq in [acc, 0]
                    const float x0 = gl0[i], x1 = gl1[i];
                    const float e0 = __expf(x0), e1 = __expf(x1);  // KD, QD
                    // de = e^{-x} (<= e^{kMaxNegLogDecay} unless flagged: then 0) and
                    // ee = e^{acc - x} <= 1, to the block end
                    float de0, ee0, de1, ee1;
                    {
                        // one exponential per channel: e^{-x} unless flagged, e^{acc - x} if
                        const float t0 = __expf(fl0 ? acc0 - x0 : -x0), t1 = __expf(fl1 ? acc1 - x1 : -x1);
                        de0 = fl0 ? 0.f : t0; ee0 = fl0 ? t0 : eacc0 * t0;
                        de1 = fl1 ? 0.f : t1; ee1 = fl1 ? t1 : eacc1 * t1;
                    }
                    const uint32_t o = sw128(r, cc >> 3) + cof;
                    uint32_t *pk = reinterpret_cast<uint32_t *>(rawp + ac * L_RAW_AC + o);
                    uint32_t *pq = reinterpret_cast<uint32_t *>(rawp + ac * L_RAW_AC + 8192 + o);
                    const uint32_t kw = *pk, qw = *pq;
                    const float kx = __uint_as_float(kw << 16), ky = __uint_as_float(kw & 0xffff0000u);
                    const float qx = __uint_as_float(qw << 16), qy = __uint_as_float(qw & 0xffff0000u);
                    // KD, QD = . e^{G - off}
                    *pk = bf2(kx * e0, ky * e1);
                    *pq = bf2(qx * e0, qy * e1);
                    // KE = K e^{end - G};  Kt = K e^{G_C - G} = KE e^{G_C - end}
                    const float ke0 = kx * ee0, ke1 = ky * ee1;
                    *reinterpret_cast<uint32_t *>(kxc + ac * 8192 + o) = bf2(ke0 * tc0, ke1 * tc1);
                    // B_rq = K e^{off_rq - G} (<= e^{kMaxNegLogDecay}; flagged channels 0),
                    // B_i = K e^{off_i - G} = KE e^{off_i - end} for the later blocks i
                    *reinterpret_cast<uint32_t *>(sm + L_BREG + ac * BREG_AC + sw128(di_col(rq) + r, cc >> 3) + cof) =
                        bf2(kx * de0, ky * de1);
#pragma unroll
                    for (int bi = 1; bi < 4; ++bi) {
                        if (bi <= rq) continue;  // rq is uniform per warp
                        *reinterpret_cast<uint32_t *>(sm + L_BREG + ac * BREG_AC + sw128(di_col(bi) + r, cc >> 3) + cof) =
                            bf2(ke0 * tb0[bi], ke1 * tb1[bi]);
                    }
                }
                fence_proxy_async_smem();
                // (every read of the staging count is behind a barrier by now)
                if (gtid < 4) reinterpret_cast<volatile uint32_t *>(kst_cnt)[gtid] = 0u;
                if (named_bar_or(BAR_G, 256, *abort_flag)) break;
                if (issuer) mbar_arrive(bars + LB_GATE);
            }
        }
        for (int m = g; active && m < nchunks; m += mstep) {
            const int gi = CH ? m : m >> 1;  // index of the chunk within the group
            const int rs = m % NRING;        // its ring slot
            uint8_t *ring_slot = ring_pair + (size_t)rs * RING_STRIDE;
            float *gr = gate_rows(m);
            uint8_t *kxc = (CH && (gi & 1)) ? sm + L_KX2 : kxt;  // this chunk's Kt
            uint8_t *rawp = raw_of(m);
            const uint32_t raw_s = smem_u32(rawp);
            const uint64_t d_raw = desc_sw128(raw_s, 16, 1024);        // [K;Q], K (K-major)
            const uint64_t d_kmn = desc_sw128(raw_s, L_RAW_AC, 1024);  // K (MN-major)
            const long long t0 = t_begin + (long long)m * C;
            const int L = chunk_len(m);
            bool ok = true;
            // ---- this chunk's tiles (rows past the sequence end read as zero); the
            //      tiles of the next chunk this group's storer loads are fetched into
            //      L2 meanwhile (KDA: m + 2; GDN: m + 3).  The previous chunk's ring
            //      tiles must have been read out of shared memory.
            if (issuer && m + (CH ? 2 : 3) < nchunks) {
                const int t2 = (int)(t0 + (CH ? 2 : 3) * C);
                tma_prefetch_l2_3d(&tm_k, 0, h, t2);
                tma_prefetch_l2_3d(&tm_k, 64, h, t2);
                tma_prefetch_l2_3d(&tm_q, 0, h, t2);
                tma_prefetch_l2_3d(&tm_q, 64, h, t2);
            }
            if constexpr (CH) {
                // KDA: the gate group has prepared KD, QD, Kt, B and the tables
                if (issuer) ok = wt.wait(bars + LB_GATE, (uint32_t)(m & 1));
            } else {
                if (issuer) ok = wt.wait(bars + LB_TMA + rbuf(m), tma_phase(m));
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
                }
            }
            // GDN with a full chunk: nothing to publish, so the MMA goes out as soon as
            // the tiles are in (the storer may still be issuing the previous chunk's
            // ring stores); an abort is seen at the barrier after it
            if (CH || L < C) {
                fence_proxy_async_smem();
                if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
            }
            // ---- D_kq = [K; Q] K^T (GDN) or [KD; QD] [B_0; B_1; B_2; B_3]^T (KDA) -------
            if (issuer && ok) {
                tc_fence_after();
                if constexpr (CH) {
                    const uint64_t db = desc_sw128(sbase + L_BREG, 16, 1024);
#pragma unroll
                    for (int k = 0; k < DK / 16; ++k) {
                        const uint32_t offa = ((k >> 2) * L_RAW_AC + (k & 3) * 32) >> 4;
                        const uint32_t offb = ((k >> 2) * BREG_AC + (k & 3) * 32) >> 4;
                        mma_bf16(tmem + TM_KD, d_raw + offa, db + offb, ID_KD, k > 0);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < DK / 16; ++k) {
                        const uint32_t off = ((k >> 2) * L_RAW_AC + (k & 3) * 32) >> 4;
                        mma_bf16(tm_kq, d_raw + off, d_raw + off, ID_KK, k > 0);
                    }
                }
                mma_commit(bar_l);
                ok = wt.wait(bar_l, bl_wait & 1);
            }
            ++bl_wait;
            // the tiles that the A/P phase below rewrites (and, KDA, the gate group's
            // Kt and e^{G_C}) went out first, as their own bulk group
            if (storer && pend) bulk_wait_read_but_last();
            // GDN: the raw buffer of this group's previous chunk (m - 2, Kt in place of K
            // read by its ring stores) takes chunk m + 1, the other group's next
            if (!CH && storer && m >= 2 && m + 1 < nchunks) issue_tma(m + 1);
            if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
            // KDA: the B region and the previous chunk's ring sources are free for the
            // gate pass of chunk m + 1
            if (CH && issuer) mbar_arrive(bars + LB_BFREE);
            tc_fence_after();
            // ---- A rows (lanes 0-63) -> fp32;  P rows (lanes 64-127) -> bf16.  GDN
            //      applies the decay here; KDA's product already carries it.
            const float *gb = gr + (CH ? GR_KB : GR_B);
            if ((lq & 1) >= lhalf) {
                float x[32];
                if constexpr (CH) {
                    // rows of block b0 (lanes 0-15) / b1 (lanes 16-31) from D_b0 / D_b1,
                    // whose first 16 (b + 1) columns are the decayed products
                    const int b0 = 2 * (lq & 1), b1 = b0 + 1;
                    float x1[32];
                    tmem_load<32>(tmem + TM_KD + di_col(b0) + lane_off + 32 * lhalf, x);
                    tmem_load<32>(tmem + TM_KD + di_col(b1) + lane_off + 32 * lhalf, x1);
                    const bool hi = lane >= 16;
                    const int nb = 16 * ((hi ? b1 : b0) + 1);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int s2 = 32 * lhalf + j;
                        x[j] = s2 < nb ? (hi ? x1[j] : x[j]) : 0.f;
                    }
                    // the exact diagonal-block terms of the fast-decaying channels
                    const float *cor = kcor_of(m);
                    if (*reinterpret_cast<const volatile int *>(cor + KCOR_FLAG)) {
                        const int rr = 32 * (lq & 1) + lane, bb = rr >> 4, il = rr & 15;
                        const float *ct = cor + (2 * bb + (lq >= 2 ? 1 : 0)) * KCOR_TRI + il * (il + 1) / 2;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int s2 = 32 * lhalf + j;
                            if ((s2 >> 4) == bb && (s2 & 15) <= il) x[j] += ct[s2 & 15];
                        }
                    }
                } else {
                    tmem_load<32>(tm_kq + lane_off + 32 * lhalf, x);
                }
                if (lq < 2) {
                    const int r = 32 * lq + lane;
                    if constexpr (!CH) decay_row(x, r, lq, lhalf, gr, false);
                    const float br = gb[r];
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        float y[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int s = 32 * lhalf + j + e;
                            y[e] = (CH && s >= r) ? 0.f : br * x[j + e];
                        }
                        *reinterpret_cast<float4 *>(AT + r * LDA + 32 * lhalf + j) = make_float4(y[0], y[1], y[2], y[3]);
                    }
                } else {
                    const int r = 32 * (lq - 2) + lane;
                    if constexpr (!CH) {
                        decay_row(x, r, lq - 2, lhalf, gr, true);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (32 * lhalf + j > r) x[j] = 0.f;
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<uint4 *>(pzt + PZ_P + sw128(r, 4 * lhalf + j)) = pack8(x + 8 * j);
                }
            } else if (lq >= 2) {
                // P rows 0-31, columns 32-63 (above the diagonal): zero; the tile
                // held ring tiles since the last chunk
#pragma unroll
                for (int j = 4; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(pzt + PZ_P + sw128(lane, j)) = make_uint4(0, 0, 0, 0);
            }
            named_bar_sync(BAR_G, 256);
            if (g == 0 && m == 0 && issuer) mbar_arrive(bars + LB_OFFSET);
            // ---- T = (I + A)^{-1} in place of A: lw 0-3 (diagonal blocks, 32-level);
            //      meanwhile lw 4 prepares the group's next GDN gates, and for KDA
            //      lw 4-7 form W's operand Kg from KD ----------------------------------
            if (lw >= 4) {
                if (storer && pend) hand_over();  // the previous chunk of this group
                if constexpr (!CH) {
                    if (lw == 4 && m + 2 < nchunks) compute_gates(m + 2);
                } else {
                    // Kg = K e^{G} = KD e^{G_{m(r)}} in place of KD (its products are done)
                    const float *fm = ktab_of(m) + 512;
#pragma unroll 2
                    for (int q2 = 0; q2 < 8; ++q2) {
                        const int idx = (gtid - 128) + 128 * q2;
                        const int ac = idx >> 9, rr = (idx >> 3) & 63, j = idx & 7;
                        float kv[8];
                        unpack8(*reinterpret_cast<const uint4 *>(rawp + ac * L_RAW_AC + sw128(rr, j)), kv);
                        const float *f = fm + 128 * (rr >> 4) + 64 * ac + 8 * j;
                        const float4 d0 = *reinterpret_cast<const float4 *>(f);
                        const float4 d1 = *reinterpret_cast<const float4 *>(f + 4);
                        kv[0] *= d0.x; kv[1] *= d0.y; kv[2] *= d0.z; kv[3] *= d0.w;
                        kv[4] *= d1.x; kv[5] *= d1.y; kv[6] *= d1.z; kv[7] *= d1.w;
                        *reinterpret_cast<uint4 *>(rawp + ac * L_RAW_AC + sw128(rr, j)) = pack8(kv);
                    }
                }
            } else {
                // (1) 16x16 diagonal blocks: warp lw inverts block lw; lane j < 16
                //     owns column j, then writes it over the block once the warp has
                //     read all of A's block.  GDN: right-looking forward substitution
                //     (measured faster there); KDA: left-looking with row loads.
                if (lane < 16) {
                    if constexpr (CH) {
                        invert_diag16(AT, 16 * lw, lane);
                    } else {
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
                }
                named_bar_sync(BAR_INV, 128);
                // (2) 32x32 halves: T_10 = -T_11 (A_10 T_00), T_32 = -T_33 (A_32 T_22);
                //     X goes to the unused upper-right 16x16 block of the half, T_10
                //     over A_10 once both warps of the half have read A_10.
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
            }
            if (named_bar_or(BAR_G, 256, *abort_flag)) break;
            // (3) T_{H1,H0} = -T_{H1} (A_{H1,H0} T_{H0}), 32x32 blocks; warp lw owns
            //     output rows 16(lw/4).., columns 8(lw%4)..; X goes to the unused
            //     upper-right block, the masked upper triangles hold scratch; the
            //     result replaces A_{H1,H0} after the barrier.
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
                    const int r = m0 + fg, kc = 8 * ks + ft;  // within H1
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
            // ---- T_b (and GDN's T_bg) in bf16, K-major rows r, columns s ----------
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                const int idx = gtid + 256 * q2, r = idx & 63, j = idx >> 6;  // lanes: rows
                float tv[8], bv[8], tb[8];
                *reinterpret_cast<float4 *>(tv) = *reinterpret_cast<const float4 *>(AT + r * LDA + 8 * j);
                *reinterpret_cast<float4 *>(tv + 4) = *reinterpret_cast<const float4 *>(AT + r * LDA + 8 * j + 4);
                *reinterpret_cast<float4 *>(bv) = *reinterpret_cast<const float4 *>(gb + 8 * j);
                *reinterpret_cast<float4 *>(bv + 4) = *reinterpret_cast<const float4 *>(gb + 8 * j + 4);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s2 = 8 * j + e;
                    tv[e] = s2 < r ? tv[e] : (s2 == r ? 1.f : 0.f);
                    tb[e] = tv[e] * bv[e];
                }
                if constexpr (!CH) {
                    float gv[8], tg[8];
                    *reinterpret_cast<float4 *>(gv) = *reinterpret_cast<const float4 *>(gr + GR_BG + 8 * j);
                    *reinterpret_cast<float4 *>(gv + 4) = *reinterpret_cast<const float4 *>(gr + GR_BG + 8 * j + 4);
#pragma unroll
                    for (int e = 0; e < 8; ++e) tg[e] = tv[e] * gv[e];
                    *reinterpret_cast<uint4 *>(pzt + PZ_X3 + sw128(r, j)) = pack8(tb);
                    *reinterpret_cast<uint4 *>(pzt + PZ_X1 + sw128(r, j)) = pack8(tg);
                } else {
                    *reinterpret_cast<uint4 *>(pzt + PZ_X1 + sw128(r, j)) = pack8(tb);
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(BAR_G, 256);
            // ---- D_ab = [P; 0] [T_bg | T_b] (GDN: rows 0-63 = [P T_bg | R]) or
            //      [P; 0] T_b (KDA: rows 0-63 = R) ------------------------------------
            if (issuer) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tm_ab, d_pz + 2 * k, d_x1b + 128 * k, CH ? ID_N64 : ID_N128, k > 0);
                mma_commit(bar_l);
                ok = wt.wait(bar_l, bl_wait & 1);
            }
            ++bl_wait;
            if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
            tc_fence_after();
            // GDN: lw 0,1 P T_bg -> X2, lw 4,5 R -> P's tile (P is consumed);
            // KDA: R -> X2, columns 32 lhalf .. by lw 0,1 and 4,5
            if (lq < 2) {
                const int r = 32 * lq + lane;
                if constexpr (CH) {
                    float x[32];
                    tmem_load<32>(tm_ab + lane_off + 32 * lhalf, x);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<uint4 *>(pzt + PZ_X2 + sw128(r, 4 * lhalf + j)) = pack8(x + 8 * j);
                } else {
                    uint8_t *dst = pzt + (lhalf == 0 ? PZ_X2 : PZ_P);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float x[32];
                        tmem_load<32>(tm_ab + lane_off + 64 * lhalf + 32 * hh, x);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(dst + sw128(r, 4 * hh + j)) = pack8(x + 8 * j);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(BAR_G, 256);
            // ---- D_ab = [X1; X2] K: GDN [T_bg; P T_bg] K, KDA [T_b; R] Kg:
            //      rows 0-63 = W, rows 64-127 = P W ---------------------------------------
            if (issuer) {
                tc_fence_after();
                const uint64_t dkb = d_kmn;  // GDN K, KDA Kg (MN-major)
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tm_ab, d_x1x2 + 2 * k, dkb + 128 * k, ID_N128, k > 0);
                mma_commit(bar_l);
                ok = wt.wait(bar_l, bl_wait & 1);
            }
            ++bl_wait;
            if (named_bar_or(BAR_G, 256, !ok || *abort_flag)) break;
            tc_fence_after();
            // ---- -W (lanes 0-63) staged in T's tile; Qh = gamma Q - P W (GDN) or
            //      Qg - P W (KDA) (lanes 64-127) staged in X1/X2 (GDN) or X3/P (KDA);
            //      GDN Kt = kh . K staged in KX.  The raw tiles are then free.
            {
                const int r = 32 * (lq & 1) + lane;
                const float gam = CH ? 1.f : gr[GR_GAM + r];
                uint8_t *wst = grp + LY::AT + lhalf * 8192;
                uint8_t *qst = pzt + (CH ? (lhalf ? PZ_P : PZ_X3) : (lhalf ? PZ_X2 : PZ_X1));
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
                            if constexpr (CH) {  // QD e^{G_{m(r)}}
                                const float *f = ktab_of(m) + 512 +
                                                 128 * (r >> 4) + 64 * lhalf + 8 * (4 * hh + j);
                                const float4 d0 = *reinterpret_cast<const float4 *>(f);
                                const float4 d1 = *reinterpret_cast<const float4 *>(f + 4);
                                qv[0] *= d0.x; qv[1] *= d0.y; qv[2] *= d0.z; qv[3] *= d0.w;
                                qv[4] *= d1.x; qv[5] *= d1.y; qv[6] *= d1.z; qv[7] *= d1.w;
                            }
#pragma unroll
                            for (int e = 0; e < 8; ++e) qv[e] = gam * qv[e] - x[8 * j + e];
                            *reinterpret_cast<uint4 *>(qst + o) = pack8(qv);
                        }
                    }
                }
                if constexpr (!CH) {
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const int idx = gtid + 256 * q2;
                        const int ac = idx >> 9, rr = (idx >> 3) & 63, j = idx & 7;
                        float kv[8];
                        unpack8(*reinterpret_cast<const uint4 *>(rawp + ac * L_RAW_AC + sw128(rr, j)), kv);
                        const float sc = gr[GR_KH + rr];
#pragma unroll
                        for (int e = 0; e < 8; ++e) kv[e] *= sc;
                        *reinterpret_cast<uint4 *>(rawp + ac * L_RAW_AC + sw128(rr, j)) = pack8(kv);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (named_bar_or(BAR_G, 256, *abort_flag)) break;
            if (storer) {
                // KDA: the raw tiles take chunk m + 2 (issued before the ring stores:
                // the TMA unit serves its requests in order)
                if (CH && m + 2 < nchunks) issue_tma(m + 2);
                // once the state CTA has read the slot's previous chunk, the ring
                // tiles and e^{G_C} go out by bulk copy; the hand-off follows
                // during the next chunk (or after the loop)
                if (m < NRING || wt.wait_peer(bars + LB_SLOTFREE + rs, (uint32_t)(((m / NRING) - 1) & 1))) {
                    // two bulk groups: first what the next chunk of this group rewrites
                    // early (the A/P phase: -W's staging in A's space, the P tile; the
                    // raw buffer's Kt, GDN; the gate group's Kt and e^{G_C}, KDA), then
                    // the rest (rewritten from the T_b phase on, after the hand-off
                    // has waited for every store)
                    const uint8_t *at8 = grp + LY::AT;
                    const uint8_t *kts = CH ? kxc : rawp;  // GDN: Kt in place of K
                    bulk_store(ring_slot + SG_KT, kts, 8192);
                    bulk_store(ring_slot + SG_AC + SG_KT, kts + (CH ? 8192 : L_RAW_AC), 8192);
                    bulk_store(ring_slot + SG_MW, at8, 8192);
                    bulk_store(ring_slot + SG_AC + SG_MW, at8 + 8192, 8192);
                    bulk_store(ring_slot + SG_TILES, gr + GR_DEC, SG_DECB);
                    if constexpr (CH) {
                        bulk_store(ring_slot + SG_AC + SG_QH, pzt + PZ_P, 8192);
                    } else {
                        bulk_store(ring_slot + SG_R, pzt + PZ_P, 8192);
                    }
                    bulk_commit();
                    if constexpr (CH) {
                        bulk_store(ring_slot + SG_QH, pzt + PZ_X3, 8192);
                        bulk_store(ring_slot + SG_R, pzt + PZ_X2, 8192);
                    } else {
                        bulk_store(ring_slot + SG_QH, pzt + PZ_X1, 8192);
                        bulk_store(ring_slot + SG_AC + SG_QH, pzt + PZ_X2, 8192);
                    }
                    bulk_store(ring_slot + SG_TB, pzt + (CH ? PZ_X1 : PZ_X3), 8192);
                    bulk_commit();
                    pend = true;
                    pend_slot = rs;
                }
            }
        }
        if (active && storer && pend && !*abort_flag) hand_over();
        // drain: every MMA this issuer launched, every tile load not yet landed
        if (storer) bulk_wait_all();
        if (*abort_flag && issuer) {
            mma_commit(bars + LB_DRAIN + g);
            mbar_wait(bars + LB_DRAIN + g, 0, kWaitLimit);
        }
    } else if (slot >= 0) {
        // ============================ state CTA ============================
        if (warp < 8) {
            // ---- chain of value half hv: warps 4hv..4hv+3, thread = key channel c
            const int hv = warp >> 2, q = warp & 3, c = 32 * q + lane;
            const int BAR_H = 1 + hv;
            const bool leader = (tid & 127) == 0;
            const uint32_t lane_off = (uint32_t)(32 * q) << 16;
            uint8_t *sb = sm + S_OFF_SB + hv * 16384;
            uint8_t *vp = sm + S_OFF_VP + hv * 8192;
            const uint64_t d_rtb = desc_sw128(sbase + SG_R, 16, 1024);
            const uint64_t d_v = desc_sw128(sbase + SG_V + 8192 * hv, 8192, 1024);
            const uint64_t d_qw = desc_sw128(sbase + SG_QH, 16, 1024);
            const uint64_t d_sb = desc_sw128(sbase + S_OFF_SB + hv * 16384, 16384, 1024);
            const uint64_t d_kt = desc_sw128(sbase + SG_KT, SG_AC, 1024);
            const uint64_t d_vp = desc_sw128(sbase + S_OFF_VP + hv * 8192, 8192, 1024);
            const uint32_t tm_ds = tmem + TM_DS + 64 * hv;
            float s_reg[64];
#pragma unroll
            for (int i = 0; i < 64; ++i)
                s_reg[i] = a.s0 ? a.s0[st_base + (size_t)(64 * hv + i) * DK + c] : 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(sb + sw128(c, j)) = pack8(s_reg + 8 * j);
            fence_proxy_async_smem();
            // D_vo[st] = [R; T_b] V_h  (needs the chunk's stage and D_vo free)
            auto issue_v = [&](int m) {
                const uint32_t so = (m & 1) * (S_STAGE >> 4);
                const uint32_t tm_vo = tmem + 64 * (2 * (m & 1) + hv);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tm_vo, d_rtb + so + 2 * k, d_v + so + 128 * k, ID_N64, k > 0);
            };
            bool v_issued = false;
            named_bar_sync(BAR_H, 128);
            for (int m = 0; m < nchunks; ++m) {
                const int st = m & 1, it = m >> 1;
                const uint32_t so = st * (S_STAGE >> 4);
                const uint32_t tm_vo = tmem + 64 * (2 * st + hv);
                bool ok = true;
                if (leader) {
                    if (!v_issued) {
                        ok = wt.wait(bars + SB_FULL + st, (uint32_t)(it & 1));
                        if (ok && m >= 2) ok = wt.wait(bars + SB_OFREE + 2 * st + hv, (uint32_t)((it - 1) & 1));
                        if (ok) {
                            tc_fence_after();
                            issue_v(m);
                        }
                    }
                    // D_vo += [Qh; -W] S_h^T
                    if (ok) {
#pragma unroll
                        for (int k = 0; k < DK / 16; ++k) {
                            const uint32_t off = ((k >> 2) * SG_AC + (k & 3) * 32) >> 4;
                            mma_bf16(tm_vo, d_qw + so + off, d_sb + 128 * k, ID_N64, 1);
                        }
                        mma_commit(bars + SB_VO + hv);
                    }
                }
                v_issued = false;
                // every chain warp sees the stage through the completed product, then
                // takes this chunk's decay of its key channel; the V' warps (lanes
                // 64-127) write V' as bf16, MN-major [r][i]
                float dec = 0.f;
                // (the leader's result reaches its whole warp before the warp-wide
                // wait, so that every lane takes the same branch)
                const bool okv = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 &&
                                 wt.warp_wait(bars + SB_VO + hv, (uint32_t)(m & 1), lane);
                if (okv) {
                    dec = reinterpret_cast<const float *>(sm + st * S_STAGE + SG_DEC)[c];
                    if (q >= 2) {
                        tc_fence_after();
                        const int r = 32 * (q - 2) + lane;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float x[32];
                            tmem_load<32>(tm_vo + lane_off + 32 * hh, x);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                *reinterpret_cast<uint4 *>(vp + sw128(r, 4 * hh + j)) = pack8(x + 8 * j);
                        }
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                if (named_bar_or(BAR_H, 128, !okv || *abort_flag)) break;
                if (leader) {
                    tc_fence_after();
                    // dS_h = Kt^T V'_h
#pragma unroll
                    for (int k = 0; k < C / 16; ++k)
                        mma_bf16(tm_ds, d_kt + so + 128 * k, d_vp + 128 * k, ID_MM, k > 0);
                    mma_commit(bars + SB_DS + hv);
                    mma_commit(bars + SB_CONS + st);
                    // the next chunk's V product, if its stage is already there
                    if (m + 1 < nchunks) {
                        const int st1 = (m + 1) & 1, it1 = (m + 1) >> 1;
                        if (mbar_try_wait(bars + SB_FULL + st1, (uint32_t)(it1 & 1)) &&
                            (m + 1 < 2 ||
                             mbar_try_wait(bars + SB_OFREE + 2 * st1 + hv, (uint32_t)((it1 - 1) & 1)))) {
                            tc_fence_after();
                            issue_v(m + 1);
                            v_issued = true;
                        }
                    }
                }
                // S_h <- S_h Diag(e^{G_C}) + dS_h  (thread c: column c)
                const bool okd = wt.warp_wait(bars + SB_DS + hv, (uint32_t)(m & 1), lane);
                if (okd) {
                    tc_fence_after();
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float ds[32];
                        tmem_load<32>(tm_ds + lane_off + 32 * hh, ds);
#pragma unroll
                        for (int i = 0; i < 32; ++i) s_reg[32 * hh + i] = dec * s_reg[32 * hh + i] + ds[i];
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4 *>(sb + sw128(c, j)) = pack8(s_reg + 8 * j);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                if (named_bar_or(BAR_H, 128, !okd || *abort_flag)) break;
            }
            if (*abort_flag) {
                if (leader) {  // every MMA this leader launched
                    mma_commit(bars + SB_DRAIN + hv);
                    mbar_wait(bars + SB_DRAIN + hv, 0, kWaitLimit);
                }
            } else if (a.s_final) {
#pragma unroll
                for (int i = 0; i < 64; ++i) a.s_final[st_base + (size_t)(64 * hv + i) * DK + c] = s_reg[i];
            }
        } else if (warp == 8 || warp == 9 || warp == 12 || warp == 13) {
            // ---- output rows of value half hv (lanes 0-63 of D_vo) ----------------
            const int hv = (warp >> 2) & 1, q = warp & 1;
            const int BAR_O = 3 + hv;
            const uint32_t lane_off = (uint32_t)(32 * q) << 16;
            const int r = 32 * q + lane;
            for (int m = 0; m < nchunks; ++m) {
                const int st = m & 1;
                const bool ok = wt.warp_wait(bars + SB_VO + hv, (uint32_t)(m & 1), lane);
                if (ok) {
                    tc_fence_after();
                    const long long t0 = t_begin + (long long)m * C;
                    const int L = chunk_len(m);
                    __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.o) +
                                         ((t0 + r) * H + h) * (long long)DV + 64 * hv;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float x[32];
                        tmem_load<32>(tmem + 64 * (2 * st + hv) + lane_off + 32 * hh, x);
                        if (r < L) {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                reinterpret_cast<uint4 *>(dst)[4 * hh + j] = pack8(x + 8 * j);
                        }
                    }
                }
                tc_fence_before();
                if (named_bar_or(BAR_O, 64, !ok || *abort_flag)) break;
                if (q == 0 && lane == 0) mbar_arrive(bars + SB_OFREE + 2 * st + hv);
            }
        } else if (warp == 10 && lane == 0) {
            // ---- loader: ring slot + V tiles of each chunk into its stage ----------
            const uint32_t peer_slotfree = map_peer(smem_u32(bars), peer);  // + 8 * (LB_SLOTFREE + st)
            for (int m = 0; m < nchunks; ++m) {
                const int st = m & 1, it = m >> 1;
                uint8_t *stage = sm + st * S_STAGE;
                bool ok = true;
                if (m >= 2) ok = wt.wait(bars + SB_CONS + st, (uint32_t)((it - 1) & 1));
                const int rs = m % NRING;
                if (ok) ok = wt.wait_peer(bars + SB_READY + rs, (uint32_t)((m / NRING) & 1));
                if (!ok) break;
                fence_proxy_async_global();
                const uint8_t *src = ring_pair + (size_t)rs * RING_STRIDE;
                const long long t0 = t_begin + (long long)m * C;
                mbar_arrive_expect_tx(bars + SB_FULL + st, S_STAGE_TX);
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    bulk_load(stage + p * 16384, src + p * 16384, 16384, bars + SB_FULL + st);
                bulk_load(stage + SG_DEC, src + SG_TILES, SG_DECB, bars + SB_FULL + st);
                tma_load_3d(stage + SG_V, &tm_v, 0, h, (int)t0, bars + SB_FULL + st);
                tma_load_3d(stage + SG_V + 8192, &tm_v, 64, h, (int)t0, bars + SB_FULL + st);
                ++issued[st];
                // the slot is read once the stage has landed: give it back
                if (!wt.wait(bars + SB_FULL + st, (uint32_t)(it & 1))) break;
                mbar_arrive_peer(peer_slotfree + 8 * (LB_SLOTFREE + rs));
            }
            if (*abort_flag)
                for (int st = 0; st < 2; ++st)
                    if (issued[st] > 0)
                        mbar_wait(bars + SB_FULL + st, (uint32_t)((issued[st] - 1) & 1), kWaitLimit);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag && slot >= 0) {
        atomicOr(a.err, kErrTimeout);
        // local CTA: every raw buffer's last tile load lands before the CTA exits
        // (both groups' storers load; all have left their loops here)
        if (rank == 0)
            for (int p = 0; p < 3; ++p)
                if (issued[p] > 0) mbar_wait(bars + LB_TMA + p, (uint32_t)((issued[p] - 1) & 1), kWaitLimit);
    }
    cluster_sync();  // no CTA leaves while its peer may still address its memory
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------- host --
// %nsmid: an upper bound of %smid on this device (which need not equal the SM
// count, nor the SM ids be contiguous).
__device__ int g_nsmid;
__global__ void nsmid_probe_kernel() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nsmid;" : "=r"(r));
    g_nsmid = (int)r;
}

// Ring slots: one per possible SM id, from %nsmid read once per device (the
// first call on a device launches a one-thread kernel on the legacy default
// stream and waits for it, so that call should come before any stream capture).
int ring_slots_for_device() {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static int slots[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (slots[dev] == 0) {
        int n = 0;
        nsmid_probe_kernel<<<1, 1>>>();
        if (cudaGetLastError() != cudaSuccess) return 0;
        if (cudaMemcpyFromSymbol(&n, g_nsmid, sizeof(int)) != cudaSuccess || n <= 0) return 0;
        slots[dev] = n;
    }
    return slots[dev];
}

size_t ring_bytes(int slots) { return (size_t)slots * NRING * RING_STRIDE; }

// Longest-first order of a packed batch's sequences (by chunk count; ties by
// index), for list scheduling of the clusters: thread i ranks sequence i among
// all of them from a shared-memory copy of the chunk counts.
constexpr int kOrderMax = 4096;  // larger batches keep the index order
__global__ void __launch_bounds__(1024) pair_order_kernel(const int32_t *cu, int n, int32_t *order) {
    __shared__ int nck[kOrderMax];
    for (int i = threadIdx.x; i < n; i += blockDim.x) nck[i] = (cu[i + 1] - cu[i] + C - 1) / C;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int ki = nck[i];
        int r = 0;
        for (int j = 0; j < n; ++j) {
            const int kj = nck[j];
            r += (kj > ki) | ((kj == ki) & (j < i));
        }
        order[r] = i;
    }
}

bool use_order(const PrefillArgs &a) { return a.cu_seqlens && a.n_seqs > 1 && a.n_seqs <= kOrderMax; }
size_t order_bytes(int n_seqs) { return ((size_t)n_seqs * sizeof(int32_t) + 255) & ~(size_t)255; }

template <bool CH>
cudaError_t launch_t(const PrefillArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                     const CUtensorMap &mv, int slots, cudaStream_t s) {
    auto kern = chunk_pair_kernel<CH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const long long items = (long long)a.n_seqs * a.H;
    uint8_t *ring = reinterpret_cast<uint8_t *>(a.scratch);
    const int32_t *order = use_order(a) ? reinterpret_cast<const int32_t *>(ring + ring_bytes(slots)) : nullptr;
    kern<<<(unsigned)(2 * items), kThreads, SMEM_BYTES, s>>>(a, mq, mk, mv, ring, slots, order);
    return cudaGetLastError();
}

}  // namespace

bool chunk_pair_supported(const gdn_dims &d) {
    return d.dtype == GDN_BF16 && d.d_k == DK && d.d_v == DV && (long long)d.B * d.T < (1LL << 31);
}

size_t chunk_pair_scratch_bytes(const gdn_dims &d) {
    // the ring, then (packed batches) the sequences' longest-first order
    return ring_bytes(ring_slots_for_device()) + (d.n_seqs > 1 ? order_bytes(d.n_seqs) : 0);
}

cudaError_t launch_chunk_pair(const PrefillArgs &a, cudaStream_t s, int *launches) {
    const long long items = (long long)a.n_seqs * a.H;
    const long long ntok = (long long)a.B * a.T;
    if (items == 0) return cudaSuccess;
    if (ntok == 0) {
        if (a.s_final && a.s_final != a.s0) {
            const size_t bytes = (size_t)a.n_seqs * a.H * a.dv * a.dk * sizeof(float);
            return a.s0 ? cudaMemcpyAsync(a.s_final, a.s0, bytes, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(a.s_final, 0, bytes, s);
        }
        return cudaSuccess;
    }
    CUtensorMap mq, mk, mv;
    if (!make_tile_map(&mq, a.q, a.dk, a.H, ntok) || !make_tile_map(&mk, a.k, a.dk, a.H, ntok) ||
        !make_tile_map(&mv, a.v, a.dv, a.H, ntok))
        return cudaErrorInvalidValue;
    const int slots = ring_slots_for_device();
    if (slots <= 0) return cudaErrorInvalidValue;
    if (use_order(a)) {
        pair_order_kernel<<<1, 1024, 0, s>>>(
            a.cu_seqlens, a.n_seqs,
            reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(a.scratch) + ring_bytes(slots)));
        const cudaError_t eo = cudaGetLastError();
        if (eo != cudaSuccess) return eo;
        if (launches) ++*launches;
    }
    cudaError_t e = a.channel ? launch_t<true>(a, mq, mk, mv, slots, s)
                              : launch_t<false>(a, mq, mk, mv, slots, s);
    if (e != cudaSuccess) return e;
    if (launches) ++*launches;
    return e;
}

}  // namespace gdn

// gdn_chunk_tc.cu -- chunkwise gated delta rule prefill on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators, TMA-staged 128B-swizzled bf16
// tiles) for bf16 inputs with d_k = d_v = 128 and scalar (GDN) decay.
//
// One CTA per (sequence, head, 64-wide slice of d_v), walking the sequence's
// chunks of C = 64 tokens (FG2-GDN paper, section 3.6: WY representation and
// UT transform inside a chunk, inter-chunk state propagation, intra-chunk
// causal product; the Gated Delta Networks page, section 3.3, for the scalar
// cumulative decay g_r, gamma_r = e^{g_r}).  Per chunk:
//
//   D_kq  = [K; Q] K^T                  rows 0-63: K K^T, rows 64-127: Q K^T
//   A_rs  = beta_r e^{g_r-g_s} (K K^T)_rs, s < r;  P_rs = e^{g_r-g_s} (Q K^T)_rs, s <= r
//   T     = (I + A)^{-1}                 blocked forward substitution (fp32, tf32 MMAs)
//   T_b   = T diag(beta),  T_bg = T diag(beta gamma)       (bf16)
//   D_w   = [T_bg; 0] K                  rows 0-63: W = T diag(beta)(gamma . K)
//   D_vp  = [0; T_b] V                   rows 64-127: U = T diag(beta) V
//   D_vp += [Q; -W] S^T                  rows 0-63: Q S^T; rows 64-127: V' = U - W S^T
//   D_ds  = K^T (kh . V'),  kh_s = e^{g_C-g_s}            (the decayed-key write)
//   D_o   = [P; 0] V'
//   o_r   = gamma_r (Q S^T)_r + (P V')_r,   S <- e^{g_C} S + D_ds^T
//
// Warp roles (384 threads):
//   warps 0-7  "local": the work that depends only on the chunk's own tokens
//              (D_kq, A, T, W, U, P), one chunk ahead of the state warps;
//   warps 8-11 "state": the sequential pass (the three S-dependent MMAs, the
//              fp32 state in registers -- thread c holds column c of the
//              state slice -- the output, and the next tile loads).
// Tiles arrive by TMA into a two-stage ring; stage layout per 64-column atom:
// [K rows 0-63 | Q rows | -W rows], so [K; Q] and [Q; -W] are both contiguous
// M = 128 operands and the raw K tile also serves as an MN-major operand.
// Every wait is bounded: on expiry the kernel records kErrTimeout, both groups
// leave their loops at the next barrier, in-flight copies and MMAs are drained
// (again with a bound) and TMEM is freed.
#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = kChunk;       // 64
constexpr int DK = 128;
constexpr int DVS = 64;         // d_v slice per CTA
constexpr int kLocal = 256;     // threads of the local group
constexpr int kState = 128;     // threads of the state group
constexpr int kThreads = kLocal + kState;
constexpr int BAR_LOCAL = 1, BAR_STATE = 2, BAR_INV = 3;  // named barrier ids
constexpr long long kWaitLimit = kDefaultWaitLimit;  // drains after an abort
constexpr int LDA = 68;         // fp32 row stride of A and T in smem

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t RAW_STAGE = 57344;    // one stage: 2 atom columns + V
constexpr uint32_t RAW_AC = 24576;       //   atom column: [K 64 rows][Q 64 rows][-W 64 rows]
constexpr uint32_t RAW_K = 0;
constexpr uint32_t RAW_Q = 8192;
constexpr uint32_t RAW_W = 16384;
constexpr uint32_t RAW_V = 49152;        //   V slice tile [64 rows][128 B]
constexpr uint32_t STAGE_LOAD_BYTES = 40960;  // Q, K (2 boxes each) and V per stage
constexpr uint32_t OFF_RAW = 0;          // stages 0 and 1
constexpr uint32_t OFF_TG = 114688;      // T diag(beta gamma) [64 rows][128 B]  } [T_bg; 0]
constexpr uint32_t OFF_Z = 122880;       // zeros                                } [0; T_b]
constexpr uint32_t OFF_TB = 131072;      // T diag(beta)
constexpr uint32_t OFF_P = 139264;       // P                                    } [P; 0]
constexpr uint32_t OFF_Z2 = 147456;      // zeros
constexpr uint32_t OFF_VP = 155648;      // V'        MN-major [64 rows r][64 i]
constexpr uint32_t OFF_VH = 163840;      // kh . V'   MN-major
constexpr uint32_t OFF_SB = 172032;      // S (bf16)  MN-major [128 rows c][64 i]
constexpr uint32_t OFF_AF = 188416;      // A fp32 [64][LDA]
constexpr uint32_t OFF_TF = OFF_AF + 64 * LDA * 4;   // T fp32 [64][LDA]
constexpr uint32_t OFF_ROW = OFF_TF + 64 * LDA * 4;  // per chunk parity: g, beta, beta e^g,
constexpr uint32_t ROW_STRIDE = 8 * 64 * 4;          // colf[64], rowf[64][4]
constexpr uint32_t OFF_HAND = OFF_ROW + 2 * ROW_STRIDE;  // per chunk parity: g[64], g_C
constexpr uint32_t HAND_STRIDE = 1024;
constexpr uint32_t OFF_BAR = OFF_HAND + 2 * HAND_STRIDE;
constexpr uint32_t SMEM_USED = OFF_BAR + 128;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // + alignment slack

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t COL_KQ = 0;    // 2 buffers x 64
constexpr uint32_t COL_W = 128;   // 128 columns
constexpr uint32_t COL_VP = 256;  // 2 buffers x 64
constexpr uint32_t COL_DS = 384;
constexpr uint32_t COL_O = 448;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);   // [K;Q] K^T
constexpr uint32_t ID_W = idesc_bf16(128, 128, false, true);    // [T_bg; 0] K
constexpr uint32_t ID_KM = idesc_bf16(128, 64, false, true);    // [0;T_b] V, [Q;-W] S^T, [P;0] V'
constexpr uint32_t ID_MM = idesc_bf16(128, 64, true, true);     // K^T (kh . V')

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

// Scale one thread's 32 entries (columns 32*half ..) of row r of a C x C
// product by the decay e^{g_r - g_s}, keeping s < r (strict) or s <= r.  Off
// the diagonal 16-blocks the decay is the product of the two block-boundary
// factors; only the row's own diagonal block takes exponentials.  Written
// without lane-dependent branches (rows of one warp span two blocks) so the
// independent load -> exp -> multiply chains overlap.
__device__ __forceinline__ void decay_row(float *x, int r, int rb, int half, const float *g,
                                          const float *colf, const float *rowf, bool incl) {
    const float gr = g[r];
    float d[16];
    if ((rb >> 1) == half) {  // uniform per warp: a warp's rows share rb >> 1
#pragma unroll
        for (int e = 0; e < 16; ++e) d[e] = __expf(gr - g[16 * rb + e]);
    } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) d[e] = 0.f;
    }
    const float f0 = rowf[4 * r + 2 * half], f1 = rowf[4 * r + 2 * half + 1];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int cb = 2 * half + (j >> 4);
        const int s = 32 * half + j;
        const float foff = (j < 16 ? f0 : f1) * colf[s];
        const bool keep = incl ? (s <= r) : (s < r);
        const float fd = (cb == rb && keep) ? d[j & 15] : 0.f;
        x[j] *= cb < rb ? foff : fd;
    }
}

// Called by one thread per group; the others sleep on a named barrier, so the
// polling does not compete with the busy warps for issue slots or the shared
// memory pipe.  No sleep between polls: mbarrier.try_wait suspends the thread
// for a while itself, and a sleep only delays the waiter (measured).
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort,
                                         long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            *abort = 1;
            return false;
        }
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base by pointer arithmetic on the shared array (an
    // integer round trip would lose the address space and turn every access
    // below into a generic one)
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    float *AF = reinterpret_cast<float *>(sm + OFF_AF);
    float *TF = reinterpret_cast<float *>(sm + OFF_TF);
    // Per-chunk gate rows (two buffers, by chunk parity):
    //   g (cumulative log decay), beta, beta e^{g}; and the decay between tokens
    //   r > s of different 16-token blocks, factored at the last token e of s's
    //   block: e^{g_r - g_s} = e^{g_r - g_e} e^{g_e - g_s}, both factors <= 1
    //   (no overflow, only the underflow the product has too):
    //   colf[s] = e^{g_e(s) - g_s},  rowf[r][b] = e^{g_r - g_{16b+15}}, b < r/16.
    auto gate_rows = [&](int st) { return reinterpret_cast<float *>(sm + OFF_ROW + st * ROW_STRIDE); };
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_tma = bars + 0;     // [2] tiles of a stage landed
    uint64_t *bar_l = bars + 2;       // local MMAs done
    uint64_t *bar_s = bars + 3;       // state MMAs done
    uint64_t *bar_vpfree = bars + 4;  // [2] a chunk's state pass is over (its buffers are free)
    uint64_t *bar_ready = bars + 6;   // a chunk's operands are ready for the state pass
    uint64_t *bar_pfree = bars + 7;   // the state pass has consumed P of a chunk
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 64);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_BAR + 68);
    const long long lim = data_wait_limit(a.err);  // data waits (the header can shorten it)
    int *tma_issued = reinterpret_cast<int *>(sm + OFF_BAR + 72);  // [2] loads issued per stage

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nsl = a.dv / DVS;
    const int item = blockIdx.x;
    const int slice = item % nsl;
    const int h = (item / nsl) % a.H;
    const int n = item / (nsl * a.H);
    const int v0 = slice * DVS;
    const int H = a.H;

    long long t_begin, t_end;
    seq_range(a, n, &t_begin, &t_end);
    const int nchunks = (int)((t_end - t_begin + C - 1) / C);
    const size_t st_base = ((size_t)n * H + h) * a.dv * DK;

    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(bars + i, 1);
        fence_mbar_init();
        *abort_flag = 0;
        tma_issued[0] = tma_issued[1] = 0;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    for (int i = tid; i < 512; i += kThreads) {
        reinterpret_cast<uint4 *>(sm + OFF_Z)[i] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4 *>(sm + OFF_Z2)[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();

    // the state group's registers: thread c holds S[v0 + i][c], i in [0, 64)
    float s_reg[DVS];
    const int c_st = tid - kLocal;  // state thread index = key channel
    if (tid >= kLocal) {
#pragma unroll
        for (int i = 0; i < DVS; ++i)
            s_reg[i] = a.s0 ? a.s0[st_base + (size_t)(v0 + i) * DK + c_st] : 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4 *>(sm + OFF_SB + sw128(c_st, j)) = pack8(s_reg + 8 * j);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto chunk_len = [&](int m) -> int {
        const long long rem = t_end - (t_begin + (long long)m * C);
        return rem < C ? (int)rem : C;
    };
    // Q, K and V tiles of chunk m into stage m % 2 (one thread).
    auto issue_tma = [&](int m) {
        const int st = m & 1;
        const long long t0 = t_begin + (long long)m * C;
        uint8_t *raw = sm + OFF_RAW + st * RAW_STAGE;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bar_tma[st], STAGE_LOAD_BYTES);
        tma_load_3d(raw + RAW_Q, &tm_q, 0, h, (int)t0, &bar_tma[st]);
        tma_load_3d(raw + RAW_AC + RAW_Q, &tm_q, 64, h, (int)t0, &bar_tma[st]);
        tma_load_3d(raw + RAW_K, &tm_k, 0, h, (int)t0, &bar_tma[st]);
        tma_load_3d(raw + RAW_AC + RAW_K, &tm_k, 64, h, (int)t0, &bar_tma[st]);
        tma_load_3d(raw + RAW_V, &tm_v, v0, h, (int)t0, &bar_tma[st]);
        ++tma_issued[st];
    };

    if (tid < kLocal) {
        // ============================ local group ============================
        const int lq = warp & 3, lhalf = warp >> 2;  // TMEM lane quadrant, column half
        const uint32_t lane_off = (uint32_t)(32 * lq) << 16;
        uint32_t bl_wait = 0, bl_commit = 0;  // completions waited on / committed to bar_l
        int tma_seen0 = 0, tma_seen1 = 0;
        // matrix descriptors: base per buffer, then + (byte offset >> 4) per K step;
        // stage 1 is stage 0 + RAW_STAGE bytes
        const uint64_t d_kq0 = desc_sw128(sbase + OFF_RAW + RAW_K, 16, 1024);
        const uint64_t d_kmn0 = desc_sw128(sbase + OFF_RAW + RAW_K, RAW_AC, 1024);
        const uint64_t d_vmn0 = desc_sw128(sbase + OFF_RAW + RAW_V, 8192, 1024);
        const uint64_t d_tg = desc_sw128(sbase + OFF_TG, 16, 1024);
        const uint64_t d_ztb = desc_sw128(sbase + OFF_Z, 16, 1024);

        // wait for chunk m's tiles, zero rows past the sequence end, issue D_kq.
        // The tile wait and the MMA issue (which blocks its thread for a few
        // hundred cycles) are done by `issuer`, a thread whose warp has nothing
        // else to do at that point.
        auto start_chunk = [&](int m, int issuer) -> bool {
            const int st = m & 1;
            bool ok = true;
            if (tid == issuer) ok = wait_bar(&bar_tma[st], (uint32_t)((st ? tma_seen1 : tma_seen0) & 1), abort_flag, lim);
            if (st) ++tma_seen1; else ++tma_seen0;
            const int L = chunk_len(m);
            if (L < C) {
                if (named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag)) return false;
                uint8_t *raw = sm + OFF_RAW + st * RAW_STAGE;
                for (int idx = tid; idx < (C - L) * 8; idx += kLocal) {
                    const int r = L + (idx >> 3), pj = idx & 7;
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    const uint32_t o = r * 128 + pj * 16;
                    *reinterpret_cast<uint4 *>(raw + RAW_Q + o) = z;
                    *reinterpret_cast<uint4 *>(raw + RAW_AC + RAW_Q + o) = z;
                    *reinterpret_cast<uint4 *>(raw + RAW_K + o) = z;
                    *reinterpret_cast<uint4 *>(raw + RAW_AC + RAW_K + o) = z;
                    *reinterpret_cast<uint4 *>(raw + RAW_V + o) = z;
                }
                fence_proxy_async_smem();
            }
            if (named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag)) return false;
            if (tid == issuer) {
                tc_fence_after();
                const uint64_t da = d_kq0 + st * (RAW_STAGE >> 4);
#pragma unroll
                for (int k = 0; k < DK / 16; ++k) {
                    const uint32_t off = ((k >> 2) * RAW_AC + (k & 3) * 32) >> 4;
                    mma_bf16(tmem + COL_KQ + 64 * st, da + off, da + off, ID_KK, k > 0);
                }
                mma_commit(bar_l);
            }
            ++bl_commit;
            return true;
        };

        // gates of a chunk, prefetched into warp 4's registers one chunk ahead
        float nla0 = 0.f, nla1 = 0.f, nbe0 = 0.f, nbe1 = 0.f;
        auto load_gates = [&](int m) {
            const long long t0 = t_begin + (long long)m * C;
            const int L = chunk_len(m), r0 = 2 * lane, r1 = 2 * lane + 1;
            nla0 = r0 < L ? a.log_alpha[(t0 + r0) * H + h] : 0.f;
            nla1 = r1 < L ? a.log_alpha[(t0 + r1) * H + h] : 0.f;
            nbe0 = r0 < L ? a.beta[(t0 + r0) * H + h] : 0.f;
            nbe1 = r1 < L ? a.beta[(t0 + r1) * H + h] : 0.f;
        };
        // gates of chunk mm (one warp): cumulative log decay, beta and the
        // factored block decays, into the gate rows of mm's parity
        auto compute_gates = [&](int mm) {
            const int st = mm & 1;
            float *g_s = gate_rows(st), *b_s = g_s + 64, *bg_s = g_s + 128;
            float *colf_s = g_s + 192, *rowf_s = g_s + 256;
            const int r0 = 2 * lane, r1 = 2 * lane + 1;
            const float la0 = nla0, la1 = nla1, be0 = nbe0, be1 = nbe1;
            if (mm + 1 < nchunks) load_gates(mm + 1);
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
            const int blk = r0 >> 4;
            const float e0 = __expf(g0), e1 = __expf(g1);
            const float c0 = __expf(gend[blk] - g0), c1 = __expf(gend[blk] - g1);
            float f0[3], f1[3];
#pragma unroll
            for (int b = 0; b < 3; ++b) {  // unconditional: no divergent exps
                f0[b] = __expf(fminf(g0 - gend[b], 0.f));
                f1[b] = __expf(fminf(g1 - gend[b], 0.f));
            }
            g_s[r0] = g0; g_s[r1] = g1;
            b_s[r0] = be0; b_s[r1] = be1;
            bg_s[r0] = be0 * e0; bg_s[r1] = be1 * e1;
            colf_s[r0] = c0; colf_s[r1] = c1;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                rowf_s[4 * r0 + b] = b < blk ? f0[b < 3 ? b : 0] : 0.f;
                rowf_s[4 * r1 + b] = b < blk ? f1[b < 3 ? b : 0] : 0.f;
            }
        };
        if (tid == 0) {
            if (nchunks > 0) issue_tma(0);
            if (nchunks > 1) issue_tma(1);
        }
        if (warp == 4 && nchunks > 0) {
            load_gates(0);
            compute_gates(0);
        }
        bool alive = nchunks > 0 ? start_chunk(0, 0) : true;

        for (int m = 0; alive && m < nchunks; ++m) {
            const int st = m & 1;
            uint8_t *raw = sm + OFF_RAW + st * RAW_STAGE;
            const float *g_s = gate_rows(st), *b_s = g_s + 64, *bg_s = g_s + 128;
            const float *colf_s = g_s + 192, *rowf_s = g_s + 256;
            bool ok = true;

            // ---- D_kq of this chunk ----------------------------------------------
            if (tid == 0) ok &= wait_bar(bar_l, bl_wait & 1, abort_flag, lim);
            ++bl_wait;
            if (named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag)) break;
            tc_fence_after();
            // A rows (K K^T: TMEM lanes 0-63, sub-partitions 0-1) and, at the same
            // time on sub-partitions 2-3, P rows (Q K^T: lanes 64-127), kept in
            // registers as bf16 until the state pass frees the P slot.
            uint4 p_hold[4];
            if (lq >= 2) {
                float x[32];
                tmem_load<32>(tmem + lane_off + COL_KQ + 64 * st + 32 * lhalf, x);
                const int r = 32 * (lq - 2) + lane;
                decay_row(x, r, r >> 4, lhalf, g_s, colf_s, rowf_s, true);
#pragma unroll
                for (int j = 0; j < 4; ++j) p_hold[j] = pack8(x + 8 * j);
            }
            if (lq < 2) {
                float x[32];
                tmem_load<32>(tmem + lane_off + COL_KQ + 64 * st + 32 * lhalf, x);
                const int r = 32 * lq + lane, br_blk = r >> 4;
                decay_row(x, r, br_blk, lhalf, g_s, colf_s, rowf_s, false);
                const float br = b_s[r];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 y = make_float4(br * x[j], br * x[j + 1], br * x[j + 2], br * x[j + 3]);
                    *reinterpret_cast<float4 *>(AF + r * LDA + 32 * lhalf + j) = y;
                }
            }
            named_bar_sync(BAR_LOCAL, kLocal);
            // ---- T = (I + A)^{-1} ------------------------------------------------
            // meanwhile warp 4 prepares the next chunk's gates (during the
            // diagonal blocks and the 32x32 level, which need warps 0-3 only)
            if (warp == 4 && m + 1 < nchunks) compute_gates(m + 1);
            // (1) 16x16 diagonal blocks: warp w < 4 inverts block w; lane j < 16
            //     owns column j.  Right-looking forward substitution: once t_m
            //     is final it is eliminated from every later row, so the chain
            //     of dependent operations is one FMA per row.
            if (warp < 4 && lane < 16) {
                const int o = 16 * warp, j = lane;
                float t[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) t[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
                for (int mm = 0; mm < 15; ++mm) {
#pragma unroll
                    for (int i = mm + 1; i < 16; ++i) t[i] -= AF[(o + i) * LDA + o + mm] * t[mm];
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) TF[(o + i) * LDA + o + j] = t[i];
            }
            if (warp < 4) named_bar_sync(BAR_INV, 128);
            const int fg = lane >> 2, ft = lane & 3;  // mma.sync fragment coordinates
            // (2) 32x32 halves: T_10 = -T_11 (A_10 T_00) and T_32 = -T_33 (A_32 T_22);
            //     warp w < 4: half w/2, 8 output columns (w%2).  X goes to the
            //     unused upper-right 16x16 block of the half.
            if (warp < 4) {
                const int o = 32 * (warp >> 1), n0 = 8 * (warp & 1);
                float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    uint32_t af[4], bf[2];
                    const int ar = o + 16 + fg, ac = o + 8 * ks + ft;
                    af[0] = to_tf32(AF[ar * LDA + ac]);
                    af[1] = to_tf32(AF[(ar + 8) * LDA + ac]);
                    af[2] = to_tf32(AF[ar * LDA + ac + 4]);
                    af[3] = to_tf32(AF[(ar + 8) * LDA + ac + 4]);
                    bf[0] = to_tf32(TF[(o + 8 * ks + ft) * LDA + o + n0 + fg]);
                    bf[1] = to_tf32(TF[(o + 8 * ks + ft + 4) * LDA + o + n0 + fg]);
                    mma_tf32_16x8x8(x, af, bf);
                }
                TF[(o + fg) * LDA + o + 16 + n0 + 2 * ft] = x[0];
                TF[(o + fg) * LDA + o + 16 + n0 + 2 * ft + 1] = x[1];
                TF[(o + fg + 8) * LDA + o + 16 + n0 + 2 * ft] = x[2];
                TF[(o + fg + 8) * LDA + o + 16 + n0 + 2 * ft + 1] = x[3];
                __syncwarp();
                float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    uint32_t af[4], bf[2];
                    const int ar = o + 16 + fg, ac = o + 16 + 8 * ks + ft;
                    af[0] = to_tf32(TF[ar * LDA + ac]);
                    af[1] = to_tf32(TF[(ar + 8) * LDA + ac]);
                    af[2] = to_tf32(TF[ar * LDA + ac + 4]);
                    af[3] = to_tf32(TF[(ar + 8) * LDA + ac + 4]);
                    bf[0] = to_tf32(TF[(o + 8 * ks + ft) * LDA + o + 16 + n0 + fg]);
                    bf[1] = to_tf32(TF[(o + 8 * ks + ft + 4) * LDA + o + 16 + n0 + fg]);
                    mma_tf32_16x8x8(y, af, bf);
                }
                TF[(o + 16 + fg) * LDA + o + n0 + 2 * ft] = -y[0];
                TF[(o + 16 + fg) * LDA + o + n0 + 2 * ft + 1] = -y[1];
                TF[(o + 24 + fg) * LDA + o + n0 + 2 * ft] = -y[2];
                TF[(o + 24 + fg) * LDA + o + n0 + 2 * ft + 1] = -y[3];
            }
            named_bar_sync(BAR_LOCAL, kLocal);
            // (3) T_{H1,H0} = -T_{H1} (A_{H1,H0} T_{H0}), 32x32 blocks; warp w owns
            //     output rows 16(w/4).., columns 8(w%4)..  X goes to the unused
            //     upper-right 32x32 block.  The upper triangles of T_{H0} and
            //     T_{H1} hold scratch, so their fragments are masked.
            {
                const int m0 = 16 * (warp >> 2), n0 = 8 * (warp & 3);
                float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    uint32_t af[4], bf[2];
                    const int ar = 32 + m0 + fg, ac = 8 * ks + ft;
                    af[0] = to_tf32(AF[ar * LDA + ac]);
                    af[1] = to_tf32(AF[(ar + 8) * LDA + ac]);
                    af[2] = to_tf32(AF[ar * LDA + ac + 4]);
                    af[3] = to_tf32(AF[(ar + 8) * LDA + ac + 4]);
                    const int br = 8 * ks + ft, bc = n0 + fg;
                    bf[0] = to_tf32(br >= bc ? TF[br * LDA + bc] : 0.f);
                    bf[1] = to_tf32(br + 4 >= bc ? TF[(br + 4) * LDA + bc] : 0.f);
                    mma_tf32_16x8x8(x, af, bf);
                }
                TF[(m0 + fg) * LDA + 32 + n0 + 2 * ft] = x[0];
                TF[(m0 + fg) * LDA + 32 + n0 + 2 * ft + 1] = x[1];
                TF[(m0 + fg + 8) * LDA + 32 + n0 + 2 * ft] = x[2];
                TF[(m0 + fg + 8) * LDA + 32 + n0 + 2 * ft + 1] = x[3];
                named_bar_sync(BAR_LOCAL, kLocal);
                float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    uint32_t af[4], bf[2];
                    const int r = m0 + fg, kc = 8 * ks + ft;  // within H1
                    af[0] = to_tf32(kc <= r ? TF[(32 + r) * LDA + 32 + kc] : 0.f);
                    af[1] = to_tf32(kc <= r + 8 ? TF[(40 + r) * LDA + 32 + kc] : 0.f);
                    af[2] = to_tf32(kc + 4 <= r ? TF[(32 + r) * LDA + 36 + kc] : 0.f);
                    af[3] = to_tf32(kc + 4 <= r + 8 ? TF[(40 + r) * LDA + 36 + kc] : 0.f);
                    bf[0] = to_tf32(TF[(8 * ks + ft) * LDA + 32 + n0 + fg]);
                    bf[1] = to_tf32(TF[(8 * ks + ft + 4) * LDA + 32 + n0 + fg]);
                    mma_tf32_16x8x8(y, af, bf);
                }
                TF[(32 + m0 + fg) * LDA + n0 + 2 * ft] = -y[0];
                TF[(32 + m0 + fg) * LDA + n0 + 2 * ft + 1] = -y[1];
                TF[(40 + m0 + fg) * LDA + n0 + 2 * ft] = -y[2];
                TF[(40 + m0 + fg) * LDA + n0 + 2 * ft + 1] = -y[3];
            }
            named_bar_sync(BAR_LOCAL, kLocal);
            // ---- T diag(beta) and T diag(beta gamma) in bf16 (K-major, s cols) ---
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int idx = tid + kLocal * it, r = idx & 63, j = idx >> 6;  // lanes: rows
                float tv[8], bv[8], gv[8], tb[8], tg[8];
                *reinterpret_cast<float4 *>(tv) = *reinterpret_cast<const float4 *>(TF + r * LDA + 8 * j);
                *reinterpret_cast<float4 *>(tv + 4) = *reinterpret_cast<const float4 *>(TF + r * LDA + 8 * j + 4);
                *reinterpret_cast<float4 *>(bv) = *reinterpret_cast<const float4 *>(b_s + 8 * j);
                *reinterpret_cast<float4 *>(bv + 4) = *reinterpret_cast<const float4 *>(b_s + 8 * j + 4);
                *reinterpret_cast<float4 *>(gv) = *reinterpret_cast<const float4 *>(bg_s + 8 * j);
                *reinterpret_cast<float4 *>(gv + 4) = *reinterpret_cast<const float4 *>(bg_s + 8 * j + 4);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s2 = 8 * j + e;
                    const float t2 = s2 < r ? tv[e] : (s2 == r ? 1.f : 0.f);
                    tb[e] = t2 * bv[e];
                    tg[e] = t2 * gv[e];
                }
                *reinterpret_cast<uint4 *>(sm + OFF_TB + sw128(r, j)) = pack8(tb);
                *reinterpret_cast<uint4 *>(sm + OFF_TG + sw128(r, j)) = pack8(tg);
            }
            fence_proxy_async_smem();
            named_bar_sync(BAR_LOCAL, kLocal);
            // ---- D_w = [T_bg; 0] K (rows 0-63: W);  D_vp = [0; T_b] V --------------
            // (D_vp of this parity and its handoff slot are free once the state
            // pass of chunk m-2 is over)
            if (tid == 4 * 32) {  // warp 4 is idle during the P stores below
                if (m >= 2) ok &= wait_bar(&bar_vpfree[st], (uint32_t)(((m >> 1) - 1) & 1), abort_flag, lim);
                tc_fence_after();
                const uint64_t dk = d_kmn0 + st * (RAW_STAGE >> 4);
                const uint64_t dv = d_vmn0 + st * (RAW_STAGE >> 4);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tmem + COL_W, d_tg + k * 2, dk + k * 128, ID_W, k > 0);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tmem + COL_VP + 64 * st, d_ztb + k * 2, dv + k * 128, ID_KM, k > 0);
                mma_commit(bar_l);
            }
            ++bl_commit;
            // ---- while those run: store P once the state pass has consumed the
            //      previous chunk's P ------------------------------------------------
            if (tid == 0 && m >= 1) ok &= wait_bar(bar_pfree, (uint32_t)((m - 1) & 1), abort_flag, lim);
            if (named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag)) break;
            if (lq >= 2) {
                const int r = 32 * (lq - 2) + lane;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4 *>(sm + OFF_P + sw128(r, 4 * lhalf + j)) = p_hold[j];
            } else if (warp == 5) {  // g and g_C for the state pass of this chunk
                float *hand = reinterpret_cast<float *>(sm + OFF_HAND + st * HAND_STRIDE);
                hand[2 * lane] = g_s[2 * lane];
                hand[2 * lane + 1] = g_s[2 * lane + 1];
                if (lane == 0) hand[64] = g_s[63];
            }
            if (tid == 0) ok &= wait_bar(bar_l, bl_wait & 1, abort_flag, lim);
            ++bl_wait;
            if (named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag)) break;
            tc_fence_after();
            // ---- the next chunk's D_kq, so that it overlaps the rest of this one
            if (m + 1 < nchunks && !start_chunk(m + 1, 6 * 32)) break;
            // ---- -W into its rows of the stage (K-major, atom column lhalf) ------
            if (lq < 2) {
                float w[64];
                tmem_load<64>(tmem + lane_off + COL_W + 64 * lhalf, w);  // lane r: W[r][c]
                const int r = 32 * lq + lane;
#pragma unroll
                for (int j = 0; j < 64; ++j) w[j] = -w[j];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(raw + lhalf * RAW_AC + RAW_W + sw128(r, j)) = pack8(w + 8 * j);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag)) break;
            if (tid == 0) mbar_arrive(bar_ready);
        }
        // drain what this group launched
        if (*abort_flag && tid == 0)
            for (uint32_t i = bl_wait; i < bl_commit; ++i) mbar_wait(bar_l, i & 1, kWaitLimit);
    } else {
        // ============================ state group ============================
        const int sq = warp & 3;  // TMEM lane quadrant = warp - 8
        const uint32_t lane_off = (uint32_t)(32 * sq) << 16;
        uint32_t bs_wait = 0, bs_commit = 0;
        const uint64_t d_qw0 = desc_sw128(sbase + OFF_RAW + RAW_Q, 16, 1024);
        const uint64_t d_kmn0 = desc_sw128(sbase + OFF_RAW + RAW_K, RAW_AC, 1024);
        const uint64_t d_sb = desc_sw128(sbase + OFF_SB, 16384, 1024);
        const uint64_t d_vp = desc_sw128(sbase + OFF_VP, 8192, 1024);
        const uint64_t d_vh = desc_sw128(sbase + OFF_VH, 8192, 1024);
        const uint64_t d_pz = desc_sw128(sbase + OFF_P, 16, 1024);
        for (int m = 0; m < nchunks; ++m) {
            const int st = m & 1;
            const long long t0 = t_begin + (long long)m * C;
            const int L = chunk_len(m);
            const float *hand = reinterpret_cast<const float *>(sm + OFF_HAND + st * HAND_STRIDE);
            bool ok = true;
            if (tid == kLocal) ok = wait_bar(bar_ready, (uint32_t)(m & 1), abort_flag, lim);
            if (named_bar_or(BAR_STATE, kState, !ok || *abort_flag)) break;
            tc_fence_after();
            const float gC = hand[64];
            const float dec = __expf(gC);
            // ---- D_vp += [Q; -W] S^T ----------------------------------------------
            if (tid == kLocal) {
                tc_fence_after();
                const uint64_t da = d_qw0 + st * (RAW_STAGE >> 4);
#pragma unroll
                for (int k = 0; k < DK / 16; ++k)
                    mma_bf16(tmem + COL_VP + 64 * st, da + (((k >> 2) * RAW_AC + (k & 3) * 32) >> 4),
                             d_sb + k * 128, ID_KM, 1);
                mma_commit(bar_s);
            }
            ++bs_commit;
            if (tid == kLocal) ok &= wait_bar(bar_s, bs_wait & 1, abort_flag, lim);
            ++bs_wait;
            if (named_bar_or(BAR_STATE, kState, !ok || *abort_flag)) break;
            tc_fence_after();
            // ---- V' (rows 64-127) and kh . V' as MN-major operands ----------------
            if (sq >= 2) {
                float vp[64];
                tmem_load<64>(tmem + lane_off + COL_VP + 64 * st, vp);
                const int r = 32 * (sq - 2) + lane;
                const float khr = __expf(gC - hand[r]);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(sm + OFF_VP + sw128(r, j)) = pack8(vp + 8 * j);
#pragma unroll
                for (int j = 0; j < 64; ++j) vp[j] *= khr;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(sm + OFF_VH + sw128(r, j)) = pack8(vp + 8 * j);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (named_bar_or(BAR_STATE, kState, !ok || *abort_flag)) break;
            // ---- D_ds = K^T (kh . V');  D_o = [P; 0] V' ----------------------------
            if (tid == kLocal) {
                tc_fence_after();
                const uint64_t dk = d_kmn0 + st * (RAW_STAGE >> 4);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tmem + COL_DS, dk + k * 128, d_vh + k * 128, ID_MM, k > 0);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tmem + COL_O, d_pz + k * 2, d_vp + k * 128, ID_KM, k > 0);
                mma_commit(bar_s);
                mma_commit(bar_pfree);
            }
            ++bs_commit;
            if (tid == kLocal) ok &= wait_bar(bar_s, bs_wait & 1, abort_flag, lim);
            ++bs_wait;
            if (named_bar_or(BAR_STATE, kState, !ok || *abort_flag)) break;
            tc_fence_after();
            // the stage is free: load chunk m+2 into it
            if (tid == kLocal && ok && m + 2 < nchunks) issue_tma(m + 2);
            // ---- S <- e^{g_C} S + dS;  o_r = e^{g_r} (Q S^T)_r + (P V')_r ----------
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float ds[32];
                tmem_load<32>(tmem + lane_off + COL_DS + 32 * hh, ds);  // lane c: dS[i][c]
#pragma unroll
                for (int i = 0; i < 32; ++i) s_reg[32 * hh + i] = dec * s_reg[32 * hh + i] + ds[i];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(sm + OFF_SB + sw128(c_st, j)) = pack8(s_reg + 8 * j);
            if (sq < 2) {
                const int r = 32 * sq + lane;
                const float er = __expf(hand[r]);
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.o) +
                                     ((t0 + r) * H + h) * (long long)a.dv + v0;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float qs[32], pv[32];
                    tmem_load<32>(tmem + lane_off + COL_VP + 64 * st + 32 * hh, qs);
                    tmem_load<32>(tmem + lane_off + COL_O + 32 * hh, pv);
#pragma unroll
                    for (int j = 0; j < 32; ++j) qs[j] = er * qs[j] + pv[j];
                    if (r < L) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            reinterpret_cast<uint4 *>(dst)[4 * hh + j] = pack8(qs + 8 * j);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (named_bar_or(BAR_STATE, kState, !ok || *abort_flag)) break;
            if (tid == kLocal) mbar_arrive(&bar_vpfree[st]);
        }
        if (*abort_flag) {
            if (tid == kLocal)
                for (uint32_t i = bs_wait; i < bs_commit; ++i) mbar_wait(bar_s, i & 1, kWaitLimit);
        } else if (a.s_final) {
#pragma unroll
            for (int i = 0; i < DVS; ++i) a.s_final[st_base + (size_t)(v0 + i) * DK + c_st] = s_reg[i];
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        atomicOr(a.err, kErrTimeout);
        // let every tile load already issued land before the CTA exits: loads of
        // a stage complete in issue order, so the last one's phase suffices
        for (int st = 0; st < 2; ++st)
            if (tma_issued[st] > 0)
                mbar_wait(&bar_tma[st], (uint32_t)((tma_issued[st] - 1) & 1), kWaitLimit);
    }
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace

// ------------------------------------------------------------------- host --
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// [tokens, H, d] bf16 viewed as a 3-D tensor (d, H, tokens); box 64 x 1 x 64.
bool make_tile_map(CUtensorMap *m, const void *base, int d, int H, long long ntok) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)ntok};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// [tokens, H, 128] bf16 viewed as a 4-D tensor (64, tokens, 2, H): one box
// (64, 64, 2, 1) brings both 64-wide halves of a 64-token tile as two
// consecutive 8 KB tiles, 128-byte swizzled (coordinates {0, t0, 0, h}).
bool make_halves_map(CUtensorMap *m, const void *base, int H, long long ntok) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {64, (cuuint64_t)ntok, 2, (cuuint64_t)H};
    cuuint64_t strides[3] = {(cuuint64_t)H * 256, 128, 256};
    cuuint32_t box[4] = {64, 64, 2, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

bool chunk_tc_supported(const gdn_dims &d) {
    return d.dtype == GDN_BF16 && d.d_k == DK && d.d_v == 128 && d.decay == GDN_DECAY_SCALAR &&
           (long long)d.B * d.T < (1LL << 31);
}

size_t chunk_tc_scratch_bytes(const gdn_dims &) { return 0; }

cudaError_t launch_chunk_tc(const PrefillArgs &a, cudaStream_t s, int *launches) {
    const long long items = (long long)a.n_seqs * a.H * (a.dv / DVS);
    const long long ntok = (long long)a.B * a.T;
    if (items == 0) return cudaSuccess;
    if (ntok == 0) {
        // no tokens at all: every sequence is empty, final = initial state
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
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chunk_tc_kernel<<<(unsigned)items, kThreads, SMEM_BYTES, s>>>(a, mq, mk, mv);
    if (launches) ++*launches;
    return cudaGetLastError();
}

}  // namespace gdn

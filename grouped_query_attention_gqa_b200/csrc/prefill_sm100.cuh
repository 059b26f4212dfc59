// GQA causal prefill on sm_100a: RoPE on load, QK^T and PV on tcgen05 with
// accumulators in tensor memory, online softmax with causal tile skipping.
//
// What is computed (page "Qwen2 architecture introduction", aicoding.csdn.net,
// §4.1.2-§4.1.3): for each batch row b and query head t, with u = t / g the
// KV group, S = Q'_t K'_u^T / sqrt(d), S_ij = -inf for j > i, A = softmax(S),
// head_t = A V_u, written to out[b, i, t, :] (the concatenated-heads layout of
// §4.1.3 step 5).  Q' and K' are the RoPE-rotated rows (rope.cuh).
//
// Two kernels:
//  * prep_kernel: Q and K rotated once, into head-major buffers Q' [B, h_q, L, d] and
//    K' [B, h_kv, L, d], with one cos/sin table per block of positions shared by Q and K (page
//    "Qwen2 / Qwen3 的实测配置差异与三个坑", docs.keinmal.top, closing note of pitfall 3).  It is a
//    streaming, bandwidth-bound pass; rotating there instead of in the attention kernel takes the
//    rotation (and its latency) off the start of every attention CTA, and every K' tile is read by
//    ~L/256 * g query tiles, so rotating K once beats rotating it on each use.
//  * attn_kernel: persistent, one CTA per SM.  Each CTA walks a list of work items, each a pair of
//    128-row query tiles of the same (b, KV group), heaviest first.  Q', K' and V tiles arrive by TMA;
//    each K'/V tile is brought into shared memory once and consumed by both query tiles (GQA reuse
//    inside the CTA; the remaining heads of the group hit the same tiles in L2).  Barrier phases run
//    on across items, so the next pair's Q' is loaded as soon as the last S of the current pair has
//    finished and its first S starts while the current pair's output is still being written.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for query tile 0   (thread = query row = TMEM lane)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer of K', V tiles (2-stage rings)
//   warp  9    tcgen05 MMA issuer (the whole warp, converged; one elected lane issues each MMA);
//              also owns the TMEM allocation
//   warp 10    TMA producer of the Q' tiles (one buffer per query tile)
//   warp 11    idle
// Each SM sub-partition hosts three warps, which caps a uniform budget at 168
// registers; the third warpgroup hands 80 of its registers per thread to the
// two softmax warpgroups (setmaxnreg: 208 / 208 / 88), which then hold a full
// 128-column score row in registers.
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [.., +d);
// P_k (bf16, two per column) overwrites the first 64 columns of S_k.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "rope.cuh"
#include "sm100_ptx.cuh"

namespace gqa {
namespace prefill {

using namespace ptx;

constexpr int BM = 128;   // query rows per tile (MMA M)
constexpr int BN = 128;   // key rows per tile (MMA N of QK^T, K of PV)
constexpr int KSTAGES = 2;
constexpr int VSTAGES = 2;
constexpr int NUM_WARPS = 12;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int WARP_TMA = 8;     // K'/V producer
constexpr int WARP_MMA = 9;
constexpr int WARP_QLOAD = 10;  // Q' producer
// Register split.  setmaxnreg.inc waits until the registers exist in the block's own
// allocation (threads x launch registers), so the shares must not add up to more than that
// (here they add up to it exactly: 256 x 208 + 128 x 88 = 384 x 168);
// the host refuses to launch if ptxas gave the kernel any other count than LAUNCH_REGS.
constexpr int LAUNCH_REGS = 168;
constexpr int SOFTMAX_REGS = 208;
constexpr int OTHER_REGS = 88;
static_assert(256 * SOFTMAX_REGS + 128 * OTHER_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t P_COL = 0;    // P_k (128 bf16 per row, two per column) fills columns 0..63 of S_k
constexpr float kRescaleThreshold = 8.0f;   // log2 units: O is rescaled only when the max grows by > 2^8
// Of every 8 consecutive pairs of exponentials of a row (off the diagonal tile), this many run on
// the FMA pipe (exp2_poly_x2) and the rest on the ex2 unit.
#ifndef GQA_EXP_POLY_OF_8
#define GQA_EXP_POLY_OF_8 2
#endif
#ifndef GQA_PREP_POS
#define GQA_PREP_POS 8
#endif
#ifndef GQA_PREP_MIN_CTAS
#define GQA_PREP_MIN_CTAS 2
#endif
constexpr int PREP_POS = GQA_PREP_POS;          // positions per CTA of the prep kernel
constexpr int PREP_THREADS = 256;

struct Params {
    __nv_bfloat16* out;        // [B, L, h_q, D]
    int B, L, h_q, h_kv, g;
    int n_qtiles;              // ceil(L / BM)
    int tiles_per_group;       // n_qtiles * g
    int total_work;            // tile pairs in all: ceil(tiles_per_group / 2) * B * h_kv
    float scale_log2;          // log2(e) / sqrt(D)
    // The work list of each CTA: items sched[sched_start[c] .. sched_start[c + 1]) for CTA c, in order
    // (built on the host, see work_item).
    const int* sched_start;
    const int* sched;
    int* err;
};

template <int D>
struct Layout {
    static constexpr int TILE = BM * D * 2;   // one 128-row bf16 tile
    static constexpr int SUB = BM * 128;      // one 64-column, 128-byte-swizzled block
    static constexpr int Q0 = 0;
    static constexpr int K0 = 2 * TILE;
    static constexpr int V0 = K0 + KSTAGES * TILE;
    static constexpr int OSTAGE = 32 * 128;            // one warp's 32 rows x 64 columns, swizzled
    static constexpr int O0 = V0 + VSTAGES * TILE;     // 8 softmax warps x OSTAGE
    static constexpr int BYTES = O0 + 8 * OSTAGE;
    // At least 120 KB so that two CTAs never share an SM: each holds all 512 TMEM columns.
    static constexpr int DYN = (BYTES < 120 * 1024 ? 120 * 1024 : BYTES) + 1024;
};

struct alignas(8) Shared {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[KSTAGES], k_empty[KSTAGES];
    uint64_t v_full[VSTAGES], v_empty[VSTAGES];
    uint64_t s_full[2], p_full[2], o_full[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

// ---------------------------------------------------------------------------------------------
// prep_kernel: for positions [p0, p0+PREP_POS): the cos/sin table, then every Q and K row at those
// positions rotated into Q' [B*h_q, L, D] and K' [B*h_kv, L, D].
// Thread t owns 16-byte chunk c = t % CH of each half row (8 rotation pairs: dims 8c.. and their partners
// 8c + D/2..) and walks the rows (b, head) r0, r0 + RPP, ... (r0 = t / CH), each at all PREP_POS positions
// of the block: one row per round, its loads issued together.  The pass issues few instructions per byte
// (one division per row, 16-byte table reads, paired fp32 rotation), which is what bounds it.
template <int D>
__global__ void __launch_bounds__(PREP_THREADS, GQA_PREP_MIN_CTAS) prep_kernel(const __nv_bfloat16* __restrict__ q,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            __nv_bfloat16* __restrict__ qr,
                                                            __nv_bfloat16* __restrict__ kr, int B, int L,
                                                            int h_q, int h_kv, RopeSpec rope, float mscale) {
    constexpr int H = D / 2;
    constexpr int CH = D / 16;                 // 16-byte chunks of a half row
    constexpr int RPP = PREP_THREADS / CH;     // rows per round of the block
    // Table row pp: (cos f_i, cos f_i+1, sin f_i, sin f_i+1) of position p0 + pp for i = 2j, as float4 j, with
    // one float4 of padding after every 4, so the CH lanes reading the 4 float4 of their chunks hit
    // distinct banks (lanes of the same chunk read the same address).
    constexpr int TROW4 = H / 2 + H / 8;
    __shared__ float4 tab[PREP_POS * TROW4];
    __shared__ double finv[H];
    const int p0 = blockIdx.x * PREP_POS;
    const int heads = h_q + h_kv;
    const int bh_n = B * heads;   // B * (h_q + h_kv) < 2^31 is checked on the host
    const int c = threadIdx.x % CH;
    const int r0 = threadIdx.x / CH;
    const int np = L - p0 < PREP_POS ? L - p0 : PREP_POS;   // positions of this block (the last may be short)

    uint4 x[PREP_POS], y[PREP_POS];
    __nv_bfloat16* dst = nullptr;   // row pp of the current round's destination: dst + pp * D
    auto load_row = [&](int bh) {
        const int b = bh / heads, h = bh - (bh / heads) * heads;
        const __nv_bfloat16* src;
        int64_t stride;
        if (h < h_q) {
            src = q + ((static_cast<int64_t>(b) * L + p0) * h_q + h) * D;
            stride = static_cast<int64_t>(h_q) * D;
            dst = qr + ((static_cast<int64_t>(b) * h_q + h) * L + p0) * D;
        } else {
            src = k + ((static_cast<int64_t>(b) * L + p0) * h_kv + (h - h_q)) * D;
            stride = static_cast<int64_t>(h_kv) * D;
            dst = kr + ((static_cast<int64_t>(b) * h_kv + (h - h_q)) * L + p0) * D;
        }
#pragma unroll
        for (int pp = 0; pp < PREP_POS; ++pp) {
            if (pp < np) {
                const uint4* row = reinterpret_cast<const uint4*>(src + pp * stride);
                x[pp] = __ldg(row + c);
                y[pp] = __ldg(row + c + CH);
            }
        }
    };
    // The first round's loads go out before the table is built.
    if (r0 < bh_n) load_row(r0);

    // theta^(-2i/D) = 2^(-(2i/D) * log2(theta)), scaled under YaRN
    for (int i = threadIdx.x; i < H; i += blockDim.x) finv[i] = rope_freq(i, D, rope);
    __syncthreads();
    for (int e = threadIdx.x; e < PREP_POS * (H / 2); e += blockDim.x) {
        const int pp = e / (H / 2), j = e % (H / 2);
        float c0 = 1.f, s0 = 0.f, c1 = 1.f, s1 = 0.f;
        if (pp < np) {
            rope_cossin(static_cast<double>(p0 + pp), finv[2 * j], c0, s0);
            rope_cossin(static_cast<double>(p0 + pp), finv[2 * j + 1], c1, s1);
        }
        // YaRN temperature on Q and K (1 without scaling)
        tab[pp * TROW4 + j + j / 4] = make_float4(c0 * mscale, c1 * mscale, s0 * mscale, s1 * mscale);
    }
    __syncthreads();

    const uint64_t neg1 = f2_pack(-1.f, -1.f);
    for (int bh = r0; bh < bh_n; bh += RPP) {
        if (bh != r0) load_row(bh);
#pragma unroll
        for (int pp = 0; pp < PREP_POS; ++pp) {
            if (pp >= np) continue;
            const uint32_t xs[4] = {x[pp].x, x[pp].y, x[pp].z, x[pp].w};
            const uint32_t ys[4] = {y[pp].x, y[pp].y, y[pp].z, y[pp].w};
            uint32_t xo[4], yo[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 t = tab[pp * TROW4 + 5 * c + w];   // pairs i = 8c + 2w, +1
                const uint64_t cs = f2_pack(t.x, t.y), sn = f2_pack(t.z, t.w);
                const uint64_t X = f2_from_bf16x2(xs[w]), Y = f2_from_bf16x2(ys[w]);
                // x' = fma(x, cos, -(y sin)), y' = fma(y, cos, x sin): the scalar rotation, two pairs at once
                const uint64_t xr = f2_fma(X, cs, f2_mul(f2_mul(Y, sn), neg1));
                const uint64_t yr = f2_fma(Y, cs, f2_mul(X, sn));
                xo[w] = f2_to_bf16x2(xr);
                yo[w] = f2_to_bf16x2(yr);
            }
            uint4* out = reinterpret_cast<uint4*>(dst + pp * D);
            out[c] = make_uint4(xo[0], xo[1], xo[2], xo[3]);
            out[c + CH] = make_uint4(yo[0], yo[1], yo[2], yo[3]);
        }
    }
}

// P = 2^(s * scale_log2 - m) for one row of 128 scores, stored as bf16 pairs from TMEM column t_p
// (the first half of the S region: chunk c overwrites S columns 16c.., already in registers); returns
// the row sum of the fp32 values.  POLY: part of the exponentials on the FMA pipe (never on a tile
// with masked entries, whose weights must be exactly 0).
template <bool POLY>
__device__ __forceinline__ float row_exp_store(const uint32_t (&sr)[4][32], float sl2, float neg_m, uint32_t t_p) {
    const uint64_t scale2 = f2_pack(sl2, sl2), shift2 = f2_pack(neg_m, neg_m);
    uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), scale2, shift2);
            float p0, p1;
            if (POLY && ((e >> 1) & 7) < GQA_EXP_POLY_OF_8) {
                exp2_poly_x2(x, p0, p1);
            } else {
                float x0, x1;
                f2_unpack(x, x0, x1);
                p0 = ex2(x0);
                p1 = ex2(x1);
            }
            acc[(e >> 1) & 1] = f2_add(acc[(e >> 1) & 1], f2_pack(p0, p1));
            pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(t_p + 16 * c, pk);
    }
    float a0, a1, b0, b1;
    f2_unpack(acc[0], a0, a1);
    f2_unpack(acc[1], b0, b1);
    return (a0 + a1) + (b0 + b1);
}

// Byte address of 16-byte chunk `cc` (8 bf16 along d) of row r in a K-major, 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t swz_off(int r, int cc) {
    return static_cast<uint32_t>((cc >> 3) * (BM * 128) + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}

// One work item = a pair of 128-row query tiles of one (b, KV group).  Items are numbered heaviest
// first: item w = pair * (B * h_kv) + (b * h_kv + u), and pair q holds tiles 2q and 2q+1 of the group's
// list (query tile descending, head ascending), so both tiles of a pair need about the same number of
// key tiles.
struct PairWork {
    int b, u, n0, n1, head0, head1;
};

__device__ __forceinline__ PairWork pair_work(const Params& p, int w) {
    PairWork r;
    const int BH = p.B * p.h_kv;
    const int pair = w / BH, bu = w % BH;
    r.b = bu / p.h_kv;
    r.u = bu % p.h_kv;
    const int i0 = 2 * pair, i1 = 2 * pair + 1;
    r.n0 = i0 < p.tiles_per_group ? p.n_qtiles - i0 / p.g : 0;   // tile needs key tiles 0 .. qt (BM == BN)
    r.n1 = i1 < p.tiles_per_group ? p.n_qtiles - i1 / p.g : 0;
    r.head0 = r.u * p.g + i0 % p.g;
    r.head1 = r.u * p.g + i1 % p.g;
    return r;
}

// The r-th item of persistent CTA c (p.total_work once the CTA's list is done): its own list, built on the
// host so that every CTA carries about the same number of key tiles.
__device__ __forceinline__ int work_item(const Params& p, int r, int c) {
    const int i = __ldg(p.sched_start + c) + r;
    return i < __ldg(p.sched_start + c + 1) ? __ldg(p.sched + i) : p.total_work;
}

template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const Params p) {
    using Lay = Layout<D>;
    extern __shared__ uint8_t dyn_smem_raw[];
    __shared__ Shared sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int k = 0; k < 2; ++k) {
            mbar_init(&sh.q_full[k], 1);
            mbar_init(&sh.q_empty[k], 1);
            mbar_init(&sh.s_full[k], 1);
            mbar_init(&sh.p_full[k], 128);
            mbar_init(&sh.o_full[k], 1);
        }
        for (int s = 0; s < KSTAGES; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
        }
        for (int s = 0; s < VSTAGES; ++s) {
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 1);
        }
        mbar_init(&sh.mma_done, 1);
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(&sh.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == WARP_QLOAD && lane == 0) prefetch_tensormap(&tm_q);
    if (warp == WARP_TMA && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int* abort = &sh.abort;

    if (warp < 8) regs_increase<SOFTMAX_REGS>();
    else regs_decrease<OTHER_REGS>();

    if (warp < 8) {
        // ================================================================ softmax / epilogue of tile k
        const int k = warp >> 2;
        const int r = (warp & 3) * 32 + lane;   // query row in the tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + static_cast<uint32_t>(k * 128);
        const uint32_t t_p = t_s + P_COL;   // P_k: bf16 pairs over the first half of S_k
        const uint32_t t_o = tmem + lane_base + static_cast<uint32_t>(256 + k * D);
        const float sl2 = p.scale_log2;
        uint32_t s_seen = 0;   // S_k results consumed (s_full phases)
        uint32_t o_seen = 0;   // PV_k products issued for the pairs handled so far (o_full phases)
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int w = work_item(p, it, cta);
            if (w >= p.total_work) break;
            const PairWork pw = pair_work(p, w);
            const int nk = k ? pw.n1 : pw.n0;
            if (nk == 0) continue;
            const int qtk = nk - 1;
            const int headk = k ? pw.head1 : pw.head0;
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < nk; ++j) {
                ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[k], s_seen & 1, p.err, abort));
                if (!ok) break;
                ++s_seen;
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(t_s + 32 * c, sr[c]);
                tmem_wait_ld();
                const bool diag = (j == qtk);
                if (diag) {   // diagonal tile: key column c sits at the same offset as query row r
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (32 * c + e > r) sr[c][e] = __float_as_uint(-INFINITY);
                }
                float mxs[8];   // eight independent running maxima, two scores per 3-input max
#pragma unroll
                for (int e = 0; e < 8; ++e) mxs[e] = __uint_as_float(sr[0][e]);
#pragma unroll
                for (int i = 8; i < 128; i += 2)
                    mxs[(i >> 1) & 7] = fmax3(mxs[(i >> 1) & 7], __uint_as_float(sr[i >> 5][i & 31]),
                                              __uint_as_float(sr[i >> 5][(i & 31) + 1]));
                const float mx = fmaxf(fmax3(mxs[0], mxs[1], mxs[2]), fmax3(fmax3(mxs[3], mxs[4], mxs[5]), mxs[6], mxs[7]));
                const float m_new = fmaxf(m_run, mx * sl2);
                if (j == 0) {
                    m_run = m_new;
                } else if (__any_sync(0xffffffffu, m_new > m_run + kRescaleThreshold)) {
                    // All MMAs issued before S_j (PV_{j-1} included) have completed: rescale O in place.
                    const float alpha = ex2(m_run - m_new);
                    m_run = m_new;
                    l_run *= alpha;
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(t_o + 32 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(t_o + 32 * c, o);
                    }
                    tmem_wait_st();
                }
                const float neg_m = -m_run;
                if (diag) l_run += row_exp_store<false>(sr, sl2, neg_m, t_p);
                else l_run += row_exp_store<true>(sr, sl2, neg_m, t_p);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sh.p_full[k]);
            }
            if (!ok) break;
            // ---- epilogue: O / l -> bf16 -> out[b, row, head, :].  The next pair's S_k may already be
            // running; its first PV_k (which overwrites O_k) waits for this warpgroup's next P.
            o_seen += nk;
            ok = __all_sync(0xffffffffu, mbar_wait(&sh.o_full[k], (o_seen - 1) & 1, p.err, abort));
            if (!ok) break;
            tc_fence_after();
            const float inv_l = 1.0f / l_run;
            // Rows 32*(warp&3) .. +31 of the tile, one 64-column half per pass: stage in this warp's slot
            // (same 128-byte-swizzled layout as the output tensor map's 64 x 32 box), TMA-store, and wait
            // for the store to have read the slot before the next pass.  Rows >= L are clipped.
            uint8_t* os = smem + Lay::O0 + warp * Lay::OSTAGE;
#pragma unroll
            for (int h = 0; h < D / 64; ++h) {
#pragma unroll
                for (int c = 2 * h; c < 2 * h + 2; ++c) {
                    uint32_t o[32];
                    tmem_ld32(t_o + 32 * c, o);
                    tmem_wait_ld();
                    uint32_t wv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        const int cc = 4 * (c - 2 * h) + v4;   // 16-byte chunk within the 64-column half
                        *reinterpret_cast<uint4*>(os + lane * 128 + ((cc ^ (lane & 7)) << 4)) =
                            make_uint4(wv[4 * v4], wv[4 * v4 + 1], wv[4 * v4 + 2], wv[4 * v4 + 3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_4d(&tm_o, os, h * 64, headk, qtk * BM + (warp & 3) * 32, pw.b);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
                __syncwarp();
            }
            tc_fence_before();
        }
    } else if (warp == WARP_TMA) {
        // ================================================================ TMA producer
        if (lane == 0) {
            const uint32_t tile_bytes = static_cast<uint32_t>(BN * D * 2);
            uint32_t kv = 0;                 // K/V tiles issued so far (ring position)
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int w = work_item(p, it, cta);
                if (w >= p.total_work) break;
                const PairWork pw = pair_work(p, w);
                const int n[2] = {pw.n0, pw.n1};
                const int nmax = n[0] > n[1] ? n[0] : n[1];
                const int kv_plane = pw.b * p.h_kv + pw.u;
                for (int j = 0; j < nmax && ok; ++j, ++kv) {
                    const int ks = kv % KSTAGES;
                    if (kv >= KSTAGES && !mbar_wait(&sh.k_empty[ks], ((kv / KSTAGES) - 1) & 1, p.err, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.k_full[ks], tile_bytes);
                    uint8_t* kdst = smem + Lay::K0 + ks * Lay::TILE;
#pragma unroll
                    for (int h = 0; h < D / 64; ++h)
                        tma_load_3d(kdst + h * Lay::SUB, &tm_k, &sh.k_full[ks], h * 64, j * BN, kv_plane);
                    const int vs = kv % VSTAGES;
                    if (kv >= VSTAGES && !mbar_wait(&sh.v_empty[vs], ((kv / VSTAGES) - 1) & 1, p.err, abort)) {
                        // K tile kv was issued without its V: count it so the drain below waits for it.
                        ++kv;
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.v_full[vs], tile_bytes);
                    uint8_t* vdst = smem + Lay::V0 + vs * Lay::TILE;
#pragma unroll
                    for (int h = 0; h < D / 64; ++h)
                        tma_load_4d(vdst + h * Lay::SUB, &tm_v, &sh.v_full[vs], h * 64, pw.u, j * BN, pw.b);
                }
            }
            // Drain: never leave the CTA with copies still landing in its shared memory.
            for (uint32_t j = (kv > KSTAGES ? kv - KSTAGES : 0); j < kv; ++j)
                mbar_wait(&sh.k_full[j % KSTAGES], (j / KSTAGES) & 1, p.err, nullptr);
            for (uint32_t j = (kv > VSTAGES ? kv - VSTAGES : 0); j < kv; ++j)
                mbar_wait(&sh.v_full[j % VSTAGES], (j / VSTAGES) & 1, p.err, nullptr);
        }
    } else if (warp == WARP_QLOAD) {
        // ================================================================ Q' producer
        if (lane == 0) {
            uint32_t qn[2] = {0u, 0u};   // Q' tiles issued into buffer k so far
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int w = work_item(p, it, cta);
                if (w >= p.total_work) break;
                const PairWork pw = pair_work(p, w);
                for (int k = 0; k < 2 && ok; ++k) {
                    const int nk = k ? pw.n1 : pw.n0;
                    if (nk == 0) continue;
                    // Wait until the previous pair's last S on this buffer has finished.
                    if (qn[k] > 0 && !mbar_wait(&sh.q_empty[k], (qn[k] - 1) & 1, p.err, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.q_full[k], static_cast<uint32_t>(BM * D * 2));
                    uint8_t* qdst = smem + Lay::Q0 + k * Lay::TILE;
                    const int head = k ? pw.head1 : pw.head0;
#pragma unroll
                    for (int h = 0; h < D / 64; ++h)
                        tma_load_3d(qdst + h * Lay::SUB, &tm_q, &sh.q_full[k], h * 64, (nk - 1) * BM, pw.b * p.h_q + head);
                    ++qn[k];
                }
            }
            for (int k = 0; k < 2; ++k)   // drain
                if (qn[k] > 0) mbar_wait(&sh.q_full[k], (qn[k] - 1) & 1, p.err, nullptr);
        }
    } else if (warp == WARP_MMA) {
        // ================================================================ MMA issuer
        // The whole warp runs the loop, converged, on warp-uniform state; one elected lane issues each
        // tcgen05 instruction.  Descriptors are formed once and advanced by constant offsets.
        {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
            const uint32_t tm = tmem;   // read from shared memory: the same in every lane
            // The descriptors' low words (start address and leading offset); the high words are constants.
            const uint32_t q_lo = static_cast<uint32_t>(sw128_desc(smem_u32(smem + Lay::Q0), 16, 1024));
            const uint32_t k_lo = static_cast<uint32_t>(sw128_desc(smem_u32(smem + Lay::K0), 16, 1024));
            const uint32_t v_lo = static_cast<uint32_t>(sw128_desc(smem_u32(smem + Lay::V0), Lay::SUB, 1024));
            constexpr uint64_t DESC_HI = sw128_desc(0, 0, 1024) & 0xFFFFFFFF00000000ull;
            constexpr uint32_t TILE16 = Lay::TILE >> 4;   // one tile in descriptor address units
            // S_k = Q_k K_j^T : M=128 (query rows), N=128 (key rows), K=D in steps of 16.
            auto issue_s = [&](int k, int ks) {
                const uint32_t qa = q_lo + static_cast<uint32_t>(k) * TILE16;
                const uint32_t ka = k_lo + static_cast<uint32_t>(ks) * TILE16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = static_cast<uint32_t>(((kk >> 2) * Lay::SUB + (kk & 3) * 32) >> 4);
                    umma_ss_warp(tm + static_cast<uint32_t>(k * 128), DESC_HI | (qa + off), DESC_HI | (ka + off),
                                 IDESC_S, kk > 0 ? 1u : 0u);
                }
            };
            // O_k += P_k V_j : M=128, N=D (V is MN-major: d contiguous), K=128 key rows in steps of 16.
            auto issue_pv = [&](int k, int vs, bool acc) {
                const uint32_t va = v_lo + static_cast<uint32_t>(vs) * TILE16;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    umma_ts_warp(tm + static_cast<uint32_t>(256 + k * D), tm + static_cast<uint32_t>(k * 128 + P_COL + kk * 8),
                                 DESC_HI | (va + static_cast<uint32_t>(kk * 16 * 128 >> 4)), IDESC_PV,
                                 (acc || kk > 0) ? 1u : 0u);
                }
            };
            uint32_t kv = 0;               // K/V tiles consumed (ring position)
            uint32_t qn[2] = {0u, 0u};     // q_full phases consumed per buffer
            uint32_t pn[2] = {0u, 0u};     // p_full phases consumed per tile
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int w = __shfl_sync(0xffffffffu, work_item(p, it, cta), 0);
                if (w >= p.total_work) break;
                const PairWork pw = pair_work(p, w);
                const int n[2] = {pw.n0, pw.n1};
                const int nmax = n[0] > n[1] ? n[0] : n[1];
                // S_k of the first key tile as soon as query tile k is in shared memory.
                const int ks0 = kv % KSTAGES;
                ok = mbar_wait_warp(&sh.k_full[ks0], (kv / KSTAGES) & 1, p.err, abort);
                for (int k = 0; k < 2 && ok; ++k) {
                    if (n[k] == 0) continue;
                    ok = mbar_wait_warp(&sh.q_full[k], qn[k] & 1, p.err, abort);
                    if (!ok) break;
                    ++qn[k];
                    tc_fence_after();
                    issue_s(k, ks0);
                    umma_commit_warp(&sh.s_full[k]);
                    if (n[k] == 1) umma_commit_warp(&sh.q_empty[k]);   // that was the last S on buffer k
                }
                if (!ok) break;
                umma_commit_warp(&sh.k_empty[ks0]);
                for (int j = 0; j < nmax && ok; ++j) {
                    const uint32_t vi = kv + j;
                    const int vs = vi % VSTAGES;
                    ok = mbar_wait_warp(&sh.v_full[vs], (vi / VSTAGES) & 1, p.err, abort);
                    if (!ok) break;
                    bool k_next = false;
                    const uint32_t ki = kv + j + 1;
                    for (int k = 0; k < 2 && ok; ++k) {
                        if (j >= n[k]) continue;
                        ok = mbar_wait_warp(&sh.p_full[k], pn[k] & 1, p.err, abort);
                        if (!ok) break;
                        ++pn[k];
                        tc_fence_after();
                        issue_pv(k, vs, j > 0);
                        umma_commit_warp(&sh.o_full[k]);
                        if (j + 1 < n[k]) {
                            if (!k_next) {
                                ok = mbar_wait_warp(&sh.k_full[ki % KSTAGES], (ki / KSTAGES) & 1, p.err, abort);
                                if (!ok) break;
                                tc_fence_after();
                                k_next = true;
                            }
                            issue_s(k, ki % KSTAGES);
                            umma_commit_warp(&sh.s_full[k]);
                            if (j + 2 == n[k]) umma_commit_warp(&sh.q_empty[k]);
                        }
                    }
                    umma_commit_warp(&sh.v_empty[vs]);
                    if (k_next) umma_commit_warp(&sh.k_empty[ki % KSTAGES]);
                }
                kv += nmax;
            }
            // Every MMA must have finished before the tensor memory is released.
            umma_commit_warp(&sh.mma_done);
            mbar_wait_warp(&sh.mma_done, 0, p.err, nullptr);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace prefill
}  // namespace gqa

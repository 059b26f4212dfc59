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
//  * prep_kernel: one cos/sin table [L, d/2] shared by Q and K, and K rotated
//    once into a head-major buffer K' [B, h_kv, L, d].  Every K' tile is then
//    read by ~L/256 * g query tiles, so rotating it once beats rotating it on
//    every use.
//  * attn_kernel: one CTA per pair of 128-row query tiles of the same
//    (b, KV group); each K'/V tile is brought into shared memory once by TMA
//    and consumed by both tiles (GQA reuse inside the CTA; the remaining heads
//    of the group hit the same tiles in L2).  Q is rotated in registers on its
//    way into shared memory.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for query tile 0   (thread = query row = TMEM lane)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer (K', V tiles; 2-stage rings)
//   warp  9    tcgen05 MMA issuer (one thread); also owns the TMEM allocation
//   warps 10-11 idle
// Each SM sub-partition hosts three warps, which caps a uniform budget at 168
// registers; the third warpgroup hands 112 of its registers per thread to the
// two softmax warpgroups (setmaxnreg), which then hold a full 128-column score
// row in registers.
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
constexpr int WARP_TMA = 8;
constexpr int WARP_MMA = 9;
// Register split.  setmaxnreg.inc waits until the registers exist in the block's own
// allocation (threads x launch registers), so the shares must add up to exactly that; the
// host refuses to launch if ptxas gave the kernel any other count than LAUNCH_REGS.
constexpr int LAUNCH_REGS = 168;
constexpr int SOFTMAX_REGS = 224;
constexpr int OTHER_REGS = 56;
static_assert(256 * SOFTMAX_REGS + 128 * OTHER_REGS == NUM_THREADS * LAUNCH_REGS, "register split");
constexpr uint32_t TMEM_COLS = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: O is rescaled only when the max grows by > 2^8
constexpr int PREP_POS = 32;                // positions per CTA of the prep kernel
constexpr int PREP_THREADS = 256;

struct Params {
    const __nv_bfloat16* q;    // [B, L, h_q, D]
    __nv_bfloat16* out;        // [B, L, h_q, D]
    const float2* cs;          // [L, D/2]  (cos, sin) of position * theta^(-2i/D)
    int B, L, h_q, h_kv, g;
    int n_qtiles;              // ceil(L / BM)
    int tiles_per_group;       // n_qtiles * g
    float scale_log2;          // log2(e) / sqrt(D)
    int* err;
};

template <int D>
struct Layout {
    static constexpr int TILE = BM * D * 2;   // one 128-row bf16 tile
    static constexpr int SUB = BM * 128;      // one 64-column, 128-byte-swizzled block
    static constexpr int Q0 = 0;
    static constexpr int K0 = 2 * TILE;
    static constexpr int V0 = K0 + KSTAGES * TILE;
    static constexpr int BYTES = V0 + VSTAGES * TILE;
    // At least 120 KB so that two CTAs never share an SM: each holds all 512 TMEM columns.
    static constexpr int DYN = (BYTES < 120 * 1024 ? 120 * 1024 : BYTES) + 1024;
};

struct alignas(8) Shared {
    uint64_t q_full[2];
    uint64_t k_full[KSTAGES], k_empty[KSTAGES];
    uint64_t v_full[VSTAGES], v_empty[VSTAGES];
    uint64_t s_full[2], p_full[2], o_full[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

// ---------------------------------------------------------------------------------------------
// prep_kernel: cos/sin table for positions [p0, p0+PREP_POS) and K' for those positions.
template <int D>
__global__ void __launch_bounds__(PREP_THREADS) prep_kernel(const __nv_bfloat16* __restrict__ k,
                                                            __nv_bfloat16* __restrict__ kr,
                                                            float2* __restrict__ cs, int B, int L,
                                                            int h_kv, double theta) {
    constexpr int H = D / 2;
    __shared__ float2 tab[PREP_POS][H];
    __shared__ double finv[H];
    const int p0 = blockIdx.x * PREP_POS;
    for (int i = threadIdx.x; i < H; i += blockDim.x) finv[i] = rope_inv_freq(i, D, theta);
    __syncthreads();
    for (int e = threadIdx.x; e < PREP_POS * H; e += blockDim.x) {
        const int pp = e / H, i = e % H;
        const int pos = p0 + pp;
        if (pos < L) {
            float c, s;
            rope_cossin(static_cast<double>(pos), finv[i], c, s);
            tab[pp][i] = make_float2(c, s);
            cs[static_cast<size_t>(pos) * H + i] = make_float2(c, s);
        }
    }
    __syncthreads();
    // One work item = 8 pairs (16-byte chunk of the first half + its partner chunk).
    constexpr int CH = D / 16;
    const int64_t items = static_cast<int64_t>(PREP_POS) * B * h_kv * CH;
    for (int64_t e = threadIdx.x; e < items; e += blockDim.x) {
        const int c = static_cast<int>(e % CH);
        const int64_t rr = e / CH;
        const int pp = static_cast<int>(rr % PREP_POS);
        const int64_t bu = rr / PREP_POS;
        const int b = static_cast<int>(bu / h_kv), u = static_cast<int>(bu % h_kv);
        const int pos = p0 + pp;
        if (pos >= L) continue;
        const uint4* src = reinterpret_cast<const uint4*>(k + ((static_cast<int64_t>(b) * L + pos) * h_kv + u) * D);
        uint4* dst = reinterpret_cast<uint4*>(kr + ((static_cast<int64_t>(b) * h_kv + u) * L + pos) * D);
        const uint4 x = __ldg(src + c);
        const uint4 y = __ldg(src + c + CH);
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
        const uint32_t ys[4] = {y.x, y.y, y.z, y.w};
        uint32_t xo[4], yo[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float2 c0 = tab[pp][8 * c + 2 * w];
            const float2 c1 = tab[pp][8 * c + 2 * w + 1];
            float a0, b0, a1, b1;
            rope_rotate(bf16lo_to_f32(xs[w]), bf16lo_to_f32(ys[w]), c0.x, c0.y, a0, b0);
            rope_rotate(bf16hi_to_f32(xs[w]), bf16hi_to_f32(ys[w]), c1.x, c1.y, a1, b1);
            xo[w] = pack_bf16x2(a0, a1);
            yo[w] = pack_bf16x2(b0, b1);
        }
        dst[c] = make_uint4(xo[0], xo[1], xo[2], xo[3]);
        dst[c + CH] = make_uint4(yo[0], yo[1], yo[2], yo[3]);
    }
}

// ---------------------------------------------------------------------------------------------
// Byte address of 16-byte chunk `cc` (8 bf16 along d) of row r in a K-major, 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t swz_off(int r, int cc) {
    return static_cast<uint32_t>((cc >> 3) * (BM * 128) + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const Params p) {
    using Lay = Layout<D>;
    extern __shared__ uint8_t dyn_smem_raw[];
    __shared__ Shared sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work assignment: blockIdx -> (pair, b, u); pairs of the heaviest query tiles come first.
    const int BH = p.B * p.h_kv;
    const int pair = blockIdx.x / BH;
    const int bu = blockIdx.x % BH;
    const int b = bu / p.h_kv;
    const int u = bu % p.h_kv;
    // Tile k of the pair: query tile qt_k of head head_k; it needs key tiles 0 .. qt_k (BM == BN).
    const int idx0 = 2 * pair, idx1 = 2 * pair + 1;
    const int n0 = idx0 < p.tiles_per_group ? p.n_qtiles - idx0 / p.g : 0;
    const int n1 = idx1 < p.tiles_per_group ? p.n_qtiles - idx1 / p.g : 0;
    const int nmax = n0 > n1 ? n0 : n1;

    if (threadIdx.x == 0) {
        mbar_init(&sh.q_full[0], 128);
        mbar_init(&sh.q_full[1], 128);
        for (int s = 0; s < KSTAGES; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
        }
        for (int s = 0; s < VSTAGES; ++s) {
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 1);
        }
        for (int k = 0; k < 2; ++k) {
            mbar_init(&sh.s_full[k], 1);
            mbar_init(&sh.p_full[k], 128);
            mbar_init(&sh.o_full[k], 1);
        }
        mbar_init(&sh.mma_done, 1);
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(&sh.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == WARP_TMA && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int* abort = &sh.abort;

    if (warp < 8) regs_increase<SOFTMAX_REGS>();
    else regs_decrease<OTHER_REGS>();

    if (warp < 8) {
        // ================================================================ softmax / epilogue
        const int k = warp >> 2;
        const int r = (warp & 3) * 32 + lane;   // query row in the tile == TMEM lane
        const int idx = k ? idx1 : idx0;
        const int nk = k ? n1 : n0;
        const int qtk = nk - 1;
        const int headk = u * p.g + idx % p.g;
        if (nk > 0) {
            const int row = qtk * BM + r;
            // ---- Q: load, rotate at position `row`, store bf16 into the swizzled tile.
            uint8_t* qs = smem + Lay::Q0 + k * Lay::TILE;
            constexpr int CH = D / 16;
            if (row < p.L) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    p.q + ((static_cast<int64_t>(b) * p.L + row) * p.h_q + headk) * D);
                const float4* csr = reinterpret_cast<const float4*>(p.cs + static_cast<int64_t>(row) * (D / 2));
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const uint4 x = __ldg(src + c);
                    const uint4 y = __ldg(src + c + CH);
                    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
                    const uint32_t ys[4] = {y.x, y.y, y.z, y.w};
                    uint32_t xo[4], yo[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const float4 t2 = __ldg(csr + 4 * c + w);   // (cos, sin) for pairs 8c+2w, 8c+2w+1
                        float a0, b0, a1, b1;
                        rope_rotate(bf16lo_to_f32(xs[w]), bf16lo_to_f32(ys[w]), t2.x, t2.y, a0, b0);
                        rope_rotate(bf16hi_to_f32(xs[w]), bf16hi_to_f32(ys[w]), t2.z, t2.w, a1, b1);
                        xo[w] = pack_bf16x2(a0, a1);
                        yo[w] = pack_bf16x2(b0, b1);
                    }
                    *reinterpret_cast<uint4*>(qs + swz_off(r, c)) = make_uint4(xo[0], xo[1], xo[2], xo[3]);
                    *reinterpret_cast<uint4*>(qs + swz_off(r, c + CH)) = make_uint4(yo[0], yo[1], yo[2], yo[3]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 2 * CH; ++c) *reinterpret_cast<uint4*>(qs + swz_off(r, c)) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            mbar_arrive(&sh.q_full[k]);

            // ---- main loop over key tiles
            const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
            const uint32_t t_s = tmem + lane_base + static_cast<uint32_t>(k * 128);
            const uint32_t t_o = tmem + lane_base + static_cast<uint32_t>(256 + k * D);
            const float sl2 = p.scale_log2;
            float m_run = -INFINITY, l_run = 0.f;
            bool ok = true;
            for (int j = 0; j < nk; ++j) {
                ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[k], j & 1, p.err, abort));
                if (!ok) break;
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(t_s + 32 * c, sr[c]);
                tmem_wait_ld();
                float mx = -INFINITY;
                if (j == qtk) {   // diagonal tile: key column c sits at the same offset as query row r
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            if (32 * c + e > r) sr[c][e] = __float_as_uint(-INFINITY);
                            mx = fmaxf(mx, __uint_as_float(sr[c][e]));
                        }
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(sr[c][e]));
                }
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
                float sum = 0.f;
                // P chunk c (16 columns of bf16 pairs) overwrites S columns 16c.., already in registers.
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float p0 = ex2(fmaf(__uint_as_float(sr[c][e]), sl2, neg_m));
                        const float p1 = ex2(fmaf(__uint_as_float(sr[c][e + 1]), sl2, neg_m));
                        sum += p0 + p1;
                        pk[e >> 1] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(t_s + 16 * c, pk);
                }
                l_run += sum;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sh.p_full[k]);
            }
            // ---- epilogue: O / l -> bf16 -> out[b, row, head, :]
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sh.o_full[k], (nk - 1) & 1, p.err, abort));
            if (ok) {
                tc_fence_after();
                const float inv_l = 1.0f / l_run;
                uint4* dst = reinterpret_cast<uint4*>(
                    p.out + ((static_cast<int64_t>(b) * p.L + row) * p.h_q + headk) * D);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(t_o + 32 * c, o);
                    tmem_wait_ld();
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
                    if (row < p.L) {
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[4 * c + v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
                    }
                }
            }
        }
    } else if (warp == WARP_TMA) {
        // ================================================================ TMA producer
        if (lane == 0 && nmax > 0) {
            const uint32_t tile_bytes = static_cast<uint32_t>(BN * D * 2);
            const int kv_plane = b * p.h_kv + u;
            int issued_k = 0, issued_v = 0;
            for (int j = 0; j < nmax; ++j) {
                const int ks = j % KSTAGES;
                if (j >= KSTAGES && !mbar_wait(&sh.k_empty[ks], ((j / KSTAGES) - 1) & 1, p.err, abort)) break;
                mbar_arrive_expect_tx(&sh.k_full[ks], tile_bytes);
                uint8_t* kdst = smem + Lay::K0 + ks * Lay::TILE;
#pragma unroll
                for (int h = 0; h < D / 64; ++h) tma_load_3d(kdst + h * Lay::SUB, &tm_k, &sh.k_full[ks], h * 64, j * BN, kv_plane);
                issued_k = j + 1;
                const int vs = j % VSTAGES;
                if (j >= VSTAGES && !mbar_wait(&sh.v_empty[vs], ((j / VSTAGES) - 1) & 1, p.err, abort)) break;
                mbar_arrive_expect_tx(&sh.v_full[vs], tile_bytes);
                uint8_t* vdst = smem + Lay::V0 + vs * Lay::TILE;
#pragma unroll
                for (int h = 0; h < D / 64; ++h) tma_load_4d(vdst + h * Lay::SUB, &tm_v, &sh.v_full[vs], h * 64, u, j * BN, b);
                issued_v = j + 1;
            }
            // Drain: never leave the CTA with copies still landing in its shared memory.
            for (int j = (issued_k > KSTAGES ? issued_k - KSTAGES : 0); j < issued_k; ++j)
                mbar_wait(&sh.k_full[j % KSTAGES], (j / KSTAGES) & 1, p.err, nullptr);
            for (int j = (issued_v > VSTAGES ? issued_v - VSTAGES : 0); j < issued_v; ++j)
                mbar_wait(&sh.v_full[j % VSTAGES], (j / VSTAGES) & 1, p.err, nullptr);
        }
    } else if (warp == WARP_MMA) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
            const uint32_t q_addr0 = smem_u32(smem + Lay::Q0);
            const uint32_t k_addr0 = smem_u32(smem + Lay::K0);
            const uint32_t v_addr0 = smem_u32(smem + Lay::V0);
            bool ok = nmax > 0;
            const int n[2] = {n0, n1};
            for (int k = 0; k < 2 && ok; ++k)
                if (n[k] > 0) ok = mbar_wait(&sh.q_full[k], 0, p.err, abort);
            // S_k = Q_k K_j^T : M=128 (query rows), N=128 (key rows), K=D in steps of 16.
            auto issue_s = [&](int k, int ks) {
                const uint32_t qa = q_addr0 + k * Lay::TILE;
                const uint32_t ka = k_addr0 + ks * Lay::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = static_cast<uint32_t>((kk >> 2) * Lay::SUB + (kk & 3) * 32);
                    umma_ss(tmem + static_cast<uint32_t>(k * 128), sw128_desc(qa + off, 16, 1024),
                            sw128_desc(ka + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
                }
            };
            // O_k += P_k V_j : M=128, N=D (V is MN-major: d contiguous), K=128 key rows in steps of 16.
            auto issue_pv = [&](int k, int vs, bool acc) {
                const uint32_t va = v_addr0 + vs * Lay::TILE;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    umma_ts(tmem + static_cast<uint32_t>(256 + k * D), tmem + static_cast<uint32_t>(k * 128 + kk * 8),
                            sw128_desc(va + kk * 16 * 128, Lay::SUB, 1024), IDESC_PV, (acc || kk > 0) ? 1u : 0u);
                }
            };
            if (ok) ok = mbar_wait(&sh.k_full[0], 0, p.err, abort);
            if (ok) {
                tc_fence_after();
                for (int k = 0; k < 2; ++k)
                    if (n[k] > 0) {
                        issue_s(k, 0);
                        umma_commit(&sh.s_full[k]);
                    }
                umma_commit(&sh.k_empty[0]);
                for (int j = 0; j < nmax && ok; ++j) {
                    const int vs = j % VSTAGES;
                    ok = mbar_wait(&sh.v_full[vs], (j / VSTAGES) & 1, p.err, abort);
                    if (!ok) break;
                    bool k_next = false;
                    for (int k = 0; k < 2 && ok; ++k) {
                        if (j >= n[k]) continue;
                        ok = mbar_wait(&sh.p_full[k], j & 1, p.err, abort);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(k, vs, j > 0);
                        umma_commit(&sh.o_full[k]);
                        if (j + 1 < n[k]) {
                            const int ks = (j + 1) % KSTAGES;
                            if (!k_next) {
                                ok = mbar_wait(&sh.k_full[ks], ((j + 1) / KSTAGES) & 1, p.err, abort);
                                if (!ok) break;
                                tc_fence_after();
                                k_next = true;
                            }
                            issue_s(k, ks);
                            umma_commit(&sh.s_full[k]);
                        }
                    }
                    umma_commit(&sh.v_empty[vs]);
                    if (k_next) umma_commit(&sh.k_empty[(j + 1) % KSTAGES]);
                }
            }
            // Every MMA must have finished before the tensor memory is released.
            umma_commit(&sh.mma_done);
            mbar_wait(&sh.mma_done, 0, p.err, nullptr);
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

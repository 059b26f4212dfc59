// Fused QKV projection + bias + RoPE on sm_100a (page "Qwen2 architecture introduction",
// aicoding.csdn.net, §4.1.3 steps 1-3): Y = X W^T + b for the stacked weight W = [W_Q^T; W_K^T; W_V^T]
// ([(h_q + 2 h_kv) d, d_model], the nn.Linear layout), split into heads; Q and K heads are rotated at
// their positions.  One pass writes everything the attention step and the KV cache need:
//   qr [B, h_q,  L, d]  rotated Q, head-major (the attention kernel's Q' layout)
//   kr [B, h_kv, L, d]  rotated K, head-major (its K' layout)
//   k  [B, L, h_kv, d]  raw K, token-major: the packed cache rows of the sequences, back to back
//                       (the rotated K instead for caches that keep keys after RoPE, p.k_rotated)
//   v  [B, L, h_kv, d]  V, token-major (cache rows; the attention kernel reads V in this layout)
//
// qkv_kernel is a persistent tcgen05 GEMM, one CTA per SM, over 128 x 256 output tiles (128 tokens,
// 256 output columns = 2 heads of d = 128 or 4 of d = 64); proj_kernel is the same GEMM with the output
// projection's epilogue (+ residual, page §4.1.3 steps 5-6):
//   warp 0     TMA producer: 64-wide K blocks of X (128 x 64) and W (256 x 64) into a 4-stage ring
//   warp 1     MMA issuer: 4 x tcgen05.mma M128 N256 K16 per K block into one of two TMEM accumulators
//   warps 2-5  epilogue: one TMEM lane (token row) per thread; per head: + bias, rotate, round, and
//              store through a per-warp shared-memory staging buffer as whole rows
// The two accumulators (2 x 256 TMEM columns) let the epilogue of one tile overlap the main loop of the
// next.  cos / sin come from a per-position table built once per (L, d, theta).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "rope.cuh"
#include "sm100_ptx.cuh"

namespace gqa {
namespace qkv {

using namespace ptx;

constexpr int BM = 128;                  // tokens per tile (MMA M, TMEM lanes)
constexpr int BK = 64;                   // K block: one 128-byte swizzle atom of bf16
constexpr int NUM_THREADS = 192;
constexpr int WARP_TMA = 0, WARP_MMA = 1;
constexpr int A_BYTES = BM * BK * 2;     // 16 KB
constexpr int EPI_WARPS = 4;
constexpr int STAGING = 32 * 128 * 2;    // one epilogue warp's 32 rows of up to 128 bf16
constexpr int RING_BYTES = 192 * 1024;   // the K-block ring
constexpr int MAX_STAGES = 6;
constexpr int TABLE_THREADS = 256;

// Tile width BN (MMA N).  256 columns (a 4-stage ring) is what the kernels are launched with: measured
// on the Qwen2-7B projections, 128-column tiles (a 6-stage ring) were slower even where they would fill
// the last wave of CTAs better -- twice the K-block traffic per FLOP and a shorter main loop to hide each
// epilogue behind.
template <int BN_>
struct Tile {
    static constexpr int BN = BN_;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = RING_BYTES / STAGE_BYTES;
    static constexpr int DYN = STAGES * STAGE_BYTES + EPI_WARPS * STAGING + 1024;
    static constexpr int TMEM_COLS = 2 * BN;   // two accumulators
    static_assert(STAGES <= MAX_STAGES, "ring deeper than the barrier arrays");
};

struct Params {
    const __nv_bfloat16* bias;   // [N] or nullptr
    const float2* tab;           // [L, d/2] (cos, sin) of pos * theta^(-2i/d)
    __nv_bfloat16* qr;
    __nv_bfloat16* kr;
    __nv_bfloat16* k;
    __nv_bfloat16* v;
    const __nv_bfloat16* resid;  // output projection: residual [T, N] or nullptr
    __nv_bfloat16* out;          // output projection: out [T, N] (may be resid itself)
    // Decode-step append (kAppend): token t is the new token of sequence t, at position seqlens[t]; q goes
    // to qr [T, h_q, d], its K and V rows to the page slot of that position in k / v, the key and value
    // pages [num_pages, page_size, h_kv, d], through the block table bt [T, max_pages].
    const int* seqlens;
    const int* bt;
    int page_size, max_pages, num_pages;
    // The caches keep their keys after RoPE: qkv's k output and the append's key rows are written rotated
    // (the append at position seqlens[t], with `rope` and the YaRN temperature `mscale`).
    int k_rotated;
    RopeSpec rope;
    float mscale;
    int T, L, N, h_q, h_kv;
    int n_ntiles, n_tiles, kblocks;
    // Work units: tiles 0 .. n_main-1 whole (BN columns); each later tile split into tail_split units of
    // BN / tail_split columns, so that a last wave with few tiles is spread over more CTAs.  n_units in all.
    int n_main, tail_split, n_units;
    int* err;
};

// Columns of a tail unit (MMA N); its weight rows come through a tensor map whose box is this high.
// A tail unit's K block (A + its weight rows) fills a fraction of a ring stage, so each stage carries
// several consecutive K blocks of it, back to back: the unit keeps as many bytes in flight as a whole
// tile (its loads, not its MMAs, bound it).
constexpr int TAIL_BN = 64;
constexpr int TAIL_KB_BYTES = A_BYTES + TAIL_BN * BK * 2;   // 24 KB

// Rows [mt * BM, +BM) and columns [n0, n0 + width) of work unit u.
struct Unit {
    int mt, n0, width;
};
template <int BN, bool TAIL>
__device__ __forceinline__ Unit unit_of(const Params& p, int u) {
    Unit r;
    if (!TAIL || u < p.n_main) {
        r.mt = u / p.n_ntiles;
        r.n0 = (u % p.n_ntiles) * BN;
        r.width = BN;
    } else {
        const int v = u - p.n_main;
        const int tile = p.n_main + v / p.tail_split;
        r.mt = tile / p.n_ntiles;
        r.width = BN / p.tail_split;
        r.n0 = (tile % p.n_ntiles) * BN + (v % p.tail_split) * r.width;
    }
    return r;
}

struct alignas(8) Shared {
    uint64_t full[MAX_STAGES], empty[MAX_STAGES];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

// ---------------------------------------------------------------------------------------------
// The cos / sin table: tab[pos * d/2 + i] = mscale * (cos, sin)(pos * f_i), f_i = rope_freq (theta^(-2i/d),
// YaRN-scaled if enabled), the angle formed in double precision (rope_cossin).
template <int D>
__global__ void __launch_bounds__(TABLE_THREADS) rope_table_kernel(float2* __restrict__ tab, int L,
                                                                   RopeSpec rope, float mscale) {
    constexpr int H = D / 2;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * TABLE_THREADS + threadIdx.x;
    if (e >= static_cast<int64_t>(L) * H) return;
    const int pos = static_cast<int>(e / H), i = static_cast<int>(e % H);
    float c, s;
    rope_cossin(static_cast<double>(pos), rope_freq(i, D, rope), c, s);
    tab[e] = make_float2(c * mscale, s * mscale);   // YaRN temperature on Q and K (1 without scaling)
}

// ---------------------------------------------------------------------------------------------
// One head (D columns starting at n0) of one token row, in place: + bias, rotate if Q or K, round, store.
// One output row per lane (dst, nullptr for a row past the end), D values in z: round to bf16 and store the
// warp's 32 rows through its shared-memory staging buffer, so that each global store instruction writes
// whole rows (D * 2 bytes each) instead of one 16-byte piece of 32 different rows.  Chunk c of row r is
// staged at chunk position c ^ (r mod CH): writing (one row per lane) and reading (CH lanes per row) are
// both free of bank conflicts.
template <int D>
__device__ __forceinline__ void store_rows(uint8_t* stage, __nv_bfloat16* dst, const float* z, int lane) {
    constexpr int CH = D / 8;             // 16-byte chunks per row
    constexpr int RPI = 32 / CH;          // rows per store instruction
    uint4* st = reinterpret_cast<uint4*>(stage);
#pragma unroll
    for (int c = 0; c < CH; ++c)
        st[lane * CH + (c ^ (lane & (CH - 1)))] =
            make_uint4(pack_bf16x2(z[8 * c], z[8 * c + 1]), pack_bf16x2(z[8 * c + 2], z[8 * c + 3]),
                       pack_bf16x2(z[8 * c + 4], z[8 * c + 5]), pack_bf16x2(z[8 * c + 6], z[8 * c + 7]));
    __syncwarp();
    const uint64_t mine = reinterpret_cast<uint64_t>(dst);
    const int c = lane % CH;
#pragma unroll
    for (int j = 0; j < 32 / RPI; ++j) {
        const int r = j * RPI + lane / CH;
        const uint64_t row = __shfl_sync(0xffffffffu, mine, r);
        const uint4 val = st[r * CH + (c ^ (r & (CH - 1)))];
        if (row) reinterpret_cast<uint4*>(row)[c] = val;
    }
    __syncwarp();   // the buffer is reused by the next call
}

// One head (D columns starting at n0) of one token row per lane, in place: + bias, rotate if Q or K, then
// the row goes to its output(s).  Lanes with valid == false (rows past the end) take part without storing.
template <int D>
__device__ __forceinline__ void store_head(const Params& p, float (&y)[D], int n0, int b, int pos, bool valid,
                                           uint8_t* stage, int lane) {
    constexpr int H = D / 2;
    if (p.bias) {
        const uint4* bb = reinterpret_cast<const uint4*>(p.bias + n0);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 w = bb[c];
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                y[8 * c + 2 * e] += bf16lo_to_f32(ws[e]);
                y[8 * c + 2 * e + 1] += bf16hi_to_f32(ws[e]);
            }
        }
    }
    const int head = n0 / D;
    // Rotation pairs (i, i + H): the (cos, sin) of a row's H frequencies are read from the table in
    // chunks of 16 frequencies (8 float4), the next chunk's loads issued before the current chunk is
    // rotated, so at most two chunks are live in registers beside the row.
    constexpr int CHUNK = 16;
    constexpr int NCH = H / CHUNK;
    const float4* trow = reinterpret_cast<const float4*>(p.tab + static_cast<int64_t>(pos) * H);
    auto rotate = [&](float* z) {
        float4 tb[2][CHUNK / 2];
#pragma unroll
        for (int c = 0; c < CHUNK / 2; ++c) tb[0][c] = trow[c];
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
            if (ch + 1 < NCH) {
#pragma unroll
                for (int c = 0; c < CHUNK / 2; ++c) tb[(ch + 1) & 1][c] = trow[(ch + 1) * (CHUNK / 2) + c];
            }
#pragma unroll
            for (int c = 0; c < CHUNK / 2; ++c) {
                const float4 cs = tb[ch & 1][c];   // (cos, sin) of frequencies i and i + 1
                const int i = ch * CHUNK + 2 * c;
                float a0, b0, a1, b1;
                rope_rotate(z[i], z[i + H], cs.x, cs.y, a0, b0);
                rope_rotate(z[i + 1], z[i + 1 + H], cs.z, cs.w, a1, b1);
                z[i] = a0;
                z[i + H] = b0;
                z[i + 1] = a1;
                z[i + 1 + H] = b1;
            }
        }
    };
    auto row_of = [&](__nv_bfloat16* base, int64_t idx) { return valid ? base + idx * D : nullptr; };
    if (head < p.h_q) {
        rotate(y);
        store_rows<D>(stage, row_of(p.qr, (static_cast<int64_t>(b) * p.h_q + head) * p.L + pos), y, lane);
    } else if (head < p.h_q + p.h_kv) {
        const int u = head - p.h_q;
        if (p.k_rotated) rotate(y);   // the cache rows keep the key after RoPE
        store_rows<D>(stage, row_of(p.k, (static_cast<int64_t>(b) * p.L + pos) * p.h_kv + u), y, lane);
        if (!p.k_rotated) rotate(y);
        store_rows<D>(stage, row_of(p.kr, (static_cast<int64_t>(b) * p.h_kv + u) * p.L + pos), y, lane);
    } else {
        const int u = head - p.h_q - p.h_kv;
        store_rows<D>(stage, row_of(p.v, (static_cast<int64_t>(b) * p.L + pos) * p.h_kv + u), y, lane);
    }
}

// The output projection's epilogue: W columns of one row per lane, + the residual, stored as rows.
// The residual is read directly, each thread its own row: measured faster than reading whole rows
// through the staging buffer, whose round trip sits on the epilogue's critical path.
template <int W>
__device__ __forceinline__ void store_resid(const Params& p, float (&y)[W], int n0, int t, bool valid,
                                            uint8_t* stage, int lane) {
    const int64_t at = static_cast<int64_t>(t) * p.N + n0;
    if (p.resid && valid) {
        const uint4* rr = reinterpret_cast<const uint4*>(p.resid + at);
#pragma unroll
        for (int c = 0; c < W / 8; ++c) {
            const uint4 w = rr[c];
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                y[8 * c + 2 * e] += bf16lo_to_f32(ws[e]);
                y[8 * c + 2 * e + 1] += bf16hi_to_f32(ws[e]);
            }
        }
    }
    store_rows<W>(stage, valid ? p.out + at : nullptr, y, lane);
}

// The decode-step append's epilogue: one head of one token row per lane, + bias, stored un-rotated (the
// decode rotates q and every cached key at its position): a query head to its q row, a key or value head
// to the token's page slot (kv_row: the slot's row of h_kv heads in the key or value pages, nullptr when
// the row is past the end or its table entry is invalid).  Where the caches keep keys after RoPE
// (p.k_rotated), a key head is rotated at the token's position `at` first.
template <int D>
__device__ __forceinline__ void store_append(const Params& p, float (&y)[D], int n0, int t, int at, bool valid,
                                             __nv_bfloat16* k_row, __nv_bfloat16* v_row, uint8_t* stage, int lane) {
    if (p.bias) {
        const uint4* bb = reinterpret_cast<const uint4*>(p.bias + n0);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const uint4 w = bb[c];
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                y[8 * c + 2 * e] += bf16lo_to_f32(ws[e]);
                y[8 * c + 2 * e + 1] += bf16hi_to_f32(ws[e]);
            }
        }
    }
    const int head = n0 / D;
    if (p.k_rotated && head >= p.h_q && head < p.h_q + p.h_kv && k_row) {
#pragma unroll
        for (int i = 0; i < D / 2; ++i) {
            float c, s;
            rope_cossin(static_cast<double>(at), rope_freq(i, D, p.rope), c, s);
            float xr, yr;
            rope_rotate(y[i], y[i + D / 2], c * p.mscale, s * p.mscale, xr, yr);
            y[i] = xr;
            y[i + D / 2] = yr;
        }
    }
    __nv_bfloat16* dst;
    if (head < p.h_q) dst = valid ? p.qr + (static_cast<int64_t>(t) * p.h_q + head) * D : nullptr;
    else if (head < p.h_q + p.h_kv) dst = k_row ? k_row + static_cast<int64_t>(head - p.h_q) * D : nullptr;
    else dst = v_row ? v_row + static_cast<int64_t>(head - p.h_q - p.h_kv) * D : nullptr;
    store_rows<D>(stage, dst, y, lane);
}

enum Epilogue { kQKV = 0, kResidual = 1, kAppend = 2 };

// ---------------------------------------------------------------------------------------------
// The persistent GEMM: Y[T, N] = X[T, K] W[N, K]^T with the epilogue EPI.  For kQKV and kAppend, D is the
// head size (tiles are processed head by head); for kResidual, D = 128 (128 columns at a time).
template <int D, int EPI, int BN_>
__device__ __forceinline__ void gemm_body(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const CUtensorMap& tm_wt,
                                          const Params& p) {
    constexpr int BN = Tile<BN_>::BN;
    constexpr int STAGES = Tile<BN_>::STAGES;
    constexpr int STAGE_BYTES = Tile<BN_>::STAGE_BYTES;
    constexpr int TMEM_COLS = Tile<BN_>::TMEM_COLS;
    constexpr int TAIL_PER_STAGE = STAGE_BYTES / TAIL_KB_BYTES;   // K blocks of a tail unit per stage
    static_assert(TAIL_PER_STAGE >= 1, "a tail K block fits a stage");
    extern __shared__ uint8_t dyn_smem_raw[];
    __shared__ Shared sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.acc_full[b], 1);
            mbar_init(&sh.acc_empty[b], 4 * 32);
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
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_w);
        if (p.tail_split > 1) prefetch_tensormap(&tm_wt);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int* abort = &sh.abort;

    if (warp == WARP_TMA) {
        // ================================================================ TMA producer
        if (lane == 0) {
            uint32_t it = 0;   // K blocks issued (ring position)
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.n_units; u += gridDim.x) {
                const Unit un = unit_of<BN, EPI == kResidual>(p, u);
                if (un.width == BN) {
                    for (int kb = 0; kb < p.kblocks; ++kb) {
                        const int s = static_cast<int>(it % STAGES);
                        if (it >= STAGES && !mbar_wait(&sh.empty[s], ((it / STAGES) - 1) & 1, p.err, abort)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&sh.full[s], STAGE_BYTES);
                        uint8_t* a = smem + s * STAGE_BYTES;
                        tma_load_2d(a, &tm_x, &sh.full[s], kb * BK, un.mt * BM);
                        tma_load_2d(a + A_BYTES, &tm_w, &sh.full[s], kb * BK, un.n0);
                        ++it;
                    }
                } else {
                    for (int kb = 0; kb < p.kblocks; kb += TAIL_PER_STAGE) {
                        const int s = static_cast<int>(it % STAGES);
                        if (it >= STAGES && !mbar_wait(&sh.empty[s], ((it / STAGES) - 1) & 1, p.err, abort)) {
                            ok = false;
                            break;
                        }
                        const int nk = kb + TAIL_PER_STAGE <= p.kblocks ? TAIL_PER_STAGE : p.kblocks - kb;
                        mbar_arrive_expect_tx(&sh.full[s], static_cast<uint32_t>(nk * TAIL_KB_BYTES));
                        for (int q = 0; q < nk; ++q) {
                            uint8_t* a = smem + s * STAGE_BYTES + q * TAIL_KB_BYTES;
                            tma_load_2d(a, &tm_x, &sh.full[s], (kb + q) * BK, un.mt * BM);
                            tma_load_2d(a + A_BYTES, &tm_wt, &sh.full[s], (kb + q) * BK, un.n0);
                        }
                        ++it;
                    }
                }
            }
            // Never leave the CTA with copies still landing in its shared memory.
            for (uint32_t j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
                mbar_wait(&sh.full[j % STAGES], (j / STAGES) & 1, p.err, nullptr);
        }
    } else if (warp == WARP_MMA) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_WHOLE = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t IDESC_TAIL = idesc_bf16_f32(BM, TAIL_BN, false);
            const uint32_t base = smem_u32(smem);
            uint32_t it = 0;
            int local = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.n_units; u += gridDim.x, ++local) {
                const bool whole = unit_of<BN, EPI == kResidual>(p, u).width == BN;
                const int buf = local & 1;
                // The epilogue must have read this accumulator out (two tiles ago) before it is overwritten.
                if (local >= 2 && !mbar_wait(&sh.acc_empty[buf], ((local >> 1) - 1) & 1, p.err, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * BN);
                if (whole) {
                    for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
                        const int s = static_cast<int>(it % STAGES);
                        if (!mbar_wait(&sh.full[s], (it / STAGES) & 1, p.err, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_addr = base + static_cast<uint32_t>(s * STAGE_BYTES);
                        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            umma_ss(d_tmem, sw128_desc(a_addr + kk * 32, 16, 1024),
                                    sw128_desc(b_addr + kk * 32, 16, 1024), IDESC_WHOLE, (kb > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&sh.empty[s]);
                    }
                } else {
                    for (int kb = 0; kb < p.kblocks; kb += TAIL_PER_STAGE, ++it) {
                        const int s = static_cast<int>(it % STAGES);
                        if (!mbar_wait(&sh.full[s], (it / STAGES) & 1, p.err, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const int nk = kb + TAIL_PER_STAGE <= p.kblocks ? TAIL_PER_STAGE : p.kblocks - kb;
                        for (int q = 0; q < nk; ++q) {
                            const uint32_t a_addr =
                                base + static_cast<uint32_t>(s * STAGE_BYTES + q * TAIL_KB_BYTES);
                            const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                            for (int kk = 0; kk < BK / 16; ++kk)
                                umma_ss(d_tmem, sw128_desc(a_addr + kk * 32, 16, 1024),
                                        sw128_desc(b_addr + kk * 32, 16, 1024), IDESC_TAIL,
                                        (kb + q > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(&sh.empty[s]);
                    }
                }
                if (!ok) break;
                umma_commit(&sh.acc_full[buf]);
            }
            // Every MMA must have finished before the tensor memory is released.
            umma_commit(&sh.mma_done);
            mbar_wait(&sh.mma_done, 0, p.err, nullptr);
        }
    } else {
        // ================================================================ epilogue (warps 2..5)
        const int quarter = warp & 3;                       // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;                  // token row within the tile
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        uint8_t* stage = smem + STAGES * STAGE_BYTES + (warp - 2) * STAGING;
        int local = 0;
        for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++local) {
            const int buf = local & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sh.acc_full[buf], (local >> 1) & 1, p.err, abort))) break;
            tc_fence_after();
            const Unit un = unit_of<BN, EPI == kResidual>(p, u);
            const int t = un.mt * BM + r;
            const bool valid = t < p.T;
            const int b = valid ? t / p.L : 0, pos = valid ? t % p.L : 0;
            // kAppend: this row's page slot (rows of all h_kv heads) in the key and value pages
            __nv_bfloat16 *k_row = nullptr, *v_row = nullptr;
            int at = 0;
            if (EPI == kAppend && valid) {
                at = __ldg(p.seqlens + t);
                const int pi = at >= 0 ? at / p.page_size : -1;
                const int page = (pi >= 0 && pi < p.max_pages) ? __ldg(p.bt + static_cast<int64_t>(t) * p.max_pages + pi) : -1;
                if (page >= 0 && page < p.num_pages) {
                    const int64_t slot = static_cast<int64_t>(page) * p.page_size + (at - pi * p.page_size);
                    k_row = p.k + slot * p.h_kv * D;
                    v_row = p.v + slot * p.h_kv * D;
                } else if (un.n0 == 0) {
                    atomicOr(p.err, kErrBadPage);   // once per row: nothing of this token is cached
                }
            }
            if (EPI == kResidual && un.width == TAIL_BN) {
                // A tail unit (output projection only): its 64 columns in one pass.
                if (un.n0 < p.N) {
                    float acc[TAIL_BN];
#pragma unroll
                    for (int c = 0; c < TAIL_BN / 32; ++c)
                        tmem_ld32(tmem + lane_base + static_cast<uint32_t>(buf * BN + 32 * c),
                                  *reinterpret_cast<uint32_t(*)[32]>(acc + 32 * c));
                    tmem_wait_ld();
                    store_resid<TAIL_BN>(p, acc, un.n0, t, valid, stage, lane);
                }
            } else {
#pragma unroll 1
                for (int hh = 0; hh < BN / D; ++hh) {
                    const int n0 = un.n0 + hh * D;
                    if (n0 >= p.N) break;
                    float acc[D];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c)
                        tmem_ld32(tmem + lane_base + static_cast<uint32_t>(buf * BN + hh * D + 32 * c),
                                  *reinterpret_cast<uint32_t(*)[32]>(acc + 32 * c));
                    tmem_wait_ld();
                    if (EPI == kQKV) store_head<D>(p, acc, n0, b, pos, valid, stage, lane);
                    else if (EPI == kAppend) store_append<D>(p, acc, n0, t, at, valid, k_row, v_row, stage, lane);
                    else store_resid<128>(p, *reinterpret_cast<float(*)[128]>(acc), n0, t, valid, stage, lane);
                }
            }
            // This thread's reads of the accumulator are complete: release it to the MMA warp.
            tc_fence_before();
            mbar_arrive(&sh.acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int D, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    qkv_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_wt, const Params p) {
    gemm_body<D, kQKV, BN>(tm_x, tm_w, tm_wt, p);
}

// One decode step's projection and cache append (page "Qwen2 architecture introduction", §4.1.3 steps 1-2
// and closing paragraph: the current token's K and V are appended to the cache each step): x [T, d_model]
// holds the new token of T sequences; q [T, h_q, D] and the page slots of positions seqlens[t] get the
// un-rotated heads.
template <int D, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    append_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  const __grid_constant__ CUtensorMap tm_wt, const Params p) {
    gemm_body<D, kAppend, BN>(tm_x, tm_w, tm_wt, p);
}

// Output projection + residual (page "Qwen2 architecture introduction", §4.1.3 steps 5-6):
// out = attn W_O + X_in, with attn the concatenated heads [T, h_q d] and W_O^T [d_model, h_q d].
template <int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    proj_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ CUtensorMap tm_wt, const Params p) {
    gemm_body<128, kResidual, BN>(tm_x, tm_w, tm_wt, p);
}

}  // namespace qkv
}  // namespace gqa
